// gemm_sm100.cuh - grouped bf16 GEMM engine on the 5th-generation tensor core.
//
//   C[r, n] = sum_k A[r, k] * B_g[n, k]      for every row r of group g
//
// A is a (rows, K) row-major bf16 matrix whose rows are grouped by expert
// (group g owns rows offsets[g] .. offsets[g+1]-1; group sizes are known only on
// the device). B_g is expert g's (N, K) row-major bf16 weight, i.e. K-major, as
// the layer stores W1/W3 (f, d) and W2 (d, f) ("Shared Expert (DeepSeek-V3)",
// "How it works", SwiGLU definition). A dense GEMM is the special case of one
// group holding every row (the shared expert and the router).
//
// Design (sm_100a):
//  * persistent: one CTA per SM walks a linear tile list; tile t maps to
//    (group, n-block, m-block) through a device prefix of per-group m-tile
//    counts, so no host synchronisation is needed to learn the group sizes;
//    within a group the m-blocks are innermost so the CTAs running at the same
//    time share one weight tile through L2;
//  * warps 0 and 6: TMA producers taking alternate stages of a kStages-deep
//    shared-memory ring guarded by full/empty mbarriers (128B-swizzled boxes,
//    no cluster multicast); the CTA-pair kernel has warp 0 only;
//  * warp 1: allocates 512 TMEM columns, one thread issues
//    tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16) and commits; a
//    tile that owns at most 64 rows (a small expert group) uses M=64 instead,
//    halving the tensor work spent on rows that are masked anyway;
//  * warps 2..5: epilogue, each owns one 32-lane quarter of TMEM; two
//    256-column accumulators let the epilogue of tile i overlap the MMAs of
//    tile i+1;
//  * epilogues: SwiGLU (the 256 accumulator columns are 128 gate columns from
//    W1 followed by the same 128 columns of W3; writes SiLU(gate)*up as bf16),
//    plain bf16, plain fp32. Rows past the group's end and columns past N are
//    masked, so partial tiles never write outside their group.
#pragma once

#include "ptx_sm100.cuh"

namespace moe {

constexpr int kBM = 128;                       // tile rows (MMA M)
constexpr int kBN = 256;                       // accumulator columns (MMA N)
constexpr int kBK = 64;                        // K per stage: one 128-byte swizzle row
constexpr int kUK = 16;                        // K per tcgen05.mma (kind::f16)
constexpr int kStages = 4;
constexpr int kATileBytes = kBM * kBK * 2;     // 16 KB
constexpr int kBHalfBytes = 128 * kBK * 2;     // 16 KB (one 128-row TMA box)
constexpr int kBTileBytes = kBN * kBK * 2;     // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kNumAcc = 2;
constexpr int kMaxGroups = 1024;               // expert groups a grouped launch may have
constexpr int kTmemCols = kNumAcc * kBN;       // 512: the whole TMEM of the SM
// Single-CTA kernel: warps 0 and 6 are TMA producers taking alternate stages,
// warp 1 issues MMAs, warps 2..5 run the epilogue. Measured on B200 with
// per-role cycle counters: one producer thread spends ~400 cycles per stage
// issuing its three TMA loads (the expect-tx arrive is ~60), against 512
// cycles of MMAs per stage, so a single producer left the tensor pipe waiting.
// The CTA-pair kernel issues two loads per CTA per stage and keeps one producer.
constexpr int kGemmThreads = 224;
constexpr int kProducer2Warp = 6;
constexpr int kPairThreads = 192;
constexpr int kEpiThreads = 128;

enum EpiMode : int { kEpiSwiGLU = 0, kEpiBF16 = 1, kEpiF32 = 2 };

// Output columns one tile produces.
__host__ __device__ constexpr int tile_cols(int mode) { return mode == kEpiSwiGLU ? 128 : 256; }

struct GemmParams {
  const int* group_offsets;  // device (num_groups+1); nullptr: one dense group of dense_rows
  const int* group_mtiles;   // device (num_groups+1) exclusive prefix of ceil(n_g / tile rows)
  // Optional second class of groups (nullptr: one class). With it, group_mtiles
  // counts only the groups of class A (the others contribute 0) and
  // group_mtiles_b only those of class B; the tiles of class A are spread
  // evenly over the launch, those of class B fill the positions between them.
  const int* group_mtiles_b;
  int num_groups;
  int dense_rows;
  int K;                     // reduction length (elements)
  int N;                     // valid output columns
  int n_tiles;               // ceil(N / tile_cols(mode))
  void* out;                 // bf16 or fp32, row-major
  long long ldo;             // elements between output rows
  int* status;               // device status word (moe_status codes)
  int k_splits;              // split-K factor (fp32 epilogue only; 1 elsewhere): split s
  int kb_per_split;          //   covers k-blocks [s*kb_per_split, ...) and writes its
  long long split_stride;    //   partial sums at out + s*split_stride
  // Optional extra dense problem run by the same launch (the shared expert):
  // x_tiles tiles spread evenly among the grouped tiles, A/B from the kernel's
  // second set of tensor maps.
  int x_tiles;               // 0: none
  int x_rows, x_K, x_N;
  void* x_out;
  long long x_ldo;
  int x_out_f32;             // plain epilogue: store fp32 instead of bf16
  // Test hook (0 in normal use): CTA 0 of the single-CTA kernel withholds the
  // loads of its first stage, so that its MMA warp's bounded wait expires and
  // the kernel takes its timeout path (status word, drain, TMEM release).
  int test_withhold;
  // Optional row gather for the grouped A operand (single-CTA kernel, grouped
  // launches without an extra problem): grouped row g of the A operand is row
  // gather_src[g] of gather_x (T rows of gather_ld_vec 16-byte vectors),
  // copied by the producer warps with cp.async instead of a TMA box of a
  // permuted copy; nullptr: A through its tensor map.
  const uint4* gather_x;
  const int* gather_src;
  int gather_ld_vec;
  int gather_T;              // rows of gather_x: a source row outside [0, T) reads zeros
};

// 16-byte copy global -> shared through the load/store path; src_bytes 0
// fills the 16 bytes with zeros (rows past a group, columns past K).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed (the
// arrival is counted in the barrier's expected count, not added to it).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// Order this thread's view of generic-proxy shared-memory writes (cp.async)
// before its later async-proxy operations (tcgen05.mma reading shared memory).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Single-CTA kernel shapes: BN accumulator columns per tile (MMA N), TM rows
// per tile. BN = 256, TM = 128 is the default in every regime: each MMA
// instruction then carries the most weight bytes, and on B200 an instruction
// costs about the same issue time whatever its size. The options: narrower
// tiles - SwiGLU BN = 128 (64 gate + 64 up columns, 64 output columns) or
// BN = 64 (32 output columns), plain BN = 128 - split a launch into more,
// shorter tiles; TM = 64 (M=64 MMAs, 64-row boxes of the grouped rows) halves
// the grouped-row bytes per stage, so that the same shared memory holds more
// stages.
// OCC = 2 CTAs resident per SM, each with half the ring and half the TMEM:
// two independent load -> MMA pipelines per SM. A load-only measurement on
// B200 showed one pipeline of 8 KB stages stuck near 30 GB/s per SM (the
// producer thread's issue cost per stage) and two near 6 TB/s in all; with the
// GEMM's 24-48 KB stages one pipeline already streams 6.5 TB/s, and the routed
// GEMMs are instead bound by the SM's MMA issue rate (about 95 cycles per
// tcgen05.mma instruction at any size), which both CTAs share - so OCC = 2 is
// an option, not the default.
template <int BN, int TM = 128, int OCC = 1>
struct SingleCfg {
  static constexpr int kABytes = TM * kBK * 2;                // grouped rows per stage
  static constexpr int kBBytes = BN * kBK * 2;                // weight rows per stage
  static constexpr int kStage = kABytes + kBBytes;
  // as many stages as the ring budget holds, at most 8: with 200 KB 4 x 48 KB,
  // 6 x 32 KB, 8 x 24 KB, 5 x 40 KB; with 96 KB (two CTAs per SM) 2 x 48 KB,
  // 3 x 32 KB, 4 x 24 KB, 2 x 40 KB
  static constexpr int kBudget = OCC == 1 ? 200 * 1024 : 96 * 1024;
  static constexpr int kStages = kBudget / kStage < 8 ? kBudget / kStage : 8;
  static constexpr int kTmemCols = 512 / OCC;                 // this CTA's TMEM columns
  static constexpr int kAcc = kTmemCols / BN;                 // accumulators in TMEM
  static constexpr int kHalfRows = BN / 2;                    // rows of one SwiGLU B box
  // barrier area after the ring: full/empty per stage, tfull/tempty per
  // accumulator, the drain barrier, the TMEM address and the abort flag
  static constexpr int kBarBytes = ((2 * kStages + 2 * kAcc + 1) * 8 + 8 + 127) / 128 * 128;
  static_assert(OCC == 1 || OCC == 2, "one or two CTAs per SM");
  static_assert(kStages >= 2 && kAcc >= 1, "ring and accumulator fit");
};

// Dynamic shared memory the kernel needs for a given number of groups.
template <int BN = 256, int TM = 128, int OCC = 1>
__host__ __device__ constexpr size_t gemm_smem_bytes(int num_groups) {
  return 1024 /* alignment slack */ +
         size_t(SingleCfg<BN, TM, OCC>::kStages) * SingleCfg<BN, TM, OCC>::kStage +
         SingleCfg<BN, TM, OCC>::kBarBytes + size_t(3) * (num_groups + 1) * sizeof(int);
}

struct TileCoord {
  int group, n_blk, row0, rows, split, mtiles;   // mtiles: m-blocks of this tile's group
};

__device__ __forceinline__ TileCoord decode_tile(int tile, const int* s_off, const int* s_mp,
                                                 int num_groups, int n_tiles, int tile_m = kBM) {
  // split-K outermost: tiles of split s follow those of split s-1
  const int per_split = s_mp[num_groups] * n_tiles;
  const int split = tile / per_split;
  tile -= split * per_split;
  // largest g with s_mp[g] * n_tiles <= tile (empty groups share a prefix value,
  // the largest index among them is the next non-empty group)
  int lo = 0, hi = num_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mp[mid] * n_tiles <= tile) lo = mid; else hi = mid;
  }
  const int mt = s_mp[lo + 1] - s_mp[lo];
  const int local = tile - s_mp[lo] * n_tiles;
  const int n_blk = local / mt;
  const int m_blk = local - n_blk * mt;
  TileCoord c;
  c.group = lo;
  c.n_blk = n_blk;
  c.row0 = s_off[lo] + m_blk * tile_m;
  c.rows = min(tile_m, s_off[lo + 1] - c.row0);
  c.split = split;
  c.mtiles = mt;
  return c;
}

// Tile t of a two-class grouped launch: the H tiles of class A sit at positions
// floor(i*(H+C)/H) of the combined list, the C tiles of class B fill the others
// in order; inside each class the usual order (group, n-block, m-block).
__device__ __forceinline__ TileCoord decode_tile_two(int tile, const int* s_off, const int* s_mp,
                                                     const int* s_mp_b, int num_groups,
                                                     int n_tiles, int tile_m) {
  const long long H = static_cast<long long>(s_mp[num_groups]) * n_tiles;
  const long long total = H + static_cast<long long>(s_mp_b[num_groups]) * n_tiles;
  if (H > 0) {
    const long long cnt = ((static_cast<long long>(tile) + 1) * H + total - 1) / total;
    const long long i = cnt - 1;
    if (i >= 0 && (i * total) / H == tile)
      return decode_tile(static_cast<int>(i), s_off, s_mp, num_groups, n_tiles, tile_m);
    return decode_tile(tile - static_cast<int>(cnt), s_off, s_mp_b, num_groups, n_tiles, tile_m);
  }
  return decode_tile(tile, s_off, s_mp_b, num_groups, n_tiles, tile_m);
}

// Tile t of a launch that may carry an extra dense problem: the X extra tiles
// sit at positions floor(i*total/X) of the combined list (so they are spread
// evenly over time and over SMs), the grouped tiles fill the others in order.
__device__ __forceinline__ TileCoord decode_tile_mixed(int tile, const int* s_off, const int* s_mp,
                                                       const int* s_mp_b, int num_groups,
                                                       const GemmParams& P, int grouped_tiles,
                                                       bool& extra, int tile_m = kBM) {
  if (P.x_tiles > 0) {
    const long long total = static_cast<long long>(grouped_tiles) + P.x_tiles;
    // number of extra positions <= tile
    const long long cnt = ((static_cast<long long>(tile) + 1) * P.x_tiles + total - 1) / total;
    const long long i = cnt - 1;
    if (i >= 0 && (i * total) / P.x_tiles == tile) {
      extra = true;
      const int mt = (P.x_rows + kBM - 1) / kBM;
      TileCoord c;
      c.group = 0;
      c.n_blk = static_cast<int>(i / mt);
      c.row0 = static_cast<int>(i % mt) * kBM;
      c.rows = min(kBM, P.x_rows - c.row0);
      c.split = 0;
      c.mtiles = mt;
      return c;
    }
    tile -= static_cast<int>(cnt);
  }
  extra = false;
  if (s_mp_b) return decode_tile_two(tile, s_off, s_mp, s_mp_b, num_groups, P.n_tiles, tile_m);
  return decode_tile(tile, s_off, s_mp, num_groups, P.n_tiles, tile_m);
}

__device__ __forceinline__ void raise_timeout(volatile int* s_abort, int* status) {
  *s_abort = 1;
  atomicExch(status, 6 /* MOE_DEVICE_TIMEOUT */);
}


template <int MODE, int BN = 256, int TM = 128, int OCC = 1>
__global__ void __launch_bounds__(kGemmThreads, OCC)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB0x, const __grid_constant__ CUtensorMap tmB1x,
                    const GemmParams P) {
  static_assert(BN == 256 || BN == 128 || (BN == 64 && MODE == kEpiSwiGLU),
                "tiles of 256 or 128 accumulator columns, or 64 for SwiGLU");
  static_assert(TM == 128 || TM == 64, "tiles of 128 or 64 rows");
  using Cfg = SingleCfg<BN, TM, OCC>;
  constexpr int kStages = Cfg::kStages;
  constexpr int kABytes = Cfg::kABytes;
  constexpr int kStageBytes = Cfg::kStage;
  constexpr int kNumAcc = Cfg::kAcc;
  constexpr int kHalfBytes = Cfg::kHalfRows * kBK * 2;       // one SwiGLU B box
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(kStages) * kStageBytes);
  uint64_t* full_bar = bars;                       // [kStages] TMA -> MMA
  uint64_t* empty_bar = bars + kStages;            // [kStages] MMA -> TMA
  uint64_t* tfull_bar = bars + 2 * kStages;        // [kNumAcc] MMA -> epilogue
  uint64_t* tempty_bar = tfull_bar + kNumAcc;      // [kNumAcc] epilogue -> MMA
  uint64_t* drain_bar = tempty_bar + kNumAcc;      // MMA drain on abort
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(smem + size_t(kStages) * kStageBytes + Cfg::kBarBytes);
  const int num_groups = P.group_offsets ? P.num_groups : 1;
  int* s_mp = s_off + (num_groups + 1);
  int* s_mp_b = P.group_mtiles_b ? s_mp + (num_groups + 1) : nullptr;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // with the row gather a stage also waits for the 32 copying lanes
      mbar_init(smem_u32(&full_bar[s]), P.gather_x ? 1 + 32 : 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < kNumAcc; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), kEpiThreads);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    if (P.x_tiles > 0) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB0x);
      tma_prefetch_desc(&tmB1x);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), Cfg::kTmemCols);
    tmem_relinquish();
  }
  // everything above overlaps the previous kernel; the group tables and the A
  // operand are written by it
  pdl_wait();
  if (P.group_offsets) {
    // every load of the tables in flight at once (one L2 round trip, not one
    // per pass of a strided loop): this sits between the dependency wait and
    // the first operand load
    constexpr int kPer = (kMaxGroups + 1 + kGemmThreads - 1) / kGemmThreads;
    int o[kPer], m[kPer], mb[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = threadIdx.x + j * kGemmThreads;
      const bool ok = i <= num_groups;
      o[j] = ok ? P.group_offsets[i] : 0;
      m[j] = ok ? P.group_mtiles[i] : 0;
      mb[j] = ok && s_mp_b ? P.group_mtiles_b[i] : 0;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = threadIdx.x + j * kGemmThreads;
      if (i <= num_groups) {
        s_off[i] = o[j];
        s_mp[i] = m[j];
        if (s_mp_b) s_mp_b[i] = mb[j];
      }
    }
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = P.dense_rows;
    s_mp[0] = 0;
    s_mp[1] = (P.dense_rows + TM - 1) / TM;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  const int grouped_tiles =
      (s_mp[num_groups] + (s_mp_b ? s_mp_b[num_groups] : 0)) * P.n_tiles * P.k_splits;
  const int total_tiles = grouped_tiles + P.x_tiles;
  // k-block range of a tile: its split's share (split-K launches carry no extra
  // problem), else the whole reduction of the tile's problem
  auto kb_range = [&](const TileCoord& tc, bool ex, int& kb_begin, int& kb_end) {
    const int nkb = ((ex ? P.x_K : P.K) + kBK - 1) / kBK;
    kb_begin = P.k_splits > 1 ? tc.split * P.kb_per_split : 0;
    kb_end = P.k_splits > 1 ? min(nkb, kb_begin + P.kb_per_split) : nkb;
  };

  if (warp == 0 || warp == kProducer2Warp) {
    // ------------------------------------------------------------ TMA producers
    // Both walk the tile and k-block sequence; producer `pid` fills the
    // k-blocks it (counted over the CTA's tiles) with it % 2 == pid, i.e.
    // alternate stages of the ring, so their issue latencies overlap.
    const int pid = warp == 0 ? 0 : 1;
    int it = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // per stage: issued at least once / last parity
    bool ok = true;
    // Grouped GEMMs stream a weight tile (evict first) when its group has a
    // single m-block, so no other tile will read it and it should not displace
    // the grouped rows that every n-block reads again; all other loads are plain.
    // (Pinning the grouped rows with evict_last was measured to push reused
    // weight tiles out of L2 and nearly double the DRAM traffic.)
    const bool grouped = P.group_offsets != nullptr;
    const uint64_t once = l2_evict_first_policy();
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      bool ex;
      const TileCoord tc = decode_tile_mixed(tile, s_off, s_mp, s_mp_b, num_groups, P, grouped_tiles, ex, TM);
      const int z = (P.group_offsets && !ex) ? tc.group : 0;
      const bool stream = grouped && !ex && tc.mtiles == 1;
      const CUtensorMap* mA = ex ? &tmA2 : &tmA;
      const CUtensorMap* mB0 = ex ? &tmB0x : &tmB0;
      const CUtensorMap* mB1 = ex ? &tmB1x : &tmB1;
      int kb_begin, kb_end;
      kb_range(tc, ex, kb_begin, kb_end);
      // row gather: lane l copies 16-byte chunk l % 8 of the tile's rows
      // l / 8 + 4 j; their source rows are looked up once per tile
      // (-1: past the group, or a source row outside [0, T): zero-filled)
      const bool gth = MODE == kEpiSwiGLU && P.gather_x != nullptr && !ex;
      int srow[TM / 4];
#pragma unroll
      for (int j = 0; j < TM / 4; ++j) {
        const int r = (lane >> 3) + 4 * j;
        const int src = (gth && r < tc.rows) ? __ldg(P.gather_src + tc.row0 + r) : -1;
        srow[j] = static_cast<unsigned>(src) < static_cast<unsigned>(P.gather_T) ? src : -1;
      }
      for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
        if ((it & 1) != pid) continue;
        if (P.test_withhold && blockIdx.x == 0 && it == 0) continue;   // test hook
        const int s = it % kStages;
        const uint32_t ph = static_cast<uint32_t>(it / kStages) & 1u;
        ok = mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, s_abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          if (lane == 0) raise_timeout(s_abort, P.status);
          break;
        }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full_bar[s]);
          const uint32_t a_dst = smem_u32(smem + size_t(s) * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const int k0 = kb * kBK;
          mbar_arrive_expect_tx(fb, gth ? kStageBytes - kABytes : kStageBytes);
          if (!gth) tma_load_2d(a_dst, mA, fb, k0, tc.row0);
          // SwiGLU: BN/2 rows of W1 then the same rows of W3; plain: BN rows
          // of the one weight in 128-row boxes (one or two)
          const CUtensorMap* b1 = MODE == kEpiSwiGLU ? mB1 : mB0;
          const int n0 = MODE == kEpiSwiGLU ? tc.n_blk * (BN / 2) : tc.n_blk * BN;
          const int n1 = MODE == kEpiSwiGLU ? n0 : n0 + 128;
          constexpr bool kTwoBoxes = MODE == kEpiSwiGLU || BN == 256;
          const uint32_t b_hi = b_dst + (MODE == kEpiSwiGLU ? kHalfBytes : kBHalfBytes);
          if (stream) {
            tma_load_3d_hint(b_dst, mB0, fb, k0, n0, z, once);
            if (kTwoBoxes) tma_load_3d_hint(b_hi, b1, fb, k0, n1, z, once);
          } else {
            tma_load_3d(b_dst, mB0, fb, k0, n0, z);
            if (kTwoBoxes) tma_load_3d(b_hi, b1, fb, k0, n1, z);
          }
        }
        if (gth) {
          // the A box in the layout the tensor map would give it: row r at
          // r * 128 bytes, 16-byte chunk c at (c ^ (r % 8)) * 16 (128-byte swizzle)
          const uint32_t a_dst = smem_u32(smem + size_t(s) * kStageBytes);
          const int c = lane & 7;
          const int vec = kb * (kBK / 8) + c;            // 16-byte vector of the x row
          const bool col_ok = vec < P.gather_ld_vec;
          // rows past the group and columns past K are zero-filled: every lane
          // issues the same copies (measured faster on the decode step than
          // skipping the rows past the group, whose per-lane branches cost more
          // than the zero-fills they save)
#pragma unroll
          for (int j = 0; j < TM / 4; ++j) {
            const int r = (lane >> 3) + 4 * j;
            const bool ok_r = srow[j] >= 0 && col_ok;
            const uint4* src = ok_r ? P.gather_x + static_cast<long long>(srow[j]) * P.gather_ld_vec + vec
                                    : P.gather_x;
            cp_async_16(a_dst + static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4)), src,
                        ok_r ? 16u : 0u);
          }
          cp_async_arrive_noinc(smem_u32(&full_bar[s]));
        } else if (MODE == kEpiSwiGLU && P.gather_x) {
          mbar_arrive(smem_u32(&full_bar[s]));      // A came by TMA: the lanes' arrivals
        }
        __syncwarp();
        issued_mask |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
      }
    }
    if (P.gather_x) cp_async_wait_all();          // this lane's row copies have landed
    if (!ok && lane == 0) {
      // give the copies already issued a bounded chance to land before teardown
      for (int i = 0; i < kStages; ++i)
        if (issued_mask & (1u << i)) {
          int never = 0;
          mbar_wait(smem_u32(&full_bar[i]), (issued_par >> i) & 1u, &never);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc128 = idesc_bf16_f32(kBM, BN);
    constexpr uint32_t idesc64 = idesc_bf16_f32(64, BN);
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t acc_ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      bool ex;
      const TileCoord tc = decode_tile_mixed(tile, s_off, s_mp, s_mp_b, num_groups, P, grouped_tiles, ex, TM);
      const uint32_t idesc = tc.rows <= 64 ? idesc64 : idesc128;
      int kb_begin, kb_end;
      kb_range(tc, ex, kb_begin, kb_end);
      ok = mbar_wait(smem_u32(&tempty_bar[acc]), acc_ph ^ 1u, s_abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        ok = mbar_wait(smem_u32(&full_bar[s]), ph, s_abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        if (lane == 0) {
          if (P.gather_x) fence_proxy_async_smem();   // rows written by cp.async
          const uint32_t a_base = smem_u32(smem + size_t(s) * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k) {
            umma_bf16(d_tmem, sdesc_kmajor_sw128(a_base + k * kUK * 2),
                      sdesc_kmajor_sw128(b_base + k * kUK * 2), idesc,
                      (kb > kb_begin || k > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty_bar[s]));   // frees the stage when these MMAs finish
        }
        __syncwarp();
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&tfull_bar[acc]));  // accumulator ready
      __syncwarp();
      if (++acc == kNumAcc) { acc = 0; acc_ph ^= 1u; }
    }
    if (!ok) {
      if (lane == 0) {
        raise_timeout(s_abort, P.status);
        umma_commit(smem_u32(drain_bar));        // wait for MMAs in flight before teardown
        int never = 0;
        mbar_wait(smem_u32(drain_bar), 0, &never);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // M=128 accumulator: row r lives in TMEM lane r. M=64 accumulator: rows
    // 16q..16q+15 live in lanes 32q..32q+15 of lane quarter q.
    const int quarter = warp & 3;                 // TMEM lanes this warp may access
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      bool ex;
      const TileCoord tc = decode_tile_mixed(tile, s_off, s_mp, s_mp_b, num_groups, P, grouped_tiles, ex, TM);
      void* const out_base = ex ? P.x_out : P.out;
      const long long ldo = ex ? P.x_ldo : P.ldo;
      const int n_valid = ex ? P.x_N : P.N;
      const bool to_f32 = MODE == kEpiF32 || (ex && P.x_out_f32);
      bool ok = mbar_wait(smem_u32(&tfull_bar[acc]), acc_ph, s_abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_timeout(s_abort, P.status);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tbase = lane_base + static_cast<uint32_t>(acc * BN);
      const bool m64 = tc.rows <= 64;
      const int r = m64 ? quarter * 16 + lane : quarter * 32 + lane;   // tile row of this thread
      const bool row_ok = (!m64 || lane < 16) && r < tc.rows;
      const long long grow = static_cast<long long>(tc.row0) + r;
      if (MODE == kEpiSwiGLU) {
        const int col0 = tc.n_blk * (BN / 2);
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(out_base);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          if (col0 + c >= n_valid) break;              // warp-uniform
          uint32_t g[32], u[32];
          tmem_ld_32cols(tbase + c, g);
          tmem_ld_32cols(tbase + BN / 2 + c, u);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = col0 + c + v * 8;
              if (col < n_valid) {
                uint32_t pk[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float g0 = __uint_as_float(g[v * 8 + 2 * q]);
                  const float g1 = __uint_as_float(g[v * 8 + 2 * q + 1]);
                  const float u0 = __uint_as_float(u[v * 8 + 2 * q]);
                  const float u1 = __uint_as_float(u[v * 8 + 2 * q + 1]);
                  const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                  const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                  pk[q] = pack_bf16x2(h0, h1);
                }
                *reinterpret_cast<uint4*>(out + grow * ldo + col) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
            }
          }
        }
      } else {
        const int col0 = tc.n_blk * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          if (col0 + c >= n_valid) break;              // warp-uniform
          uint32_t a[32];
          tmem_ld_32cols(tbase + c, a);
          tmem_ld_wait();
          if (!row_ok) continue;
          if (!to_f32) {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(out_base);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = col0 + c + v * 8;
              if (col < n_valid) {
                uint32_t pk[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  pk[q] = pack_bf16x2(__uint_as_float(a[v * 8 + 2 * q]),
                                      __uint_as_float(a[v * 8 + 2 * q + 1]));
                *reinterpret_cast<uint4*>(out + grow * ldo + col) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
            }
          } else {
            float* out = reinterpret_cast<float*>(out_base) + tc.split * P.split_stride;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const int col = col0 + c + v * 4;
              float* dst = out + grow * ldo + col;
              if (col + 4 <= n_valid) {
                *reinterpret_cast<float4*>(dst) =
                    make_float4(__uint_as_float(a[v * 4]), __uint_as_float(a[v * 4 + 1]),
                                __uint_as_float(a[v * 4 + 2]), __uint_as_float(a[v * 4 + 3]));
              } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  if (col + q < n_valid) dst[q] = __uint_as_float(a[v * 4 + q]);
              }
            }
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&tempty_bar[acc]));
      if (++acc == kNumAcc) { acc = 0; acc_ph ^= 1u; }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}


// ---------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs on two SMs computes
// one M=256 tile of NW*256 accumulator columns. Each CTA loads its own 128 rows
// of A and its own half of B (the W1 half on the even CTA and the W3 half on
// the odd one for the SwiGLU epilogue, N rows 0-127 / 128-255 of every 256
// otherwise) into shared memory; the even CTA issues the MMAs, which read both
// CTAs' shared memory, and each CTA's TMEM receives its own 128 accumulator
// rows. Per MMA each SM supplies 8 KB of operands instead of 12 KB.
//   * TMA loads of both CTAs count their bytes on the even CTA's full barrier;
//   * the MMA commits are multicast to the empty / tmem-full barriers of both;
//   * both CTAs' epilogue threads arrive on the even CTA's tmem-empty barriers.
// TMEM holds two 256-column regions. NW=1: each tile uses one region, two
// tiles alternate (the epilogue of one overlaps the MMAs of the next). NW=2
// (wide tiles, 256x512): each tile uses both regions; the operand bytes per
// FLOP drop by a quarter, and each region is released as soon as the epilogue
// has drained it, so the next tile's MMAs into region 0 overlap the epilogue
// of region 1.
constexpr int kPairTileM = 256;

template <int NW>
struct PairCfg {
  static constexpr int kBBytes = NW * kBHalfBytes;            // this CTA's B rows per stage
  static constexpr int kStageBytes = kATileBytes + kBBytes;   // 32 KB (NW=1), 48 KB (NW=2)
  static constexpr int kStages = NW == 1 ? 6 : 4;
};

template <int NW>
__host__ __device__ constexpr size_t gemm_pair_smem_bytes(int num_groups) {
  return 1024 + size_t(PairCfg<NW>::kStages) * PairCfg<NW>::kStageBytes + 256 +
         size_t(2) * (num_groups + 1) * sizeof(int);
}

// Output columns one pair tile produces.
__host__ __device__ constexpr int pair_tile_cols(int mode, int nw) {
  return (mode == kEpiSwiGLU ? 128 : 256) * nw;
}

template <int MODE, int NW>
__global__ void __launch_bounds__(kPairThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB1, const GemmParams P) {
  using Cfg = PairCfg<NW>;
  constexpr int kS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(kS) * Cfg::kStageBytes);
  uint64_t* full_bar = bars;                          // [kS] (even CTA's are used)
  uint64_t* empty_bar = bars + kS;                    // [kS] both CTAs
  uint64_t* tfull_bar = bars + 2 * kS;                // [2] both CTAs
  uint64_t* tempty_bar = tfull_bar + 2;               // [2] per TMEM region (even CTA's)
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  static_assert((2 * kS + 2 + 2 + 1) * 8 + 8 <= 256, "pair barriers fit their 256 bytes");
  int* s_off = reinterpret_cast<int*>(smem + size_t(kS) * Cfg::kStageBytes + 256);
  const int num_groups = P.group_offsets ? P.num_groups : 1;
  int* s_mp = s_off + (num_groups + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank & 1u) == 0u;
  const uint32_t leader_rank = rank & ~1u;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 2 * kEpiThreads);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();
  if (P.group_offsets) {
    for (int i = threadIdx.x; i <= num_groups; i += blockDim.x) {
      s_off[i] = P.group_offsets[i];
      s_mp[i] = P.group_mtiles[i];
    }
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = P.dense_rows;
    s_mp[0] = 0;
    s_mp[1] = (P.dense_rows + kPairTileM - 1) / kPairTileM;
  }
  // barrier initialisation and the TMEM allocation must be visible to the
  // other CTA of the pair before either signals the other
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  const int total_tiles = s_mp[num_groups] * P.n_tiles;
  const int num_kb = (P.K + kBK - 1) / kBK;
  const int half = leader ? 0 : 1;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Grouped GEMMs stream a weight tile (evict first) when its group has a
    // single m-block, so no other tile will read it; all other loads are plain.
    const bool grouped = P.group_offsets != nullptr;
    const uint64_t once = l2_evict_first_policy();
    int s = 0;
    uint32_t ph = 0;
    uint32_t issued_mask = 0, issued_par = 0;
    bool ok = true;
    for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
      const TileCoord tc = decode_tile(tile, s_off, s_mp, num_groups, P.n_tiles, kPairTileM);
      const int z = P.group_offsets ? tc.group : 0;
      const bool stream = grouped && tc.mtiles == 1;
      const int my_row0 = tc.row0 + half * kBM;
      const CUtensorMap* bmap = (MODE == kEpiSwiGLU && half) ? &tmB1 : &tmB0;
      for (int kb = 0; kb < num_kb; ++kb) {
        ok = mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, s_abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          if (lane == 0) raise_timeout(s_abort, P.status);
          break;
        }
        if (lane == 0) {
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[s]), leader_rank);
          const uint32_t a_dst = smem_u32(smem + size_t(s) * Cfg::kStageBytes);
          const uint32_t b_dst = a_dst + kATileBytes;
          const int k0 = kb * kBK;
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), 2 * Cfg::kStageBytes);
          tma_load_2d_pair(a_dst, &tmA, fb, k0, my_row0);
#pragma unroll
          for (int j = 0; j < NW; ++j) {
            const int n = MODE == kEpiSwiGLU ? tc.n_blk * 128 * NW + j * 128
                                             : tc.n_blk * 256 * NW + j * 256 + half * 128;
            if (stream)
              tma_load_3d_pair_hint(b_dst + j * kBHalfBytes, bmap, fb, k0, n, z, once);
            else
              tma_load_3d_pair(b_dst + j * kBHalfBytes, bmap, fb, k0, n, z);
          }
        }
        __syncwarp();
        issued_mask |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
        if (++s == kS) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok && leader && lane == 0) {
      // the even CTA's full barriers count both CTAs' bytes: give the copies in
      // flight a bounded chance to land before teardown
      for (int i = 0; i < kS; ++i)
        if (issued_mask & (1u << i)) {
          int never = 0;
          mbar_wait(smem_u32(&full_bar[i]), (issued_par >> i) & 1u, &never);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPairTileM, kBN);
      int s = 0;
      uint32_t ph = 0;
      int slot = 0;                // NW=1: TMEM region of this tile
      uint32_t slot_ph = 0;        // phase of the region barriers this tile waits on
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        for (int kb = 0; kb < num_kb && ok; ++kb) {
          ok = mbar_wait(smem_u32(&full_bar[s]), ph, s_abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t a_base = smem_u32(smem + size_t(s) * Cfg::kStageBytes);
          const uint32_t b_base = a_base + kATileBytes;
#pragma unroll
          for (int j = 0; j < NW; ++j) {
            const int region = NW == 1 ? slot : j;
            if (kb == 0) {
              // the region must have been drained by both epilogues
              ok = mbar_wait(smem_u32(&tempty_bar[region]), slot_ph ^ 1u, s_abort);
              ok = __all_sync(0xffffffffu, ok);
              if (!ok) break;
              tc_fence_after_sync();
            }
            if (lane == 0) {
              const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(region * kBN);
#pragma unroll
              for (int k = 0; k < kBK / kUK; ++k)
                umma_bf16_pair(d_tmem, sdesc_kmajor_sw128(a_base + k * kUK * 2),
                               sdesc_kmajor_sw128(b_base + j * kBHalfBytes + k * kUK * 2),
                               idesc, (kb > 0 || k > 0) ? 1u : 0u);
            }
            __syncwarp();
          }
          if (!ok) break;
          if (lane == 0) umma_commit_pair(smem_u32(&empty_bar[s]));   // frees the stage in both CTAs
          __syncwarp();
          if (++s == kS) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair(smem_u32(&tfull_bar[NW == 1 ? slot : 0]));
        __syncwarp();
        if (NW == 1) {
          if (++slot == 2) { slot = 0; slot_ph ^= 1u; }
        } else {
          slot_ph ^= 1u;
        }
      }
      if (!ok) {
        if (lane == 0) {
          raise_timeout(s_abort, P.status);
          umma_commit_pair(smem_u32(drain_bar));
          int never = 0;
          mbar_wait(smem_u32(drain_bar), 0, &never);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // row of this CTA's 128-row half
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int slot = 0;
    uint32_t slot_ph = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const TileCoord tc = decode_tile(tile, s_off, s_mp, num_groups, P.n_tiles, kPairTileM);
      const int tb = NW == 1 ? slot : 0;
      bool ok = mbar_wait(smem_u32(&tfull_bar[tb]), slot_ph, s_abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_timeout(s_abort, P.status);
        break;
      }
      tc_fence_after_sync();
      const bool row_ok = r < tc.rows - half * kBM;
      const long long grow = static_cast<long long>(tc.row0) + half * kBM + r;
#pragma unroll 1
      for (int j = 0; j < NW; ++j) {
        const int region = NW == 1 ? slot : j;
        const uint32_t tbase = lane_base + static_cast<uint32_t>(region * kBN);
        if (MODE == kEpiSwiGLU) {
          const int col0 = tc.n_blk * 128 * NW + j * 128;
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(P.out);
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            if (col0 + c >= P.N) break;
            uint32_t g[32], u[32];
            tmem_ld_32cols(tbase + c, g);
            tmem_ld_32cols(tbase + 128 + c, u);
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int col = col0 + c + v * 8;
                if (col < P.N) {
                  uint32_t pk[4];
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    const float g0 = __uint_as_float(g[v * 8 + 2 * q]);
                    const float g1 = __uint_as_float(g[v * 8 + 2 * q + 1]);
                    const float u0 = __uint_as_float(u[v * 8 + 2 * q]);
                    const float u1 = __uint_as_float(u[v * 8 + 2 * q + 1]);
                    pk[q] = pack_bf16x2(g0 / (1.0f + __expf(-g0)) * u0,
                                        g1 / (1.0f + __expf(-g1)) * u1);
                  }
                  *reinterpret_cast<uint4*>(out + grow * P.ldo + col) =
                      make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
              }
            }
          }
        } else {
          const int col0 = tc.n_blk * 256 * NW + j * 256;
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            if (col0 + c >= P.N) break;
            uint32_t a[32];
            tmem_ld_32cols(tbase + c, a);
            tmem_ld_wait();
            if (!row_ok) continue;
            if (MODE == kEpiBF16) {
              __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(P.out);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int col = col0 + c + v * 8;
                if (col < P.N) {
                  uint32_t pk[4];
#pragma unroll
                  for (int q = 0; q < 4; ++q)
                    pk[q] = pack_bf16x2(__uint_as_float(a[v * 8 + 2 * q]),
                                        __uint_as_float(a[v * 8 + 2 * q + 1]));
                  *reinterpret_cast<uint4*>(out + grow * P.ldo + col) =
                      make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
              }
            } else {
              float* out = reinterpret_cast<float*>(P.out);
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const int col = col0 + c + v * 4;
                float* dst = out + grow * P.ldo + col;
                if (col + 4 <= P.N) {
                  *reinterpret_cast<float4*>(dst) =
                      make_float4(__uint_as_float(a[v * 4]), __uint_as_float(a[v * 4 + 1]),
                                  __uint_as_float(a[v * 4 + 2]), __uint_as_float(a[v * 4 + 3]));
                } else {
#pragma unroll
                  for (int q = 0; q < 4; ++q)
                    if (col + q < P.N) dst[q] = __uint_as_float(a[v * 4 + q]);
                }
              }
            }
          }
        }
        // this region is drained: release it to the even CTA's MMA issuer
        tc_fence_before_sync();
        if (leader)
          mbar_arrive(smem_u32(&tempty_bar[region]));
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[region]), leader_rank));
      }
      if (NW == 1) {
        if (++slot == 2) { slot = 0; slot_ph ^= 1u; }
      } else {
        slot_ph ^= 1u;
      }
    }
  }

  // neither CTA may leave while the other can still signal its barriers
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace moe
