// router_sm100.cuh - the fused router: for a tile of 128 tokens, the router
// scores s = x W_g^T on the 5th-generation tensor core, the softmax over the N_r
// experts, the top-k with ties to the lower expert index, the gates and the
// expert histogram, in one launch ("What is an "expert," really?", glossary:
// router / gate, top-k, softmax; panel 2: a linear scorer, softmax blend
// weights, keep the top k). With few tiles the last cluster of the grid also
// turns the histogram into per-tile bases and expert totals, so the
// permutation kernel can follow directly.
//
// Design (sm_100a, N_r <= 512, top_k <= 16):
//  * a cluster of CS CTAs (CS <= 8) owns one 128-token tile; CTA r computes the
//    scores of its slice of E = N_r/CS <= 64 experts over the whole K range
//    (one TMEM accumulator), so no partial sums are exchanged;
//  * warp 0 loads A (x rows, one 128x64 box) and B (the slice's W_g rows, boxes
//    of up to 128 rows) per 64-wide K block through TMA (no multicast); warp 1
//    issues tcgen05.mma M=128, N=E;
//  * all 16 warps copy the accumulator to shared memory; then one warp per
//    token (lanes over the slice's experts) takes the slice's softmax
//    statistics (the largest gate score and the sum of exp(score - largest))
//    and its top-k candidates (selection key, expert, gate score) in k rounds
//    of two warp reductions;
//  * with one slice (CS = 1) these are the token's top k and softmax and the
//    warp writes the gates itself; otherwise lane j stores candidate j, and
//    lane 0 the statistics, into the shared memory of the CTA that routes the
//    token (CTA m / (128/CS) for token m of the tile) through distributed
//    shared memory, and after a cluster barrier one warp per token of this
//    CTA's 128/CS tokens selects the top k of the CS * k candidates (largest
//    key, ties to the lower expert index); the softmax over all N_r experts
//    follows from the slices' statistics;
//  * every loop over tokens or columns stays rolled: each CTA runs the code
//    about once, so its length (instruction fetch), not its arithmetic, sets
//    the time;
//  * a shared histogram per CTA; reading the cluster's histograms, each CTA
//    writes its experts' offsets inside the tile and the first CTA the tile's
//    totals, one column of the tile histogram.
#pragma once

#include "gemm_sm100.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtThreads = 1024;  // 32 warps: 32 tokens selected at once per CTA
constexpr int kRtMaxCluster = 8;
constexpr int kRtMaxStages = 8;
constexpr int kRtMaxExperts = 512;
constexpr int kRtMaxTopK = 16;

struct RouterParams {
  int T, d, n_routed, top_k, renorm, bias_select_only;
  const float* bias;     // device (N_r) or null
  int cs;                // CTAs per cluster = expert slices of one token tile
  int e_per;             // experts per slice (multiple of 16, <= 256): MMA N
  int ncols;             // accumulator columns read (e_per rounded up to 32)
  int num_kb;            // 64-wide K blocks of d
  int own_rows;          // tokens each CTA merges (128 / cs)
  int n_chunks;          // ceil(T / 128): columns of tile_counts
  int box_rows;          // rows of one W_g TMA box
  int nbox;              // W_g boxes per stage
  int stages;
  int stage_bytes;       // A box + B boxes of one stage
  int ring_bytes;
  int tmem_cols;
  int fold_scan;         // 1: the grid's last cluster scans the tile histogram
  int* idx;              // (T, top_k)
  float* gate;           // (T, top_k)
  int* tile_counts;      // [N_r][n_chunks] pairs per expert and tile (scanned in place)
  int* sub_base;         // [N_r][n_chunks * cs] an expert's pairs in the tile before each CTA's tokens
  int* counts;           // (N_r), written when fold_scan
  int* ticket;           // zero between forwards
  int* status;           // device status word
};

// Shared memory of the candidates a CTA receives: for each of the CS slices and
// each of its 128/CS tokens (128 rows in all), KMAX candidates (top_k <= KMAX)
// as (key, expert, gate score), plus the slice's (max, sum) statistics.
template <int KMAX>
__host__ __device__ constexpr size_t router_cand_bytes() {
  return size_t(kBM) * KMAX * 12 + size_t(kBM) * 8;
}

constexpr int kRtMaxSliceCols = 64;   // accumulator columns of one slice

// Scratch laid over the ring once the scores are complete: the slice's scores
// [token][ncols + 1] in fp32.
__host__ __device__ constexpr size_t router_scratch_bytes() {
  return size_t(kBM) * (kRtMaxSliceCols + 1) * 4;
}

// Dynamic shared memory of a launch: ring, candidates, histogram, barriers.
template <int KMAX>
__host__ __device__ constexpr size_t router_smem_bytes(int ring_bytes, int n_routed) {
  return 1024 + size_t(ring_bytes) + router_cand_bytes<KMAX>() +
         size_t((n_routed + 3) / 4 * 4) * 4 + 256;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// Order-preserving map of a selection key to an unsigned integer: NaN ranks
// as -inf, -0 equals +0, and -inf maps to 0x007fffff, above the 0 that marks
// an empty candidate.
__device__ __forceinline__ uint32_t order_key(float k) {
  k = k == k ? k : -INFINITY;
  k = k == 0.0f ? 0.0f : k;
  const uint32_t b = __float_as_uint(k);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// k rounds of selection over the warp's candidates (lane l holds key[i],
// expert[i], gate score[i] for i < N; key 0 marks an empty one): each round
// takes the largest key and, among equal keys, the lowest expert (two warp
// reductions); only the winning lane rescans its own. Lane j < k receives the
// j-th winner's key, expert and gate score.
template <int N>
__device__ __forceinline__ void select_rounds(const uint32_t (&key)[N], const int (&ex)[N],
                                              const float (&val)[N], int k, int lane,
                                              uint32_t& my_k, int& my_e, float& my_g) {
  uint32_t taken = 0;
  uint32_t lk = 0u;
  int li = 0x7fffffff, slot = 0;
  auto rescan = [&]() {
    lk = 0u;
    li = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (!((taken >> i) & 1u) && (key[i] > lk || (key[i] == lk && key[i] != 0u && ex[i] < li))) {
        lk = key[i];
        li = ex[i];
        slot = i;
      }
  };
  rescan();
  my_k = 0u;
  my_e = 0x7fffffff;
  my_g = 0.0f;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    const uint32_t gmax = __reduce_max_sync(0xffffffffu, lk);
    const unsigned be =
        __reduce_min_sync(0xffffffffu, static_cast<unsigned>(lk == gmax ? li : 0x7fffffff));
    const bool win = lk == gmax && static_cast<unsigned>(li) == be;
    const unsigned wmask = __ballot_sync(0xffffffffu, win);
    const int wl = wmask ? __ffs(wmask) - 1 : 0;   // one lane holds the winner
    float wv = 0.0f;
#pragma unroll
    for (int i = 0; i < N; ++i) wv = i == slot ? val[i] : wv;
    wv = __shfl_sync(0xffffffffu, wv, wl);
    if (lane == j) {
      my_k = gmax;
      my_e = static_cast<int>(be);
      my_g = wv;
    }
    if (lane == wl && wmask) {
      taken |= 1u << slot;
      rescan();
    }
  }
}

// One warp, one token, one slice: lane l holds the slice's experts e0 + l and
// e0 + l + 32 (n_valid of them are experts; their logit biases in bias[]). Returns to every lane the slice's
// largest gate score m and sum of exp(score - m) (0 for an empty slice), and
// to lane j < k the j-th candidate by selection key (ties to the lower expert)
// as (key, expert, gate score); key 0 where the slice has fewer than k experts.
__device__ __forceinline__ void slice_select(const float* srow, int n_valid, int e0,
                                             const float (&bias)[2], int bias_select_only,
                                             int k, int lane, float& m, float& sum,
                                             uint32_t& my_key, int& my_e, float& my_g) {
  uint32_t key[2];
  int ex[2];
  float g[2];
  m = -INFINITY;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int c = lane + 32 * i;
    const bool v = c < n_valid;
    const float raw = v ? srow[c] : 0.0f;
    const float kv = raw + bias[i];   // 0 without a logit bias
    g[i] = bias_select_only ? raw : kv;
    key[i] = v ? order_key(kv) : 0u;
    ex[i] = v ? e0 + c : 0x7fffffff;
    if (v) m = fmaxf(m, g[i]);
  }
  m = warp_max(m);
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (lane + 32 * i < n_valid) s += expf(g[i] - m);
  sum = warp_sum(s);
  select_rounds<2>(key, ex, g, k, lane, my_key, my_e, my_g);
}

template <int KMAX>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWg, const RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // candidates received for this CTA's tokens, [slice * own + token][slot]
  uint32_t* c_key = reinterpret_cast<uint32_t*>(ring + P.ring_bytes);
  int* c_idx = reinterpret_cast<int*>(c_key + kBM * KMAX);
  float* c_val = reinterpret_cast<float*>(c_idx + kBM * KMAX);
  float* c_max = c_val + kBM * KMAX;               // [slice * own + token] largest gate score
  float* c_sum = c_max + kBM;                      // [slice * own + token] sum of exp(score - largest)
  int* s_hist = reinterpret_cast<int*>(c_sum + kBM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_hist + (P.n_routed + 3) / 4 * 4);
  uint64_t* full_bar = bars;                        // [stages] TMA -> MMA
  uint64_t* empty_bar = bars + kRtMaxStages;        // [stages] MMA -> TMA
  uint64_t* tfull_bar = bars + 2 * kRtMaxStages;    // MMA -> TMEM readers
  uint64_t* drain_bar = tfull_bar + 1;              // MMA drain on abort
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = const_cast<int*>(s_abort) + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile = blockIdx.x / P.cs;
  const int row0 = tile * kBM;
  const int e0 = static_cast<int>(rank) * P.e_per;           // first expert of the slice
  const int n_valid = max(0, min(P.e_per, P.n_routed - e0)); // experts of the slice
  const int nkb = n_valid > 0 ? P.num_kb : 0;
  const int k = P.top_k;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(tfull_bar), 1);
    mbar_init(smem_u32(drain_bar), 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmWg);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), P.tmem_cols);
    tmem_relinquish();
  }
  for (int e = threadIdx.x; e < P.n_routed; e += kRtThreads) s_hist[e] = 0;
  // everything above overlaps the previous kernel; x may be its output, and
  // the outputs below may still be read by it
  pdl_wait();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const int box_bytes = P.box_rows * kBK * 2;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t issued_mask = 0, issued_par = 0;
    bool ok = true;
    for (int it = 0; it < nkb; ++it) {
      const int s = it % P.stages;
      const uint32_t ph = static_cast<uint32_t>(it / P.stages) & 1u;
      ok = mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, s_abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_timeout(s_abort, P.status);
        break;
      }
      if (lane == 0) {
        const uint32_t fb = smem_u32(&full_bar[s]);
        const uint32_t a_dst = smem_u32(ring + size_t(s) * P.stage_bytes);
        const int k0 = it * kBK;
        mbar_arrive_expect_tx(fb, P.stage_bytes);
        tma_load_2d(a_dst, &tmX, fb, k0, row0);
        for (int j = 0; j < P.nbox; ++j)
          tma_load_2d(a_dst + kATileBytes + j * box_bytes, &tmWg, fb, k0, e0 + j * P.box_rows);
      }
      __syncwarp();
      issued_mask |= 1u << s;
      issued_par = (issued_par & ~(1u << s)) | (ph << s);
    }
    if (!ok && lane == 0) {
      // give the copies already issued a bounded chance to land before the
      // CTA exits
      for (int i = 0; i < P.stages; ++i)
        if (issued_mask & (1u << i)) {
          int never = 0;
          mbar_wait(smem_u32(&full_bar[i]), (issued_par >> i) & 1u, &never);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, P.e_per);
    bool ok = true;
    for (int it = 0; it < nkb; ++it) {
      const int s = it % P.stages;
      const uint32_t ph = static_cast<uint32_t>(it / P.stages) & 1u;
      ok = mbar_wait(smem_u32(&full_bar[s]), ph, s_abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after_sync();
      if (lane == 0) {
        const uint32_t a_base = smem_u32(ring + size_t(s) * P.stage_bytes);
        const uint32_t b_base = a_base + kATileBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / kUK; ++kk)
          umma_bf16(tmem_base, sdesc_kmajor_sw128(a_base + kk * kUK * 2),
                    sdesc_kmajor_sw128(b_base + kk * kUK * 2), idesc,
                    (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit(smem_u32(&empty_bar[s]));   // frees the stage when these MMAs finish
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (!ok) {
        raise_timeout(s_abort, P.status);
        umma_commit(smem_u32(drain_bar));        // wait for MMAs in flight before teardown
        int never = 0;
        mbar_wait(smem_u32(drain_bar), 0, &never);
      } else if (nkb > 0) {
        umma_commit(smem_u32(tfull_bar));        // accumulator complete
      } else {
        mbar_arrive(smem_u32(tfull_bar));        // empty slice: nothing to wait for
      }
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- scores to shared memory
  // warps 0..15 each copy a quarter of the slice's columns of one TMEM lane
  // quarter (warps w, w+4, w+8, w+12 share lanes 32*(w%4)..) into the score
  // rows [token][ncols + 1] laid over the ring (every MMA has completed, so
  // every stage has been read)
  float* s_score = reinterpret_cast<float*>(ring);
  const int lds = P.ncols + 1;   // odd stride: the 32 rows of a warp's stores hit 32 banks
  {
    bool ok = mbar_wait(smem_u32(tfull_bar), 0, s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) raise_timeout(s_abort, P.status);
    tc_fence_after_sync();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int cpp = P.ncols / 4;                  // a multiple of 8
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    if (nkb > 0 && ok && warp < 16) {
#pragma unroll 1
      for (int c = (warp >> 2) * cpp; c < ((warp >> 2) + 1) * cpp; c += 8) {
        uint32_t a[8];
        tmem_ld_8cols(taddr + c, a);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) s_score[row * lds + c + i] = __uint_as_float(a[i]);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- slice top-k
  // one warp per token (lane l holds the slice's experts l and l + 32): the
  // slice's largest gate score and sum of exp(score - largest), and its top-k
  // by selection key with ties to the lower expert; lane j ends with the j-th
  {
    const bool have = nkb > 0 && *s_abort == 0;
    const int own_r = P.own_rows;
    float bias[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = lane + 32 * i;
      bias[i] = (P.bias && c < n_valid) ? __ldg(P.bias + e0 + c) : 0.0f;
    }
#pragma unroll 1
    for (int row = warp; row < kBM; row += kRtThreads / 32) {
      float m, sum;
      uint32_t my_key;
      int my_e;
      float my_g;
      slice_select(s_score + row * lds, have ? n_valid : 0, e0, bias, P.bias_select_only,
                   k, lane, m, sum, my_key, my_e, my_g);
      if (P.cs == 1) {
        // one slice holds every expert: the token's softmax and top k
        const int t = row0 + row;
        const float my_p = lane < k ? expf(my_g - m) / sum : 0.0f;
        const float sel = warp_sum(my_p);
        if (t < P.T && lane < k) {
          const long long o = static_cast<long long>(t) * k + lane;
          P.idx[o] = my_e;
          P.gate[o] = P.renorm ? my_p / sel : my_p;
          if (static_cast<unsigned>(my_e) < static_cast<unsigned>(P.n_routed))
            atomicAdd(&s_hist[my_e], 1);
        }
      } else {
        // to the CTA that routes this token: slot (this slice, token) of its buffers
        const uint32_t owner = static_cast<uint32_t>(row / own_r);
        const int slot_row =
            static_cast<int>(rank) * own_r + (row - static_cast<int>(owner) * own_r);
        if (lane < k) {
          st_cluster_u32(mapa_shared(smem_u32(c_key + slot_row * KMAX + lane), owner), my_key);
          st_cluster_u32(mapa_shared(smem_u32(c_idx + slot_row * KMAX + lane), owner),
                         static_cast<uint32_t>(my_e));
          st_cluster_u32(mapa_shared(smem_u32(c_val + slot_row * KMAX + lane), owner),
                         __float_as_uint(my_g));
        }
        if (lane == 0) {
          st_cluster_u32(mapa_shared(smem_u32(c_max + slot_row), owner), __float_as_uint(m));
          st_cluster_u32(mapa_shared(smem_u32(c_sum + slot_row), owner), __float_as_uint(sum));
        }
      }
    }
  }

  // ---------------------------------------------------------------- merge
  // every slice's candidates have arrived; one warp per token of this CTA
  // selects the top k of the CS * k candidates (largest key, ties to the lower
  // expert index); the softmax over all N_r experts follows from the slices'
  // (max, sum)
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  tc_fence_after_sync();
  if (P.cs > 1) {
    const int own = P.own_rows;
    const int tok0 = row0 + static_cast<int>(rank) * own;
    const int ntok = min(own, P.T - tok0);
    const int n_c = P.cs * k;                    // candidates of a token (<= 128)
#pragma unroll 1
    for (int tl = warp; tl < ntok; tl += kRtThreads / 32) {
      const float sm = lane < P.cs ? c_max[lane * own + tl] : -INFINITY;
      const float M = warp_max(sm);
      const float ss = lane < P.cs ? c_sum[lane * own + tl] : 0.0f;
      const float S = warp_sum(ss > 0.0f ? ss * expf(sm - M) : 0.0f);
      uint32_t ck[4];
      int ci[4];
      float cv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qq = lane + 32 * i;             // candidate (slice qq / k, slot qq % k)
        const int sl = qq / k;
        const int at = (sl * own + tl) * KMAX + (qq - sl * k);
        ck[i] = qq < n_c ? c_key[at] : 0u;
        ci[i] = qq < n_c ? c_idx[at] : 0x7fffffff;
        cv[i] = qq < n_c ? c_val[at] : 0.0f;
      }
      uint32_t my_k;
      int my_e;
      float my_g;
      select_rounds<4>(ck, ci, cv, k, lane, my_k, my_e, my_g);
      const float my_p = lane < k ? expf(my_g - M) / S : 0.0f;
      const float sel = warp_sum(my_p);
      if (lane < k) {
        const long long o = static_cast<long long>(tok0 + tl) * k + lane;
        P.idx[o] = my_e;
        P.gate[o] = P.renorm ? my_p / sel : my_p;
        if (static_cast<unsigned>(my_e) < static_cast<unsigned>(P.n_routed))
          atomicAdd(&s_hist[my_e], 1);
      }
    }
  }

  // histograms: from the cluster's per-CTA counts, every CTA writes each
  // expert's pairs in lower-ranked CTAs of the tile (its offset inside the
  // tile) and the first CTA the tile's totals
  __syncthreads();
  cluster_sync();
  {
    const uint32_t hbase = smem_u32(s_hist);
    const int n_sub = P.n_chunks * P.cs;
    for (int e = threadIdx.x; e < P.n_routed; e += kRtThreads) {
      int pre = 0, tot = 0;
      for (int s2 = 0; s2 < P.cs; ++s2) {
        const int h = s2 == static_cast<int>(rank)
                          ? s_hist[e]
                          : static_cast<int>(ld_cluster_u32(mapa_shared(
                                hbase + static_cast<uint32_t>(e * 4), static_cast<uint32_t>(s2))));
        pre += s2 < static_cast<int>(rank) ? h : 0;
        tot += h;
      }
      P.sub_base[static_cast<long long>(e) * n_sub + blockIdx.x] = pre;
      if (rank == 0) P.tile_counts[static_cast<long long>(e) * P.n_chunks + tile] = tot;
    }
  }
  // no CTA leaves while another can still read its shared memory
  cluster_sync();

  if (P.fold_scan && rank == 0) {
    // last cluster to finish: exclusive prefix over tiles of every expert's
    // counts (in place; one thread per expert) and the expert totals; then the
    // ticket is reset for the next forward (every cluster took exactly one)
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      *s_last = atomicAdd(P.ticket, 1) == static_cast<int>(gridDim.x) / P.cs - 1 ? 1 : 0;
    __syncthreads();
    if (*s_last) {
      __threadfence();
      // one thread per expert (other clusters' counts: read through L2), eight
      // tiles' counts loaded before the first of them is rewritten
#pragma unroll 1
      for (int e = threadIdx.x; e < P.n_routed; e += kRtThreads) {
        int* rowp = P.tile_counts + static_cast<long long>(e) * P.n_chunks;
        int run = 0;
#pragma unroll 1
        for (int c0 = 0; c0 < P.n_chunks; c0 += 8) {
          int v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = c0 + j < P.n_chunks ? __ldcg(rowp + c0 + j) : 0;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c0 + j < P.n_chunks) {
              rowp[c0 + j] = run;
              run += v[j];
            }
        }
        P.counts[e] = run;
      }
      if (threadIdx.x == 0) *P.ticket = 0;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, P.tmem_cols);
}

}  // namespace moe
