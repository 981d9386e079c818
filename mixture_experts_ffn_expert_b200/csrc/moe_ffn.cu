// moe_ffn.cu - host planner and C ABI of libmoe_ffn.so (declared in
// include/moe_ffn.h): validates arguments, lays out the caller's workspace,
// encodes the TMA tensor maps and enqueues the layer's kernels on the caller's
// stream. It never synchronises the host in moe_forward and never allocates
// device memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "moe_ffn.h"
#include "gemm_sm100.cuh"
#include "route.cuh"
#include "router_sm100.cuh"

static_assert(moe::kMaxGroups >= moe::kMaxRouted,
              "a grouped GEMM launch holds the tables of every routed expert");

namespace {

thread_local std::string g_last_error;
thread_local int g_last_status = MOE_OK;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  g_last_status = status;
  return status;
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr int kMaxKernels = 16;
constexpr int kTimingRing = 4;   // event sets: forward i records into set i % kTimingRing

struct Layout {
  size_t status, ticket, scores, idx, gate, chunk_counts, sub_base, counts, offsets, mtiles,
      mtiles2, mtiles64, mt_hot, mt_cold, perm_src, inv_pos;
  size_t xperm, hidden, yrouted, hshared, yshared, total;
  int lds;            // row stride of the fp32 router scores
  int tpc;            // tokens per block of route_scatter
  int n_chunks;       // blocks of route_scatter
  int sub_tokens;     // tokens per sub-chunk of the histogram (a multiple of tpc)
  int n_base;         // columns of chunk_counts: one per group of subs_per_base sub-chunks
  int subs_per_base;
  int router_splits;  // split-K factor of the router GEMM (partials summed by route_topk)
  int router_kb_per;  // k-blocks per split
  bool fused;         // router scores + softmax + top-k in one kernel (route_fused)
  moe::RouterParams rt;   // its launch shape (sizes only; pointers set per forward)
  size_t rt_smem;         // its dynamic shared memory
};

// Router score tiles are 128 columns wide: the epilogue of a tile (TMEM to
// registers to fp32 stores, about 0.6 us per 32 columns on B200) is the
// router GEMM's longest phase when the reduction is split K-wise over the SMs,
// so narrower tiles on twice the CTAs halve it (512-expert decode step: the
// epilogue took 4.9 us with 256-column tiles, 2.3 us with 128).
constexpr int kRouterCols = 128;
constexpr size_t kRouterMinSmem = 116 * 1024;   // one fused-router CTA per SM (see below)

}  // namespace

struct moe_plan {
  int d, f, n_routed, top_k, n_shared, renorm;
  // GEMMs whose expected rows per group reach these use the CTA-pair kernel.
  // Measured on B200: the pair kernel wins for the routed down projection
  // (plain epilogue) but not for the SwiGLU GEMMs, where the single-CTA kernel
  // runs at the same throughput per clock and draws less power, so it holds a
  // higher clock under the power cap. MOE_OPTION_PAIR_MIN_ROWS sets both.
  long long pair_min_rows_plain = 256;
  long long pair_min_rows_swiglu = 1LL << 62;
  // CTA-pair tiles 512 accumulator columns wide: -1 automatic, 0 never, 1 always
  int wide_tiles = -1;
  // shared expert as extra tiles of the routed single-CTA GEMM launches: -1
  // automatic (a small shared expert, at most half the SMs' worth of tiles,
  // when the routed launches use their default tiles), 0 never, 1 whenever
  // possible. Measured on B200 (CUDA-graph steps, L2 flushed): the 512-expert
  // decode step 133.1 us merged against 135.8 us with the shared expert forked
  // onto the side stream, the 31-expert tiny layer 38.9 vs 43.6 us. A large
  // shared expert stays separate: merged it ran the launches at a lower clock
  // under the power cap and lost 5% on the DeepSeek-V3 layer shape.
  int merge_shared = -1;
  // output columns of a single-CTA routed SwiGLU tile: 0 automatic (128), 32,
  // 64 or 128
  int swiglu_tile_cols = 0;
  // interleave the tiles of experts with several m-blocks among the others in
  // single-CTA 128-row routed GEMMs: -1 automatic (when the expected rows per
  // expert are from 32 to 191, i.e. most experts stream weights but some reuse
  // them), 0 never, 1 always
  int interleave = -1;
  // rows of a single-CTA routed GEMM tile: 0 automatic (128), 64 or 128
  int tile_rows = 0;
  // resident CTAs per SM of single-CTA routed GEMMs: 0 automatic (1), 1 or 2
  int ctas_per_sm = 0;
  // output columns of a single-CTA routed down tile: 0 automatic (256), 128 or 256
  int down_tile_cols = 0;
  // the single-CTA routed gate/up GEMM gathers its rows from x through the
  // permutation (no row copies): 1 on, 0 off, -1 automatic (below 32 expected
  // rows per expert, the decode regime)
  int gather_rows = -1;
  // shared expert beside weight-streaming routed GEMMs: -1 automatic, 0 never, 1 always.
  // Measured on B200 (DeepSeek-V3-shaped prefill): beside the routed GEMMs on 16
  // SMs the layer took 7.09 ms per step against 6.19 ms inline (the capped
  // routed GEMMs slowed more than the shared GEMMs saved), so automatic means never.
  int shared_concurrent = -1;
  // router: 1 the fused router whenever supported (N_r <= 512, top_k <= 32),
  // 0 the split router (scores GEMM, then softmax + top-k), -1 automatic = the
  // split router. Measured on B200 (CUDA-graph steps, L2 flushed): 512-expert
  // decode 162 us fused vs 137 us split, the 31-expert tiny layer 62 vs 43 us,
  // DeepSeekMoE-small and coarse 3-4% slower fused, DeepSeek-V3 prefill within
  // noise. The fused kernel takes about the split kernels' summed time, but a
  // 128-token tile is one cluster, so small batches select on few SMs, and a
  // cluster of large-shared-memory CTAs cannot start early beside its
  // predecessor the way the small split kernels do.
  int fused_router = -1;
  // seats per expert per forward (token dropping); 0: unlimited (dropless)
  int64_t capacity = 0;
  // capacity factor in thousandths: seats = ceil(factor * T * top_k / N_r) per
  // forward over T tokens; 0: off (capacity above applies)
  int64_t capacity_permille = 0;
  // 1: the logit bias only chooses the experts, the gates come from unbiased scores
  int bias_select_only = 0;
  // one-shot test hook: the next forward's routed gate/up GEMM (single-CTA
  // kernel) lets one bounded wait expire
  int test_withhold = 0;
  int device, num_sms;
  const float* bias = nullptr;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  int64_t last_T = -1;
  bool timing = false;
  int n_launch = 0;
  char names[kMaxKernels][48] = {};   // kernel of each launch, with the GEMM variant
  // per kernel a start and an end event, recorded on the stream it runs on
  cudaEvent_t ev[kTimingRing][2 * kMaxKernels] = {};
  int ring_launches[kTimingRing] = {};
  long long timed_forwards = 0;     // forwards that recorded events
  int cur_set = 0;
  bool events_made = false;
  // stream and events for a shared expert forked beside the routing (a small
  // one that is not merged) or beside the routed GEMMs (SHARED_CONCURRENT)
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  // device address of the allocation-free forward's static scratch in this
  // plan's context (looked up at plan creation), and whether a forward of this
  // plan has used it since moe_plan_device_status last read its status word
  void* noalloc_scratch = nullptr;
  bool noalloc_used = false;
};

namespace {

// Launch shape of the fused router for T tokens (see router_sm100.cuh): a
// cluster of CS CTAs per 128-token tile, CTA r scoring experts
// [r*E, (r+1)*E) over the whole K range. CS is the power of two that makes the
// slices about 64 experts (E <= 256), at most 8.
moe::RouterParams router_shape(const moe_plan* p, int64_t T, size_t* smem) {
  moe::RouterParams r{};
  const int nr = p->n_routed;
  const int mt = static_cast<int>((T + moe::kBM - 1) / moe::kBM);
  auto up = [](int v, int m) { return (v + m - 1) / m * m; };
  int cs = 1;
  while (cs < moe::kRtMaxCluster && (nr + cs - 1) / cs > 64) cs *= 2;
  r.T = static_cast<int>(T);
  r.d = p->d;
  r.n_routed = nr;
  r.top_k = p->top_k;
  r.renorm = p->renorm;
  r.bias_select_only = p->bias_select_only;
  r.cs = cs;
  r.e_per = up((nr + cs - 1) / cs, 16);
  r.ncols = up(r.e_per, 32);
  r.num_kb = (p->d + moe::kBK - 1) / moe::kBK;
  r.own_rows = moe::kBM / cs;
  r.n_chunks = mt;                 // one column of the histogram per 128-token tile
  r.box_rows = r.e_per < 128 ? r.e_per : 128;
  r.nbox = (r.e_per + r.box_rows - 1) / r.box_rows;
  r.stage_bytes = moe::kATileBytes + r.nbox * r.box_rows * moe::kBK * 2;
  int stages = (168 * 1024) / r.stage_bytes;
  if (stages > r.num_kb) stages = r.num_kb;
  stages = stages < 2 ? 2 : (stages > moe::kRtMaxStages ? moe::kRtMaxStages : stages);
  r.stages = stages;
  // the ring also holds the statistics phase's scratch once the scores are done
  const int scratch = static_cast<int>(moe::router_scratch_bytes());
  const int ring = stages * r.stage_bytes;
  r.ring_bytes = up(ring > scratch ? ring : scratch, 1024);
  int cols = 32;
  while (cols < r.ncols) cols *= 2;
  r.tmem_cols = cols;
  // fold the tile scan into the router's last cluster while there are few
  // tiles (one thread per expert walks them)
  r.fold_scan = r.n_chunks <= 64 ? 1 : 0;
  // at least kRouterMinSmem so that two router CTAs never share an SM: each
  // allocates tensor memory and then waits at cluster barriers, and two
  // clusters interleaved on two SMs could otherwise wait on each other
  const size_t bytes = moe::router_smem_bytes(r.ring_bytes, nr);
  *smem = bytes < kRouterMinSmem ? kRouterMinSmem : bytes;
  return r;
}

Layout make_layout(const moe_plan* p, int64_t T) {
  Layout L{};
  const int64_t A = T * p->top_k;
  const int nsf = p->n_shared * p->f;
  L.fused = p->fused_router == 1 && p->n_routed <= moe::kRtMaxExperts &&
            p->top_k <= moe::kRtMaxTopK;
  L.lds = static_cast<int>(align_up(p->n_routed, 8));
  if (L.fused) {
    // the router's histogram has one column per 128-token tile, plus each CTA's
    // offsets inside its tile (sub-chunks of 128/CS tokens); route_scatter's
    // blocks take 8..128/CS tokens, about two blocks per SM
    L.rt = router_shape(p, T, &L.rt_smem);
    L.sub_tokens = L.rt.own_rows;
    L.subs_per_base = L.rt.cs;
    L.n_base = L.rt.n_chunks;
    int tpc = 8;
    while (tpc < L.sub_tokens && static_cast<int64_t>(tpc) * 2 * p->num_sms < T) tpc *= 2;
    L.tpc = tpc;
    L.n_chunks = static_cast<int>((T + tpc - 1) / tpc);
    L.router_splits = 0;
    L.router_kb_per = 0;
  } else {
    // chunking of the routing kernels: about two chunks per SM, 8..128 tokens each
    int64_t tpc = (T + 2 * p->num_sms - 1) / (2 * p->num_sms);
    tpc = tpc < 8 ? 8 : (tpc > 128 ? 128 : tpc);
    L.tpc = static_cast<int>(tpc);
    L.n_chunks = static_cast<int>((T + tpc - 1) / tpc);
    L.sub_tokens = L.tpc;
    L.subs_per_base = 1;
    L.n_base = L.n_chunks;
    // split-K of the router GEMM so that it occupies most SMs even for few tokens
    const int64_t tiles =
        ((T + moe::kBM - 1) / moe::kBM) * ((p->n_routed + kRouterCols - 1) / kRouterCols);
    const int num_kb = (p->d + moe::kBK - 1) / moe::kBK;
    // at most 4 splits: the partial sums cost route_topk instruction fetch and
    // loads (on the 512-expert decode step 4 splits measured 2.2 us faster
    // than 8), and 4 keeps a lane's partial scores at 4 x 32 at most (N_r <= 1024)
    const int64_t cap = 4;
    int64_t sp = tiles > 0 ? p->num_sms / tiles : 1;
    sp = sp < 1 ? 1 : (sp > cap ? cap : sp);
    if (sp > num_kb) sp = num_kb;
    L.router_kb_per = static_cast<int>((num_kb + sp - 1) / sp);
    L.router_splits = (num_kb + L.router_kb_per - 1) / L.router_kb_per;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.status = take(256);          // status word at +0, router ticket at +64
  L.ticket = L.status + 64;
  L.scores = take(L.fused ? 0 : size_t(L.router_splits) * T * L.lds * 4);
  L.idx = take(size_t(A) * 4);
  L.gate = take(size_t(A) * 4);
  L.chunk_counts = take(size_t(p->n_routed) * (L.n_base > 0 ? L.n_base : 1) * 4);
  L.sub_base = take(L.fused ? size_t(p->n_routed) * (L.n_base > 0 ? L.n_base : 1) * L.subs_per_base * 4
                            : 0);
  L.counts = take(size_t(p->n_routed) * 4);
  L.offsets = take(size_t(p->n_routed + 1) * 4);
  L.mtiles = take(size_t(p->n_routed + 1) * 4);
  L.mtiles2 = take(size_t(p->n_routed + 1) * 4);
  L.mtiles64 = take(size_t(p->n_routed + 1) * 4);
  L.mt_hot = take(size_t(p->n_routed + 1) * 4);
  L.mt_cold = take(size_t(p->n_routed + 1) * 4);
  L.perm_src = take(size_t(A) * 4);
  L.inv_pos = take(size_t(A) * 4);
  L.xperm = take(size_t(A) * p->d * 2);
  L.hidden = take(size_t(A) * p->f * 2);
  L.yrouted = take(size_t(A) * p->d * 2);
  L.hshared = take(size_t(T) * nsf * 2);
  L.yshared = take(p->n_shared > 0 ? size_t(T) * p->d * 4 : 0);
  L.total = o;
  return L;
}

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 matrix (rows, cols) row-major, optionally stacked `batch` times; box of
// 64 columns (128 B, one swizzle row) x box_rows rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, uint64_t batch, uint64_t rows, uint64_t cols,
              uint32_t box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = batch > 0 ? 3 : 2;
  if (batch == 0) dims[2] = 1;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- launches
struct Launcher {
  moe_plan* p;
  cudaStream_t st;     // the caller's stream
  int status = MOE_OK;
  int grid_cap = INT_MAX;   // most CTAs a GEMM launch may use (SMs left to a concurrent one)

  void begin(const char* name, cudaStream_t s, const char* variant = "") {
    if (p->n_launch < kMaxKernels) {
      snprintf(p->names[p->n_launch], sizeof(p->names[0]), "%s%s", name, variant);
      if (p->timing) cudaEventRecord(p->ev[p->cur_set][2 * p->n_launch], s);
    }
  }
  bool end(const char* what, cudaStream_t s) {
    if (p->timing && p->n_launch < kMaxKernels)
      cudaEventRecord(p->ev[p->cur_set][2 * p->n_launch + 1], s);
    ++p->n_launch;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      status = fail(MOE_CUDA_ERROR, "%s launch failed: %s", what, cudaGetErrorString(e));
      return false;
    }
    return true;
  }
  void finish() {
    if (p->timing && p->n_launch <= kMaxKernels) {
      p->ring_launches[p->cur_set] = p->n_launch;
      ++p->timed_forwards;
    }
  }
};

// Every kernel is launched with programmatic stream serialisation, so that it
// can start its prologue while the previous kernel of the stream finishes; each
// kernel waits (griddepcontrol.wait) before reading what its predecessor wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// CTA-pair GEMM: clusters of two CTAs, one M=256 tile per pair; prm.group_mtiles
// must be the prefix of 256-row m-tiles and prm.n_tiles count tiles of
// pair_tile_cols(MODE, NW) columns. max_tiles bounds the number of tiles.
template <int MODE, int NW>
bool launch_gemm_pair(Launcher& L, cudaStream_t s, const char* name, const CUtensorMap& a,
                      const CUtensorMap& b0, const CUtensorMap& b1, const moe::GemmParams& prm,
                      int max_tiles) {
  const int num_groups = prm.group_offsets ? prm.num_groups : 1;
  const size_t smem = moe::gemm_pair_smem_bytes<NW>(num_groups);
  int pairs = (L.p->num_sms < L.grid_cap ? L.p->num_sms : L.grid_cap) / 2;
  if (max_tiles < pairs) pairs = max_tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(moe::kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  L.begin(name, s, NW == 2 ? "[pair512]" : "[pair]");
  cudaLaunchKernelEx(&cfg, moe::moe_gemm_pair_kernel<MODE, NW>, a, b0, b1, prm);
  return L.end(name, s);
}

// Launch a pair GEMM over N output columns with expected_mtiles 256-row
// m-tiles, choosing the tile width: wide (512 accumulator columns) tiles move a
// quarter fewer operand bytes per FLOP, but give fewer tiles and cannot overlap
// a whole tile's epilogue with the next tile's MMAs, so automatically they are
// used for long reductions (at least 64 k-blocks) with at least 3 waves of tiles.
template <int MODE>
bool launch_pair_auto(Launcher& L, cudaStream_t s, const char* name, const CUtensorMap& a,
                      const CUtensorMap& b0, const CUtensorMap& b1, moe::GemmParams prm,
                      int N, int expected_mtiles, int max_mtiles) {
  const int cols1 = moe::pair_tile_cols(MODE, 1), cols2 = moe::pair_tile_cols(MODE, 2);
  const int nt2 = (N + cols2 - 1) / cols2;
  bool wide = L.p->wide_tiles > 0;
  if (L.p->wide_tiles < 0)
    wide = prm.K >= 64 * moe::kBK &&
           static_cast<long long>(expected_mtiles) * nt2 >= 3LL * (L.p->num_sms / 2);
  if (wide) {
    prm.n_tiles = nt2;
    return launch_gemm_pair<MODE, 2>(L, s, name, a, b0, b1, prm, max_mtiles * nt2);
  }
  prm.n_tiles = (N + cols1 - 1) / cols1;
  return launch_gemm_pair<MODE, 1>(L, s, name, a, b0, b1, prm, max_mtiles * prm.n_tiles);
}

// Single-CTA GEMM with BN accumulator columns per tile. x (optional) holds the
// A, B0, B1 maps of the extra dense problem that prm.x_tiles describes;
// max_tiles bounds the grouped tiles only.
template <int MODE, int BN = 256, int TM = 128, int OCC = 1>
bool launch_gemm(Launcher& L, cudaStream_t s, const char* name, const CUtensorMap& a,
                 const CUtensorMap& b0, const CUtensorMap& b1, const moe::GemmParams& prm,
                 int max_tiles, const CUtensorMap* x = nullptr) {
  const int num_groups = prm.group_offsets ? prm.num_groups : 1;
  const size_t smem = moe::gemm_smem_bytes<BN, TM, OCC>(num_groups);
  const long long tiles = static_cast<long long>(max_tiles) + (x ? prm.x_tiles : 0);
  const int sms = (L.p->num_sms < L.grid_cap ? L.p->num_sms : L.grid_cap) * OCC;
  int grid = tiles < sms ? static_cast<int>(tiles) : sms;
  if (grid < 1) grid = 1;
  moe::GemmParams q = prm;
  if (!x) q.x_tiles = 0;
  // variant tag of a routed launch: output columns when not the widest tile,
  // 64-row tiles, two CTAs per SM, or the shared expert merged in (the dense
  // launches - router scores, shared expert - have fixed tiles)
  char tag[32] = "";
  const int out_cols = MODE == moe::kEpiSwiGLU ? BN / 2 : BN;
  const bool narrow =
      prm.group_offsets != nullptr && out_cols < (MODE == moe::kEpiSwiGLU ? 128 : 256);
  if (q.x_tiles > 0)
    snprintf(tag, sizeof(tag), "[+shared]");
  else if (narrow || TM == 64 || OCC == 2)
    snprintf(tag, sizeof(tag), "[%s%s%s%s%s]",
             narrow ? (out_cols == 32 ? "n32" : out_cols == 64 ? "n64" : "n128") : "",
             narrow && TM == 64 ? "," : "", TM == 64 ? "m64" : "",
             (narrow || TM == 64) && OCC == 2 ? "," : "", OCC == 2 ? "x2" : "");
  L.begin(name, s, tag);
  launch_pdl(moe::moe_gemm_kernel<MODE, BN, TM, OCC>, dim3(grid), dim3(moe::kGemmThreads), smem,
             s, a, b0, b1, x ? x[0] : a, x ? x[1] : b0, x ? x[2] : b1, q);
  return L.end(name, s);
}

// The same launch with one or two resident CTAs per SM (MOE_OPTION_CTAS_PER_SM).
template <int MODE, int BN = 256, int TM = 128>
bool launch_gemm_occ(bool two, Launcher& L, cudaStream_t s, const char* name,
                     const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                     const moe::GemmParams& prm, int max_tiles, const CUtensorMap* x = nullptr) {
  return two ? launch_gemm<MODE, BN, TM, 2>(L, s, name, a, b0, b1, prm, max_tiles, x)
             : launch_gemm<MODE, BN, TM, 1>(L, s, name, a, b0, b1, prm, max_tiles, x);
}

// Shared-memory attributes of a two-CTAs-per-SM instantiation: its dynamic
// shared memory, and the largest shared-memory carveout so that two fit.
template <int MODE, int BN, int TM>
cudaError_t set_occ2_attributes() {
  auto* k = moe::moe_gemm_kernel<MODE, BN, TM, 2>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(moe::gemm_smem_bytes<BN, TM, 2>(moe::kMaxRouted)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                             int(cudaSharedmemCarveoutMaxShared));
  return e;
}

typedef cudaFuncAttribute cudaAttr;

int set_kernel_attributes() {
  const int sp1 = int(moe::gemm_pair_smem_bytes<1>(moe::kMaxRouted));
  const int sp2 = int(moe::gemm_pair_smem_bytes<2>(moe::kMaxRouted));
  const cudaAttr attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  const cudaError_t ep[6] = {
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiSwiGLU, 1>, attr, sp1),
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiBF16, 1>, attr, sp1),
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiF32, 1>, attr, sp1),
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiSwiGLU, 2>, attr, sp2),
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiBF16, 2>, attr, sp2),
      cudaFuncSetAttribute(moe::moe_gemm_pair_kernel<moe::kEpiF32, 2>, attr, sp2)};
  for (cudaError_t e : ep)
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
  const size_t smem = moe::gemm_smem_bytes(moe::kMaxRouted);
  const cudaError_t e0[4] = {
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU, 128>, attr,
                           int(moe::gemm_smem_bytes<128>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU, 128, 64>, attr,
                           int(moe::gemm_smem_bytes<128, 64>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU, 256, 64>, attr,
                           int(moe::gemm_smem_bytes<256, 64>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiBF16, 256, 64>, attr,
                           int(moe::gemm_smem_bytes<256, 64>(moe::kMaxRouted)))};
  for (cudaError_t e : e0)
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
  cudaError_t e1 = cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  cudaError_t e2 = cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiBF16>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  cudaError_t e3 = cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiF32>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess)
    return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s",
                cudaGetErrorString(e1 != cudaSuccess ? e1 : (e2 != cudaSuccess ? e2 : e3)));
  const cudaError_t en[5] = {
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU, 64, 64>, attr,
                           int(moe::gemm_smem_bytes<64, 64>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiSwiGLU, 64, 128>, attr,
                           int(moe::gemm_smem_bytes<64, 128>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiBF16, 128, 64>, attr,
                           int(moe::gemm_smem_bytes<128, 64>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiBF16, 128, 128>, attr,
                           int(moe::gemm_smem_bytes<128, 128>(moe::kMaxRouted))),
      cudaFuncSetAttribute(moe::moe_gemm_kernel<moe::kEpiF32, 128, 128>, attr,
                           int(moe::gemm_smem_bytes<128, 128>(moe::kMaxRouted)))};
  for (cudaError_t e : en)
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
  const cudaError_t eo[10] = {set_occ2_attributes<moe::kEpiSwiGLU, 64, 64>(),
                             set_occ2_attributes<moe::kEpiSwiGLU, 64, 128>(),
                             set_occ2_attributes<moe::kEpiBF16, 128, 64>(),
                             set_occ2_attributes<moe::kEpiBF16, 128, 128>(),
                             set_occ2_attributes<moe::kEpiSwiGLU, 128, 64>(),
                             set_occ2_attributes<moe::kEpiSwiGLU, 128, 128>(),
                             set_occ2_attributes<moe::kEpiSwiGLU, 256, 64>(),
                             set_occ2_attributes<moe::kEpiSwiGLU, 256, 128>(),
                             set_occ2_attributes<moe::kEpiBF16, 256, 64>(),
                             set_occ2_attributes<moe::kEpiBF16, 256, 128>()};
  for (cudaError_t e : eo)
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
  const int rsm = 227 * 1024;
  const cudaError_t er[5] = {cudaFuncSetAttribute(moe::route_fused_kernel<1>, attr, rsm),
                             cudaFuncSetAttribute(moe::route_fused_kernel<2>, attr, rsm),
                             cudaFuncSetAttribute(moe::route_fused_kernel<4>, attr, rsm),
                             cudaFuncSetAttribute(moe::route_fused_kernel<8>, attr, rsm),
                             cudaFuncSetAttribute(moe::route_fused_kernel<16>, attr, rsm)};
  for (cudaError_t e : er)
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
  return MOE_OK;
}

// Fused router launch: clusters of rt.cs CTAs, one cluster per 128-token tile.
cudaError_t launch_router(const Layout& Lw, const moe::RouterParams& rt, const CUtensorMap& mX,
                          const CUtensorMap& mWg, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  const int mt = (rt.T + moe::kBM - 1) / moe::kBM;
  cfg.gridDim = dim3(static_cast<unsigned>(mt * rt.cs));
  cfg.blockDim = dim3(moe::kRtThreads);
  cfg.dynamicSmemBytes = Lw.rt_smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(rt.cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // scores per lane of the selection: N_r <= 32 * NPL
  const int npl = (rt.n_routed + 31) / 32;
  if (npl <= 1) return cudaLaunchKernelEx(&cfg, moe::route_fused_kernel<1>, mX, mWg, rt);
  if (npl <= 2) return cudaLaunchKernelEx(&cfg, moe::route_fused_kernel<2>, mX, mWg, rt);
  if (npl <= 4) return cudaLaunchKernelEx(&cfg, moe::route_fused_kernel<4>, mX, mWg, rt);
  if (npl <= 8) return cudaLaunchKernelEx(&cfg, moe::route_fused_kernel<8>, mX, mWg, rt);
  return cudaLaunchKernelEx(&cfg, moe::route_fused_kernel<16>, mX, mWg, rt);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Seats per expert for a forward over T tokens: the explicit capacity, or the
// capacity factor times an expert's even share of the T*top_k routed pairs,
// rounded up (at least 1); 0 means unlimited.
int64_t capacity_seats(const moe_plan* p, int64_t T) {
  if (p->capacity_permille > 0) {
    const int64_t num = p->capacity_permille * T * p->top_k;
    const int64_t den = 1000LL * p->n_routed;
    const int64_t c = (num + den - 1) / den;
    return c < 1 ? 1 : c;
  }
  return p->capacity;
}

}  // namespace

// ---------------------------------------------------------------------------
// Static scratch of the allocation-free forward (moe_forward_noalloc).
//
// Some callers cannot allocate device memory at all: a plugin inside a host
// application that owns the whole device-memory budget through its own pool,
// or a latency-critical loop where cudaMalloc would synchronise the device.
// For them the layer's scratch lives in one file-scope device array instead
// of a caller workspace. Every GPU that loads this library holds the array
// (kNoAllocScratchBytes) until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array in the current device's context. In host code
// the array's name only stands in for the symbol, so the address is looked up
// with the plan's device current, when the plan is created, and kept in the
// plan (which is bound to that context).
int noalloc_scratch_address(void** out) {
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess || !ptr) {
    cudaGetLastError();
    return fail(MOE_CUDA_ERROR, "cudaGetSymbolAddress of the static scratch failed: %s",
                cudaGetErrorString(e));
  }
  *out = ptr;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_plan_t moe_plan_create(int d, int f, int n_routed, int top_k, int n_shared, int renorm) {
  g_last_status = MOE_OK;
  if (d < 1 || f < 1 || n_routed < 1 || top_k < 1 || n_shared < 0 || top_k > n_routed) {
    fail(MOE_INVALID_CONFIG,
         "invalid expert configuration d=%d f=%d n_routed=%d top_k=%d n_shared=%d", d, f,
         n_routed, top_k, n_shared);
    return nullptr;
  }
  if (d % 8 || f % 8 || n_routed > moe::kMaxRouted || top_k > moe::kMaxTopK ||
      static_cast<long long>(n_shared) * f > (1LL << 24) || d > (1 << 24) || f > (1 << 24)) {
    fail(MOE_UNSUPPORTED,
         "unsupported shape: need d, f multiples of 8, n_routed <= %d, top_k <= %d, "
         "n_shared*f <= 2^24",
         moe::kMaxRouted, moe::kMaxTopK);
    return nullptr;
  }
  int dev = 0, sms = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    fail(MOE_CUDA_ERROR, "no usable CUDA device");
    return nullptr;
  }
  if (major != 10 || minor != 0) {
    fail(MOE_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev,
         major, minor);
    return nullptr;
  }
  if (set_kernel_attributes() != MOE_OK) return nullptr;
  if (!encode_fn()) {
    fail(MOE_CUDA_ERROR, "cuTensorMapEncodeTiled is not available from the driver");
    return nullptr;
  }
  moe_plan* p = new moe_plan();
  p->d = d;
  p->f = f;
  p->n_routed = n_routed;
  p->top_k = top_k;
  p->n_shared = n_shared;
  p->renorm = renorm ? 1 : 0;
  p->device = dev;
  p->num_sms = sms;
  if (cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&p->fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&p->join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    fail(MOE_CUDA_ERROR, "could not create the plan's side stream and events");
    moe_plan_destroy(p);
    return nullptr;
  }
  if (noalloc_scratch_address(&p->noalloc_scratch) != MOE_OK) {
    moe_plan_destroy(p);
    return nullptr;
  }
  return p;
}

int moe_last_status(void) { return g_last_status; }

int moe_plan_set_option(moe_plan_t p, int option, int64_t value) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  switch (option) {
    case MOE_OPTION_PAIR_MIN_ROWS:
      if (value < 0) return fail(MOE_INVALID_ARG, "pair_min_rows must be >= 0");
      p->pair_min_rows_plain = p->pair_min_rows_swiglu = value;
      return MOE_OK;
    case MOE_OPTION_WIDE_TILES:
      if (value < -1 || value > 1) return fail(MOE_INVALID_ARG, "wide_tiles must be -1, 0 or 1");
      p->wide_tiles = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_MERGE_SHARED:
      if (value < -1 || value > 1)
        return fail(MOE_INVALID_ARG, "merge_shared must be -1, 0 or 1");
      p->merge_shared = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_TEST_WAIT_TIMEOUT:
      if (value < 0 || value > 1) return fail(MOE_INVALID_ARG, "test hook must be 0 or 1");
      p->test_withhold = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_BIAS_SELECTION_ONLY:
      if (value < 0 || value > 1) return fail(MOE_INVALID_ARG, "bias selection-only must be 0 or 1");
      p->bias_select_only = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_EXPERT_CAPACITY:
      if (value < 0) return fail(MOE_INVALID_ARG, "expert capacity must be >= 0");
      p->capacity = value;
      p->capacity_permille = 0;
      return MOE_OK;
    case MOE_OPTION_SHARED_CONCURRENT:
      if (value < -1 || value > 1)
        return fail(MOE_INVALID_ARG, "shared_concurrent must be -1, 0 or 1");
      p->shared_concurrent = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_INTERLEAVE:
      if (value < -1 || value > 1) return fail(MOE_INVALID_ARG, "interleave must be -1, 0 or 1");
      p->interleave = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_CTAS_PER_SM:
      if (value < 0 || value > 2) return fail(MOE_INVALID_ARG, "ctas per SM must be 0, 1 or 2");
      p->ctas_per_sm = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_TILE_ROWS:
      if (value != 0 && value != 64 && value != 128)
        return fail(MOE_INVALID_ARG, "tile rows must be 0, 64 or 128");
      p->tile_rows = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_GATHER_ROWS:
      if (value < -1 || value > 1) return fail(MOE_INVALID_ARG, "gather_rows must be -1, 0 or 1");
      p->gather_rows = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_DOWN_TILE_COLS:
      if (value != 0 && value != 128 && value != 256)
        return fail(MOE_INVALID_ARG, "down tile columns must be 0, 128 or 256");
      p->down_tile_cols = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_SWIGLU_TILE_COLS:
      if (value != 0 && value != 32 && value != 64 && value != 128)
        return fail(MOE_INVALID_ARG, "swiglu tile columns must be 0, 32, 64 or 128");
      p->swiglu_tile_cols = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_FUSED_ROUTER:
      if (value < -1 || value > 1) return fail(MOE_INVALID_ARG, "fused_router must be -1, 0 or 1");
      p->fused_router = static_cast<int>(value);
      return MOE_OK;
    case MOE_OPTION_CAPACITY_FACTOR_PERMILLE:
      if (value < 0 || value > (1LL << 20))
        return fail(MOE_INVALID_ARG, "capacity factor (permille) must be in [0, 2^20]");
      p->capacity_permille = value;
      p->capacity = 0;
      return MOE_OK;
    default:
      return fail(MOE_INVALID_ARG, "unknown option %d", option);
  }
}

int moe_plan_set_logit_bias(moe_plan_t p, const float* bias) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u))
    return fail(MOE_INVALID_ARG, "bias must be 4-byte aligned");
  p->bias = bias;
  return MOE_OK;
}

size_t moe_workspace_bytes(moe_plan_t p, int64_t T) {
  if (!p || T < 0) return 0;
  return make_layout(p, T).total;
}

int moe_plan_set_workspace(moe_plan_t p, void* ws, size_t bytes) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_INVALID_ARG, "workspace must be 256-byte aligned");
  p->ws = static_cast<char*>(ws);
  p->ws_bytes = ws ? bytes : 0;
  p->last_T = -1;
  if (ws) {
    cudaError_t e = cudaMemset(ws, 0, 256);   // device status word
    if (e != cudaSuccess) return fail(MOE_CUDA_ERROR, "cudaMemset: %s", cudaGetErrorString(e));
  }
  return MOE_OK;
}

int moe_forward(moe_plan_t p, int64_t T, const moe_bf16_t* x, const moe_bf16_t* W_g,
                const moe_bf16_t* W1, const moe_bf16_t* W3, const moe_bf16_t* W2,
                const moe_bf16_t* W1s, const moe_bf16_t* W3s, const moe_bf16_t* W2s,
                moe_bf16_t* out, void* stream) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (T < 0) return fail(MOE_INVALID_ARG, "T must be >= 0");
  if (T == 0) {
    p->n_launch = 0;
    p->last_T = 0;
    return MOE_OK;
  }
  if (T * p->top_k > (1LL << 30))
    return fail(MOE_UNSUPPORTED, "T*top_k = %lld exceeds 2^30 rows", (long long)(T * p->top_k));
  if (!x || !W_g || !W1 || !W3 || !W2 || !out)
    return fail(MOE_INVALID_ARG, "x, W_g, W1, W3, W2 and out must be non-null");
  if ((p->n_shared > 0) != (W1s != nullptr) || (p->n_shared > 0) != (W3s != nullptr) ||
      (p->n_shared > 0) != (W2s != nullptr))
    return fail(MOE_INVALID_ARG, "W1s, W3s, W2s must be non-null exactly when n_shared > 0");
  const void* ptrs[] = {x, W_g, W1, W3, W2, out, W1s, W3s, W2s};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return fail(MOE_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!p->ws) return fail(MOE_INVALID_ARG, "no workspace set (moe_plan_set_workspace)");
  const Layout Lw = make_layout(p, T);
  if (Lw.total > p->ws_bytes)
    return fail(MOE_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, T=%lld needs %zu",
                p->ws_bytes, (long long)T, Lw.total);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device)
    return fail(MOE_INVALID_ARG, "plan was created on device %d, current device is %d",
                p->device, dev);
  if (p->timing && !p->events_made) {
    for (int r = 0; r < kTimingRing; ++r)
      for (int i = 0; i < 2 * kMaxKernels; ++i) cudaEventCreate(&p->ev[r][i]);
    p->events_made = true;
  }
  if (p->timing) p->cur_set = static_cast<int>(p->timed_forwards % kTimingRing);

  const int d = p->d, f = p->f, nr = p->n_routed, k = p->top_k;
  const int nsf = p->n_shared * f;
  const int64_t A = T * k;
  char* ws = p->ws;
  int* status = reinterpret_cast<int*>(ws + Lw.status);
  float* scores = reinterpret_cast<float*>(ws + Lw.scores);
  int* idx = reinterpret_cast<int*>(ws + Lw.idx);
  float* gate = reinterpret_cast<float*>(ws + Lw.gate);
  int* chunk_counts = reinterpret_cast<int*>(ws + Lw.chunk_counts);
  int* sub_base = Lw.fused ? reinterpret_cast<int*>(ws + Lw.sub_base) : nullptr;
  int* counts = reinterpret_cast<int*>(ws + Lw.counts);
  int* offsets = reinterpret_cast<int*>(ws + Lw.offsets);
  int* mtiles = reinterpret_cast<int*>(ws + Lw.mtiles);
  int* mtiles2 = reinterpret_cast<int*>(ws + Lw.mtiles2);
  int* mtiles64 = reinterpret_cast<int*>(ws + Lw.mtiles64);
  int* mt_hot = reinterpret_cast<int*>(ws + Lw.mt_hot);
  int* mt_cold = reinterpret_cast<int*>(ws + Lw.mt_cold);
  int* perm_src = reinterpret_cast<int*>(ws + Lw.perm_src);
  int* inv_pos = reinterpret_cast<int*>(ws + Lw.inv_pos);
  void* xperm = ws + Lw.xperm;
  void* hidden = ws + Lw.hidden;
  void* yrouted = ws + Lw.yrouted;
  void* hshared = ws + Lw.hshared;
  float* yshared = p->n_shared > 0 ? reinterpret_cast<float*>(ws + Lw.yshared) : nullptr;

  CUtensorMap mX, mWg, mXp, mW1, mW3, mH, mW2, mW1s, mW3s, mHs, mW2s;
  bool ok = make_map(&mX, x, 0, T, d) && make_map(&mWg, W_g, 1, nr, d) &&
            make_map(&mXp, xperm, 0, A, d) && make_map(&mW1, W1, nr, f, d) &&
            make_map(&mW3, W3, nr, f, d) && make_map(&mH, hidden, 0, A, f) &&
            make_map(&mW2, W2, nr, d, f);
  if (ok && p->n_shared > 0)
    ok = make_map(&mW1s, W1s, 1, nsf, d) && make_map(&mW3s, W3s, 1, nsf, d) &&
         make_map(&mHs, hshared, 0, T, nsf) && make_map(&mW2s, W2s, 1, d, nsf);
  if (!ok) return fail(MOE_CUDA_ERROR, "cuTensorMapEncodeTiled rejected a tensor map");

  cudaGetLastError();  // clear any stale error so launch checks are precise
  p->n_launch = 0;
  p->last_T = T;
  Launcher L{p, static_cast<cudaStream_t>(stream)};

  cudaStream_t main_st = L.st;
  // The shared SwiGLU (coefficient 1, outside the routing) is independent of
  // the routing. When it is small (at most half the SMs' worth of tiles, the
  // decode regime) it runs as extra tiles of the routed GEMM launches, which
  // have room for them in their last wave, or else on the plan's side stream,
  // forked here and joined before the combine, beside the latency-bound
  // routing kernels (where it spills into the first routed GEMM wave's SMs and
  // the join costs the combine its early launch); a larger one would take SMs
  // from the routing chain, so it runs inline on the main stream after the
  // routed GEMMs instead.
  const int shared_mt = static_cast<int>((T + 127) / 128);
  // seats per expert and the expected rows per expert group (a division: the
  // thresholds may be huge, and a product with N_r could overflow)
  const int64_t seats = capacity_seats(p, T);
  const int seat_limit = seats > 0 && seats < INT_MAX ? static_cast<int>(seats) : INT_MAX;
  const long long rows_per_expert = A / nr < seat_limit ? A / nr : seat_limit;
  const bool shared_small =
      p->n_shared > 0 && shared_mt * ((nsf + 127) / 128) <= p->num_sms / 2;
  const bool routed_pair_swiglu = rows_per_expert >= p->pair_min_rows_swiglu;
  const bool shared_pair = static_cast<long long>(T) >= p->pair_min_rows_swiglu;
  // automatic merging leaves explicitly chosen routed tile shapes alone (a
  // merged launch runs the default 128-row x 256-column tiles)
  const bool default_tiles = (p->swiglu_tile_cols == 0 || p->swiglu_tile_cols == 128) &&
                             p->tile_rows != 64 && p->ctas_per_sm != 2;
  const bool merge_pref =
      p->merge_shared == 1 || (p->merge_shared == -1 && shared_small && default_tiles);
  const bool merge_small = shared_small && merge_pref && !routed_pair_swiglu && !shared_pair;
  // A larger shared expert runs beside the routed GEMMs when those stream
  // weights (few rows per expert: their tensor pipes idle most of the time):
  // forked at the start onto shared_sms SMs, sized so that its tensor-bound
  // work takes about as long as the routed weight stream on the other SMs
  // (at about 253 FLOP per HBM byte, the measured B200 ridge); the routed
  // GEMMs are capped to the remaining SMs.
  int shared_sms = 0;
  if (p->n_shared > 0 && !shared_small &&
      p->shared_concurrent == 1) {
    const double t_sh = 6.0 * double(T) * d * nsf / 253.0;
    const double t_r = 6.0 * double(d) * f * (A < nr ? A : nr);
    int sm = static_cast<int>(1.5 * p->num_sms * t_sh / (t_sh + t_r)) + 1;
    sm = sm < 8 ? 8 : (sm > p->num_sms / 4 ? p->num_sms / 4 : sm);
    shared_sms = sm;
  }
  const bool shared_forked = (shared_small && !merge_small) || shared_sms > 0;
  cudaStream_t shared_st = shared_forked ? p->side : main_st;
  const int shared_mt2 = static_cast<int>((T + 255) / 256);
  auto launch_shared_gate_up = [&]() -> int {
    moe::GemmParams g{};
    g.dense_rows = static_cast<int>(T);
    g.K = d;
    g.N = nsf;
    g.n_tiles = (nsf + 127) / 128;
    g.out = hshared;
    g.ldo = nsf;
    g.status = status;
    g.k_splits = 1;
    g.kb_per_split = (d + moe::kBK - 1) / moe::kBK;
    if (shared_pair ? !launch_pair_auto<moe::kEpiSwiGLU>(L, shared_st, "shared_gate_up", mX, mW1s,
                                                         mW3s, g, nsf, shared_mt2, shared_mt2)
                    : !launch_gemm<moe::kEpiSwiGLU>(L, shared_st, "shared_gate_up", mX, mW1s, mW3s,
                                                    g, shared_mt * g.n_tiles))
      return L.status;
    return MOE_OK;
  };
  auto launch_shared_down = [&]() -> int {
    moe::GemmParams h{};
    h.dense_rows = static_cast<int>(T);
    h.K = nsf;
    h.N = d;
    h.n_tiles = (d + 255) / 256;
    h.out = yshared;
    h.ldo = d;
    h.status = status;
    h.k_splits = 1;
    h.kb_per_split = (nsf + moe::kBK - 1) / moe::kBK;
    if (shared_pair ? !launch_pair_auto<moe::kEpiF32>(L, shared_st, "shared_down", mHs, mW2s, mW2s,
                                                      h, d, shared_mt2, shared_mt2)
                    : !launch_gemm<moe::kEpiF32>(L, shared_st, "shared_down", mHs, mW2s, mW2s, h,
                                                 shared_mt * h.n_tiles))
      return L.status;
    return MOE_OK;
  };
  auto launch_shared = [&]() -> int {
    if (launch_shared_gate_up() != MOE_OK) return L.status;
    return launch_shared_down();
  };
  if (shared_forked) {
    if (cudaEventRecord(p->fork, main_st) != cudaSuccess ||
        cudaStreamWaitEvent(p->side, p->fork, 0) != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "fork of the shared-expert stream failed");
    if (shared_sms > 0) L.grid_cap = shared_sms;
    if (launch_shared() != MOE_OK) return L.status;
    L.grid_cap = INT_MAX;
    if (cudaEventRecord(p->join, p->side) != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "join record of the shared-expert stream failed");
  }
  if (Lw.fused) {
    // 1-3. fused router: scores on the tensor core, softmax, top-k, gates, the
    //      chunk histogram and (when small) its scan, in one launch
    CUtensorMap mWgR;
    // rank-2 map (the kernel issues 2-D loads), boxes of rt.box_rows expert rows
    if (!make_map(&mWgR, W_g, 0, nr, d, static_cast<uint32_t>(Lw.rt.box_rows)))
      return fail(MOE_CUDA_ERROR, "cuTensorMapEncodeTiled rejected the router map");
    moe::RouterParams rt = Lw.rt;
    rt.bias = p->bias;
    rt.idx = idx;
    rt.gate = gate;
    rt.tile_counts = chunk_counts;
    rt.sub_base = sub_base;
    rt.counts = counts;
    rt.ticket = reinterpret_cast<int*>(ws + Lw.ticket);
    rt.status = status;
    L.begin("route_fused", main_st);
    launch_router(Lw, rt, mX, mWgR, main_st);
    if (!L.end("route_fused", main_st)) return L.status;
  } else {
  // 1. router scores s = x W_g^T (fp32 partial sums of a split-K), dense over T rows
  {
    moe::GemmParams g{};
    g.dense_rows = static_cast<int>(T);
    g.K = d;
    g.N = nr;
    g.n_tiles = (nr + kRouterCols - 1) / kRouterCols;
    g.out = scores;
    g.ldo = Lw.lds;
    g.status = status;
    g.k_splits = Lw.router_splits;
    g.kb_per_split = Lw.router_kb_per;
    g.split_stride = static_cast<long long>(T) * Lw.lds;
    const int tiles = static_cast<int>((T + 127) / 128) * g.n_tiles * g.k_splits;
    if (!launch_gemm<moe::kEpiF32, kRouterCols>(L, main_st, "router_gemm", mX, mWg, mWg, g,
                                                 tiles))
      return L.status;
  }
  // 2. softmax + top-k + gates + per-chunk histogram
  {
    const size_t smem = size_t(nr) * 4;
    const int npl = (nr + 31) / 32;
    const int sp = Lw.router_splits;
    L.begin("route_topk", main_st);
#define MOE_TOPK(N, S)                                                                      \
  launch_pdl(moe::route_topk_kernel<N, S>, dim3(Lw.n_chunks), dim3(moe::kRouteThreads),     \
             smem, main_st, (const float*)scores, Lw.lds, sp,                               \
             static_cast<long long>(T) * Lw.lds, p->bias, static_cast<int>(T), nr, k,       \
             p->renorm, p->bias_select_only, Lw.tpc, Lw.n_chunks, idx, gate, chunk_counts)
#define MOE_TOPK_S(N)                                                                       \
  if (sp <= 1) MOE_TOPK(N, 1);                                                              \
  else if (sp <= 2) MOE_TOPK(N, 2);                                                         \
  else MOE_TOPK(N, 4)
    if (npl <= 1) { MOE_TOPK_S(1); }
    else if (npl <= 2) { MOE_TOPK_S(2); }
    else if (npl <= 4) { MOE_TOPK_S(4); }
    else if (npl <= 8) { MOE_TOPK_S(8); }
    else if (npl <= 16) { MOE_TOPK_S(16); }
    else if (sp <= 1) MOE_TOPK(32, 1);
    else if (sp <= 2) MOE_TOPK(32, 2);
    else MOE_TOPK(32, 4);
#undef MOE_TOPK_S
#undef MOE_TOPK
    if (!L.end("route_topk", main_st)) return L.status;
  }
  }
  // 3. per-expert prefix over chunks and expert totals (one warp per expert),
  //    unless the fused router's last CTA did it
  if (!(Lw.fused && Lw.rt.fold_scan)) {
    const int warps = moe::kRouteThreads / 32;
    L.begin("route_scan", main_st);
    launch_pdl(moe::route_scan_kernel, dim3((nr + warps - 1) / warps), dim3(moe::kRouteThreads),
               0, main_st, chunk_counts, Lw.n_base, nr, counts);
    if (!L.end("route_scan", main_st)) return L.status;
  }
  const int max_mtiles = static_cast<int>((A + 127) / 128 + (A < nr ? A : nr));
  const int max_mtiles2 = static_cast<int>((A + 255) / 256 + (A < nr ? A : nr));
  const bool routed_pair = rows_per_expert >= p->pair_min_rows_plain;
  const int expected_mtiles2 = static_cast<int>((A + 255) / 256);
  // A shared expert that is not forked can run as extra dense tiles of the
  // routed single-CTA launches, spread among the grouped tiles: the shared
  // GEMMs then need no launches (and tails) of their own, and a small one
  // fills the routed launches' last waves.
  const bool merge_ok = p->n_shared > 0 && !shared_forked && !shared_pair && merge_pref;
  const bool merge_gu = merge_ok && !routed_pair_swiglu;
  const bool merge_dn = merge_gu && !routed_pair;
  // Tile shapes of the routed GEMMs (step 5 and 6 below). Automatically
  //    every single-CTA routed GEMM uses the widest tile (128 rows x 256
  //    accumulator columns, one CTA per SM), also when the groups hold a few
  //    rows and the GEMM streams weights: on B200 one tcgen05.mma instruction
  //    occupies the issuing thread about 95 cycles whatever its size, so an
  //    N=256 MMA moves twice the weight bytes per cycle of an N=128 one.
  //    Measured on the 512-expert decode step: gate/up 64 us with these tiles,
  //    70 us with 64x128 tiles, 72 us with 64x64 tiles at two CTAs per SM, 88
  //    us with 64x256 tiles at two CTAs per SM. Narrower or shorter tiles and
  //    two CTAs per SM stay available as options.
  const bool single_gu = !routed_pair_swiglu && !merge_gu;
  const bool single_dn = !routed_pair && !merge_dn;
  const bool occ2_gu = single_gu && p->ctas_per_sm == 2;
  const bool occ2_dn = single_dn && p->ctas_per_sm == 2;
  int gu_cols = 128;   // output columns of a gate/up tile
  if (single_gu && p->swiglu_tile_cols != 0) gu_cols = p->swiglu_tile_cols;
  int dn_cols = 256;   // output columns of a down tile
  if (single_dn && p->down_tile_cols != 0) dn_cols = p->down_tile_cols;
  const bool narrow_gu = gu_cols < 128;
  const bool short_gu = single_gu && p->tile_rows == 64;
  const bool short_dn = single_dn && p->tile_rows == 64;
  const int max_mtiles64 = static_cast<int>((A + 63) / 64 + (A < nr ? A : nr));
  // 128-row single-CTA routed GEMMs in the weight-streaming regime run the
  // tiles of experts with several m-blocks (tensor-heavy: each weight tile is
  // reused through L2) spread evenly among the weight-streaming experts' tiles,
  // so that tensor and HBM work overlap instead of alternating
  // (not when every group streams: decode 161.8 vs 163.7 us without it)
  const bool interleave =
      p->interleave == 1 ||
      (p->interleave == -1 && rows_per_expert >= 32 && rows_per_expert < 192);
  // The single-CTA gate/up GEMM can gather its rows from x itself (through
  // perm_src), so that the permutation kernel writes no row copies. Measured
  // on B200: the 512-expert decode step 1-3% faster with it; the tensor-bound
  // layers slower (the cp.async gather of a 16 KB A stage costs the producer
  // warps far more than one TMA box: coarse +37%, DeepSeekMoE-small +8%); and
  // DeepSeek-V3 prefill 7% slower although 16% fewer cycles, because the extra
  // load traffic lowers the power-capped clock (1046 vs 1338 MHz). So
  // automatically only below 32 expected rows per expert.
  const bool gather_rows =
      (p->gather_rows == 1 || (p->gather_rows == -1 && rows_per_expert < 32)) &&
      !routed_pair_swiglu;
  // 4. offsets + m-tile prefix, stable permutation, 16-byte row copies (with a
  //    seat limit, only each expert's first `capacity` pairs get rows; none
  //    when the gate/up GEMM gathers them)
  {
    const size_t smem = size_t(moe::kMaxRouted + nr) * 4 + size_t(2) * Lw.tpc * k * 4;
    // split the row copy into column slices of at least 32 vectors so that
    // about four blocks per SM copy (one block per chunk leaves most SMs with
    // one or two resident blocks, too few loads in flight)
    int slices = (4 * p->num_sms) / Lw.n_chunks;
    const int max_slices = d / 8 / 32;
    if (slices > max_slices) slices = max_slices;
    if (slices < 1 || gather_rows) slices = 1;
    // the m-tile prefixes the routed GEMM launches below will read: 128-row
    // tiles always, 256-row (CTA pair), 64-row and the two interleave classes
    // only when used
    const int pass_mask = 1 | ((routed_pair_swiglu || routed_pair) ? 2 : 0) |
                          ((short_gu || short_dn) ? 4 : 0) | (interleave ? 8 | 16 : 0);
    L.begin("route_scatter", main_st);
    launch_pdl(moe::route_scatter_kernel, dim3(Lw.n_chunks, slices), dim3(moe::kRouteThreads), smem,
               main_st, (const int*)idx, (const int*)chunk_counts, Lw.n_base,
               (const int*)sub_base, Lw.subs_per_base, Lw.sub_tokens, (const int*)counts,
               static_cast<int>(T), k, nr, Lw.tpc, Lw.n_chunks, moe::kBM, seat_limit,
               reinterpret_cast<const uint4*>(x), d / 8,
               gather_rows ? static_cast<uint4*>(nullptr) : reinterpret_cast<uint4*>(xperm),
               perm_src, inv_pos, offsets, mtiles, mtiles2, mtiles64, mt_hot, mt_cold, pass_mask,
               status);
    if (!L.end("route_scatter", main_st)) return L.status;
  }
  const CUtensorMap xgu[3] = {mX, mW1s, mW3s};
  const CUtensorMap xdn[3] = {mHs, mW2s, mW2s};
  // the routed GEMMs leave the concurrent shared expert its SMs
  if (shared_sms > 0) L.grid_cap = p->num_sms - shared_sms;
  CUtensorMap mXp64, mH64;
  if ((short_gu && !make_map(&mXp64, xperm, 0, A, d, 64)) ||
      (short_dn && !make_map(&mH64, hidden, 0, A, f, 64)))
    return fail(MOE_CUDA_ERROR, "cuTensorMapEncodeTiled rejected a tensor map");
  {
    moe::GemmParams g{};
    g.group_offsets = offsets;
    g.group_mtiles = routed_pair_swiglu ? mtiles2 : (short_gu ? mtiles64 : mtiles);
    g.num_groups = nr;
    g.K = d;
    g.N = f;
    g.n_tiles = (f + gu_cols - 1) / gu_cols;
    g.out = hidden;
    g.ldo = f;
    g.status = status;
    g.k_splits = 1;
    g.kb_per_split = (d + moe::kBK - 1) / moe::kBK;
    if (!routed_pair_swiglu) {
      g.test_withhold = p->test_withhold;
      p->test_withhold = 0;
    }
    if (gather_rows) {
      g.gather_x = reinterpret_cast<const uint4*>(x);
      g.gather_src = perm_src;
      g.gather_ld_vec = d / 8;
      g.gather_T = static_cast<int>(T);
    }
    if (merge_gu) {
      g.x_tiles = shared_mt * ((nsf + 127) / 128);
      g.x_rows = static_cast<int>(T);
      g.x_K = d;
      g.x_N = nsf;
      g.x_out = hshared;
      g.x_ldo = nsf;
    }
    const int mtmax = short_gu ? max_mtiles64 : max_mtiles;
    bool launched;
    if (narrow_gu) {
      CUtensorMap mW1n, mW3n;
      const uint32_t box = static_cast<uint32_t>(gu_cols);
      if (!make_map(&mW1n, W1, nr, f, d, box) || !make_map(&mW3n, W3, nr, f, d, box))
        return fail(MOE_CUDA_ERROR, "cuTensorMapEncodeTiled rejected a tensor map");
      if (gu_cols == 32)
        launched = short_gu
                       ? launch_gemm_occ<moe::kEpiSwiGLU, 64, 64>(occ2_gu, L, main_st,
                                                                  "grouped_gate_up", mXp64, mW1n,
                                                                  mW3n, g, mtmax * g.n_tiles)
                       : launch_gemm_occ<moe::kEpiSwiGLU, 64>(occ2_gu, L, main_st,
                                                              "grouped_gate_up", mXp, mW1n, mW3n,
                                                              g, mtmax * g.n_tiles);
      else
        launched = short_gu
                       ? launch_gemm_occ<moe::kEpiSwiGLU, 128, 64>(occ2_gu, L, main_st,
                                                                   "grouped_gate_up", mXp64,
                                                                   mW1n, mW3n, g,
                                                                   mtmax * g.n_tiles)
                       : launch_gemm_occ<moe::kEpiSwiGLU, 128>(occ2_gu, L, main_st,
                                                               "grouped_gate_up", mXp, mW1n,
                                                               mW3n, g, mtmax * g.n_tiles);
    } else if (routed_pair_swiglu) {
      launched = launch_pair_auto<moe::kEpiSwiGLU>(L, main_st, "grouped_gate_up", mXp, mW1, mW3, g,
                                                   f, expected_mtiles2, max_mtiles2);
    } else if (short_gu) {
      launched = launch_gemm_occ<moe::kEpiSwiGLU, 256, 64>(occ2_gu, L, main_st, "grouped_gate_up",
                                                           mXp64, mW1, mW3, g, mtmax * g.n_tiles);
    } else {
      if (interleave && !merge_gu) {
        g.group_mtiles = mt_hot;
        g.group_mtiles_b = mt_cold;
      }
      launched = launch_gemm_occ<moe::kEpiSwiGLU>(occ2_gu, L, main_st, "grouped_gate_up", mXp, mW1,
                                                  mW3, g, mtmax * g.n_tiles,
                                                  merge_gu ? xgu : nullptr);
    }
    if (!launched) return L.status;
  }
  // 6. grouped down GEMM
  {
    moe::GemmParams g{};
    g.group_offsets = offsets;
    g.group_mtiles = routed_pair ? mtiles2 : (short_dn ? mtiles64 : mtiles);
    g.num_groups = nr;
    g.K = f;
    g.N = d;
    g.n_tiles = (d + dn_cols - 1) / dn_cols;
    g.out = yrouted;
    g.ldo = d;
    g.status = status;
    g.k_splits = 1;
    g.kb_per_split = (f + moe::kBK - 1) / moe::kBK;
    if (merge_dn) {
      g.x_tiles = shared_mt * ((d + 255) / 256);
      g.x_rows = static_cast<int>(T);
      g.x_K = nsf;
      g.x_N = d;
      g.x_out = yshared;
      g.x_ldo = d;
      g.x_out_f32 = 1;
    }
    bool launched;
    if (routed_pair)
      launched = launch_pair_auto<moe::kEpiBF16>(L, main_st, "grouped_down", mH, mW2, mW2, g, d,
                                                 expected_mtiles2, max_mtiles2);
    else if (short_dn)
      launched = dn_cols == 128
                     ? launch_gemm_occ<moe::kEpiBF16, 128, 64>(occ2_dn, L, main_st, "grouped_down",
                                                               mH64, mW2, mW2, g,
                                                               max_mtiles64 * g.n_tiles)
                     : launch_gemm_occ<moe::kEpiBF16, 256, 64>(occ2_dn, L, main_st, "grouped_down",
                                                               mH64, mW2, mW2, g,
                                                               max_mtiles64 * g.n_tiles);
    else {
      if (interleave && !merge_dn) {
        g.group_mtiles = mt_hot;
        g.group_mtiles_b = mt_cold;
      }
      launched = dn_cols == 128
                     ? launch_gemm_occ<moe::kEpiBF16, 128>(occ2_dn, L, main_st, "grouped_down",
                                                           mH, mW2, mW2, g, max_mtiles * g.n_tiles)
                     : launch_gemm_occ<moe::kEpiBF16>(occ2_dn, L, main_st, "grouped_down", mH,
                                                      mW2, mW2, g, max_mtiles * g.n_tiles,
                                                      merge_dn ? xdn : nullptr);
    }
    if (!launched) return L.status;
  }
  L.grid_cap = INT_MAX;
  // 7. the shared expert (inline, merged, or joined from the side stream), then
  //    the weighted combine + shared add with one bf16 rounding
  if (p->n_shared > 0 && !shared_forked) {
    if (!merge_gu && launch_shared_gate_up() != MOE_OK) return L.status;
    if (!merge_dn && launch_shared_down() != MOE_OK) return L.status;
  }
  if (shared_forked && cudaStreamWaitEvent(main_st, p->join, 0) != cudaSuccess)
    return fail(MOE_CUDA_ERROR, "join of the shared-expert stream failed");
  {
    const int d_vec = d / 8;
    const dim3 grid(static_cast<unsigned>(T),
                    static_cast<unsigned>((d_vec + moe::kCombineCols - 1) / moe::kCombineCols));
    L.begin("combine", main_st);
    launch_pdl(moe::combine_kernel, grid, dim3(moe::kCombineThreads), 0, main_st,
               reinterpret_cast<const uint4*>(yrouted), (const float*)yshared,
               (const int*)inv_pos, (const float*)gate, k, d_vec, reinterpret_cast<uint4*>(out),
               Lw.fused ? reinterpret_cast<int*>(ws + Lw.ticket) : static_cast<int*>(nullptr));
    if (!L.end("combine", main_st)) return L.status;
  }
  L.finish();
  return MOE_OK;
}

int moe_get_routing(moe_plan_t p, int64_t T, int32_t* idx, float* w, int32_t* counts,
                    int32_t* offsets, void* stream) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (T != p->last_T || T < 0) return fail(MOE_INVALID_ARG, "T does not match the last forward");
  if (T == 0) return MOE_OK;
  const Layout Lw = make_layout(p, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t A = size_t(T) * p->top_k;
  cudaError_t e = cudaSuccess;
  if (idx && e == cudaSuccess)
    e = cudaMemcpyAsync(idx, p->ws + Lw.idx, A * 4, cudaMemcpyDeviceToDevice, st);
  if (w && e == cudaSuccess)
    e = cudaMemcpyAsync(w, p->ws + Lw.gate, A * 4, cudaMemcpyDeviceToDevice, st);
  if (counts && e == cudaSuccess)
    e = cudaMemcpyAsync(counts, p->ws + Lw.counts, size_t(p->n_routed) * 4,
                        cudaMemcpyDeviceToDevice, st);
  if (offsets && e == cudaSuccess)
    e = cudaMemcpyAsync(offsets, p->ws + Lw.offsets, size_t(p->n_routed + 1) * 4,
                        cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(MOE_CUDA_ERROR, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
  return MOE_OK;
}

int moe_get_permutation(moe_plan_t p, int64_t T, int32_t* perm_src, int32_t* inv_pos,
                        void* stream) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (T != p->last_T || T < 0) return fail(MOE_INVALID_ARG, "T does not match the last forward");
  if (T == 0) return MOE_OK;
  const Layout Lw = make_layout(p, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t A = size_t(T) * p->top_k;
  cudaError_t e = cudaSuccess;
  if (perm_src)
    e = cudaMemcpyAsync(perm_src, p->ws + Lw.perm_src, A * 4, cudaMemcpyDeviceToDevice, st);
  if (inv_pos && e == cudaSuccess)
    e = cudaMemcpyAsync(inv_pos, p->ws + Lw.inv_pos, A * 4, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(MOE_CUDA_ERROR, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
  return MOE_OK;
}

int moe_plan_device_status(moe_plan_t p) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  // the plan's workspace, and the static scratch when this plan's allocation-free
  // forwards have used it since the last read
  void* words[2] = {p->ws, p->noalloc_used ? p->noalloc_scratch : nullptr};
  int worst = MOE_OK;
  for (void* w : words) {
    if (!w) continue;
    int v = 0;
    cudaError_t e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(w, 0, sizeof(int));
    if (e != cudaSuccess)
      return fail(MOE_CUDA_ERROR, "device status read: %s", cudaGetErrorString(e));
    if (v != MOE_OK) worst = v;
  }
  p->noalloc_used = false;
  if (worst != MOE_OK)
    return fail(worst, "device status %d: %s", worst, moe_strerror(worst));
  return MOE_OK;
}

int moe_plan_enable_timing(moe_plan_t p, int enable) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  p->timing = enable != 0;
  return MOE_OK;
}

int moe_plan_kernel_times(moe_plan_t p, int back, float* ms, int cap) {
  if (!p) return -fail(MOE_INVALID_ARG, "null plan");
  if (!p->events_made) return -fail(MOE_INVALID_ARG, "timing is not enabled");
  if (back < 0 || back >= kTimingRing || back >= p->timed_forwards)
    return -fail(MOE_INVALID_ARG, "no timed forward %d steps back", back);
  const int set = static_cast<int>((p->timed_forwards - 1 - back) % kTimingRing);
  const int n = p->ring_launches[set];
  if (n == 0) return 0;
  // the last kernel (the combine) runs after every other one (it joins the
  // side stream when the shared expert was forked), so its end event is last
  cudaError_t e = cudaEventSynchronize(p->ev[set][2 * n - 1]);
  if (e != cudaSuccess) return -fail(MOE_CUDA_ERROR, "event sync: %s", cudaGetErrorString(e));
  for (int i = 0; i < n && i < cap; ++i) {
    float t = 0.0f;
    e = cudaEventElapsedTime(&t, p->ev[set][2 * i], p->ev[set][2 * i + 1]);
    if (e != cudaSuccess) return -fail(MOE_CUDA_ERROR, "event time: %s", cudaGetErrorString(e));
    ms[i] = t;
  }
  return n;
}

const char* moe_plan_kernel_name(moe_plan_t p, int i) {
  if (!p || i < 0 || i >= p->n_launch || i >= kMaxKernels) return nullptr;
  return p->names[i];
}

int moe_plan_last_launch_count(moe_plan_t p) { return p ? p->n_launch : 0; }

int64_t moe_plan_capacity_seats(moe_plan_t p, int64_t T) {
  if (!p || T < 0) return -fail(MOE_INVALID_ARG, "null plan or negative T");
  return capacity_seats(p, T);
}

}  // extern "C"

extern "C" {

int moe_forward_noalloc(moe_plan_t p, int64_t T, const moe_bf16_t* x, const moe_bf16_t* W_g,
                        const moe_bf16_t* W1, const moe_bf16_t* W3, const moe_bf16_t* W2,
                        const moe_bf16_t* W1s, const moe_bf16_t* W3s, const moe_bf16_t* W2s,
                        moe_bf16_t* out, void* stream) {
  if (!p) return fail(MOE_INVALID_ARG, "null plan");
  if (T < 0) return fail(MOE_INVALID_ARG, "T must be >= 0");
  const size_t need = make_layout(p, T).total;
  if (need > kNoAllocScratchBytes)
    return fail(MOE_WORKSPACE_TOO_SMALL,
                "T=%lld needs %zu bytes of scratch; the static scratch of moe_forward_noalloc "
                "holds %zu bytes (use moe_forward with a caller workspace)",
                (long long)T, need, kNoAllocScratchBytes);
  if (!p->noalloc_scratch)
    return fail(MOE_CUDA_ERROR, "the plan has no address for the static scratch");
  // Run the regular forward on the static scratch, with timing off so that no
  // events are created, then give the plan back its own workspace and the state
  // its getters report (routing, permutation, launch count and kernel names
  // keep describing the last moe_forward, whose routing is still in the
  // plan's workspace). The status word at the start of the scratch is not
  // cleared here: a bounded-wait timeout stays visible to moe_plan_device_status.
  // The router's ticket must start at zero; every call clears it, so that two
  // calls that overlapped (which race) cannot leave it disturbed for the next.
  if (T > 0) {
    const Layout Ln = make_layout(p, T);
    cudaError_t e = cudaMemsetAsync(static_cast<char*>(p->noalloc_scratch) + Ln.ticket, 0,
                                    sizeof(int), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(MOE_CUDA_ERROR, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  }
  char* saved_ws = p->ws;
  const size_t saved_bytes = p->ws_bytes;
  const bool saved_timing = p->timing;
  const int64_t saved_T = p->last_T;
  const int saved_launch = p->n_launch;
  char saved_names[kMaxKernels][48];
  memcpy(saved_names, p->names, sizeof(saved_names));
  p->ws = static_cast<char*>(p->noalloc_scratch);
  p->ws_bytes = kNoAllocScratchBytes;
  p->timing = false;
  const int rc = moe_forward(p, T, x, W_g, W1, W3, W2, W1s, W3s, W2s, out, stream);
  p->ws = saved_ws;
  p->ws_bytes = saved_bytes;
  p->timing = saved_timing;
  p->last_T = saved_T;
  p->n_launch = saved_launch;
  memcpy(p->names, saved_names, sizeof(saved_names));
  if (rc == MOE_OK && T > 0) p->noalloc_used = true;
  return rc;
}

void moe_plan_destroy(moe_plan_t p) {
  if (!p) return;
  if (p->events_made)
    for (int r = 0; r < kTimingRing; ++r)
      for (int i = 0; i < 2 * kMaxKernels; ++i) cudaEventDestroy(p->ev[r][i]);
  if (p->side) cudaStreamDestroy(p->side);
  if (p->fork) cudaEventDestroy(p->fork);
  if (p->join) cudaEventDestroy(p->join);
  delete p;
}

const char* moe_strerror(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_INVALID_CONFIG: return "invalid expert configuration";
    case MOE_INVALID_ARG: return "invalid argument";
    case MOE_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_CUDA_ERROR: return "CUDA error";
    case MOE_UNSUPPORTED: return "unsupported shape";
    case MOE_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case MOE_DEVICE_INCONSISTENT: return "a kernel found inconsistent routing state";
    default: return "unknown status";
  }
}

const char* moe_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
