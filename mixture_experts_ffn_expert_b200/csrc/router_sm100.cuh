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
//    scores of its slice of E = N_r/CS experts over the whole K range (one
//    TMEM accumulator of <= 256 columns), so no partial sums are exchanged;
//  * warp 0 loads A (x rows, one 128x64 box) and B (the slice's W_g rows, boxes
//    of up to 128 rows) per 64-wide K block through TMA (no multicast); warp 1
//    issues tcgen05.mma M=128, N=E;
//  * warps 4..7 read the accumulator, one thread per token (its TMEM lane): the
//    slice's softmax statistics (its largest gate score and the sum of
//    exp(score - largest)) and its top-k candidates (selection key, expert, gate
//    score), kept sorted in registers - all 128 tokens of the tile at once;
//  * after a cluster barrier, one warp per token of this CTA's 128/CS tokens
//    gathers the CS slices' candidates and statistics through distributed
//    shared memory and selects the top k among them with warp reductions
//    (largest key, then lowest index: ties to the lower expert index); the
//    softmax over all N_r experts follows from the statistics;
//  * a shared histogram per CTA; reading the cluster's histograms, each CTA
//    writes its experts' offsets inside the tile and the first CTA the tile's
//    totals, one column of the tile histogram.
#pragma once

#include "gemm_sm100.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtThreads = 512;   // 16 warps: 16 tokens merged at once per CTA
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

// Shared memory of the candidates: KMAX per token of the tile (top_k <= KMAX)
// as (key, expert, gate score), plus the token's (max, sum) statistics.
template <int KMAX>
__host__ __device__ constexpr size_t router_cand_bytes() {
  return size_t(kBM) * KMAX * 12 + size_t(kBM) * 8;
}

// Dynamic shared memory of a launch: ring, candidates, histogram, barriers.
template <int KMAX>
__host__ __device__ constexpr size_t router_smem_bytes(int ring_bytes, int n_routed) {
  return 1024 + size_t(ring_bytes) + router_cand_bytes<KMAX>() +
         size_t((n_routed + 3) / 4 * 4) * 4 + 256;
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

template <int KMAX>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWg, const RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // candidates of the 128 tokens of the tile from this CTA's slice, [token][slot]
  uint32_t* c_key = reinterpret_cast<uint32_t*>(ring + P.ring_bytes);
  int* c_idx = reinterpret_cast<int*>(c_key + kBM * KMAX);
  float* c_val = reinterpret_cast<float*>(c_idx + kBM * KMAX);
  float* c_max = c_val + kBM * KMAX;               // [token] largest gate score of the slice
  float* c_sum = c_max + kBM;                      // [token] sum of exp(score - largest)
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
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ slice statistics
    // one thread per token of the tile (its TMEM lane): the slice's largest
    // gate score, the sum of exp(score - largest), and its top-k candidates
    bool ok = mbar_wait(smem_u32(tfull_bar), 0, s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) raise_timeout(s_abort, P.status);
    tc_fence_after_sync();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool have = nkb > 0 && *s_abort == 0;    // uniform over the CTA
    uint32_t ck[KMAX];
    int ci[KMAX];
    float cv[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ck[j] = 0u;
      ci[j] = 0x7fffffff;
      cv[j] = 0.0f;
    }
    uint32_t kth = 0u;   // key of the current k-th candidate (0 while fewer than k)
    float lmax = -INFINITY;
    // pass 1: the largest gate score
    for (int c = 0; have && c < P.ncols; c += 32) {
      uint32_t a[32];
      tmem_ld_32cols(taddr + c, a);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c + i < n_valid) {
          const float raw = __uint_as_float(a[i]);
          const float g = (P.bias && !P.bias_select_only) ? raw + __ldg(P.bias + e0 + c + i) : raw;
          lmax = fmaxf(lmax, g);
        }
    }
    // pass 2: the sum of exponentials and the candidates, in ascending expert
    // order (a later expert displaces a candidate only with a larger key, so
    // equal keys keep the lower expert first)
    float lsum = 0.0f;
    for (int c = 0; have && c < P.ncols; c += 32) {
      uint32_t a[32];
      tmem_ld_32cols(taddr + c, a);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (c + i >= n_valid) continue;
        const int e = e0 + c + i;
        const float raw = __uint_as_float(a[i]);
        const float key = P.bias ? raw + __ldg(P.bias + e) : raw;
        const float g = P.bias_select_only ? raw : key;
        lsum += expf(g - lmax);
        const uint32_t ok_ = order_key(key);
        if (ok_ > kth) {
          int pos = k - 1;
#pragma unroll
          for (int j = KMAX - 1; j >= 1; --j)
            if (j <= k - 1 && ok_ > ck[j - 1]) {
              ck[j] = ck[j - 1];
              ci[j] = ci[j - 1];
              cv[j] = cv[j - 1];
              pos = j - 1;
            }
#pragma unroll
          for (int j = 0; j < KMAX; ++j) {
            if (j == pos) {
              ck[j] = ok_;
              ci[j] = e;
              cv[j] = g;
            }
            if (j == k - 1) kth = ck[j];
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
        c_key[row * KMAX + j] = ck[j];
        c_idx[row * KMAX + j] = ci[j];
        c_val[row * KMAX + j] = cv[j];
      }
    c_max[row] = lmax;
    c_sum[row] = lsum;
  }

  // ---------------------------------------------------------------- merge
  // every CTA's candidates are written; one warp per token of this CTA gathers
  // the CS slices' candidates (k each, sorted) and statistics
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const int own = P.own_rows;
  const int tok0 = row0 + static_cast<int>(rank) * own;
  const int ntok = min(own, P.T - tok0);
  const int n_cand = P.cs * k;                     // <= 8 * 16 = 128: <= 4 per lane
  for (int tl = warp; tl < ntok; tl += kRtThreads / 32) {
    const int row = static_cast<int>(rank) * own + tl;   // row of the tile
    // slice statistics: M = the largest gate score, S = the sum over all
    // experts of exp(score - M), from each slice's (max, sum)
    float sm = -INFINITY, ss = 0.0f;
    if (lane < P.cs) {
      sm = __uint_as_float(ld_cluster_u32(
          mapa_shared(smem_u32(c_max + row), static_cast<uint32_t>(lane))));
      ss = __uint_as_float(ld_cluster_u32(
          mapa_shared(smem_u32(c_sum + row), static_cast<uint32_t>(lane))));
    }
    float M = sm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float S = lane < P.cs ? ss * expf(sm - M) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    // candidates: lane holds entries lane + 32*i of the (slice, slot) list
    uint32_t okey[4];
    int oidx[4];
    float oval[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      okey[i] = 0u;
      oidx[i] = 0x7fffffff;
      oval[i] = 0.0f;
      if (c < n_cand) {
        const int src = c / k, slot = c - src * k;
        const uint32_t off = static_cast<uint32_t>((row * KMAX + slot) * 4);
        okey[i] = ld_cluster_u32(mapa_shared(smem_u32(c_key) + off, static_cast<uint32_t>(src)));
        oidx[i] = static_cast<int>(
            ld_cluster_u32(mapa_shared(smem_u32(c_idx) + off, static_cast<uint32_t>(src))));
        oval[i] = __uint_as_float(
            ld_cluster_u32(mapa_shared(smem_u32(c_val) + off, static_cast<uint32_t>(src))));
      }
    }
    // k rounds of warp reductions: the largest key, then the lowest expert
    // index holding it; each lane keeps its best untaken candidate
    uint32_t taken = 0, lk = 0u;
    int li = 0x7fffffff;
    float lv = 0.0f;
    auto rescan = [&]() {
      lk = 0u;
      li = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (!((taken >> i) & 1u) && (okey[i] > lk || (okey[i] == lk && oidx[i] < li))) {
          lk = okey[i];
          li = oidx[i];
          lv = oval[i];
        }
    };
    rescan();
    float my_gw = 0.0f;
    int my_e = -1;
    for (int j = 0; j < k; ++j) {
      const uint32_t gmax = __reduce_max_sync(0xffffffffu, lk);
      const int be = static_cast<int>(
          __reduce_min_sync(0xffffffffu, static_cast<unsigned>(lk == gmax ? li : 0x7fffffff)));
      // the one lane holding the winner takes it and rescans
      const unsigned holder = __ballot_sync(0xffffffffu, lk == gmax && li == be);
      const int hl = __ffs(holder) - 1;
      const float gw = __shfl_sync(0xffffffffu, lv, hl);
      if (lane == j) { my_gw = gw; my_e = be; }
      if (lane == hl) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (oidx[i] == be && !((taken >> i) & 1u)) taken |= 1u << i;
        rescan();
      }
    }
    const float my_p = lane < k ? expf(my_gw - M) / S : 0.0f;
    float sel_sum = my_p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sel_sum += __shfl_xor_sync(0xffffffffu, sel_sum, o);
    if (lane < k) {
      const long long o = static_cast<long long>(tok0 + tl) * k + lane;
      P.idx[o] = my_e;
      P.gate[o] = P.renorm ? my_p / sel_sum : my_p;
      atomicAdd(&s_hist[my_e], 1);
    }
  }

  // histograms: from the cluster's per-CTA counts, every CTA writes each
  // expert's pairs in lower-ranked CTAs of the tile (its offset inside the
  // tile) and the first CTA the tile's totals
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
      for (int e = threadIdx.x; e < P.n_routed; e += kRtThreads) {
        int* rowp = P.tile_counts + static_cast<long long>(e) * P.n_chunks;
        // all of the expert's tile counts are loaded before the first store
        // (at most 64 tiles when the scan is folded)
        int v[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] = c < P.n_chunks ? __ldcg(rowp + c) : 0;
        int run = 0;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < P.n_chunks) {
            rowp[c] = run;
            run += v[c];
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
