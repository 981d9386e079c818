// router_sm100.cuh - the fused router: for a tile of 128 tokens, the router
// scores s = x W_g^T on the 5th-generation tensor core, the softmax over the N_r
// experts, the warp-shuffle top-k with ties to the lower expert index, the gates
// and the per-chunk expert histogram, in one launch ("What is an "expert,"
// really?", glossary: router / gate, top-k, softmax; panel 2: a linear scorer,
// softmax blend weights, keep the top k). With few chunks the last CTA of the
// grid also turns the histogram into per-chunk bases and expert totals, so the
// permutation kernel can follow directly.
//
// Design (sm_100a, N_r <= 512):
//  * a cluster of CS CTAs (CS <= 8) owns one 128-token tile; CTA r of the
//    cluster reduces over its own K range (split-K) for ALL experts, so each
//    CTA streams 1/CS of the token rows and of W_g through TMA (no multicast);
//  * warp 0 loads A (x rows, one 128x64 box) and B (W_g rows, boxes of up to
//    128 rows) per 64-wide K block; warp 1 issues tcgen05.mma M=128 into one
//    or two TMEM accumulators of <= 256 columns;
//  * the partial scores are reduced across the cluster through distributed
//    shared memory: each CTA copies its accumulator (warps 4..7, one TMEM lane
//    quarter each) into its own shared memory, and after a cluster barrier the
//    CTA that routes tokens m .. m + 128/CS - 1 reads those rows from every CTA
//    of the cluster (coalesced 16-byte loads) and adds the CS partials in rank
//    order (deterministic), up to 256 experts per round;
//  * every warp then routes tokens of its CTA with route_token (one warp per
//    token, N_r/32 scores per lane), writes idx and gates, and counts experts in
//    a shared histogram; reading the cluster's histograms, each CTA writes its
//    experts' offsets within the tile (the pairs of lower-ranked CTAs) and the
//    first CTA the tile's totals, one column of the tile histogram.
#pragma once

#include "gemm_sm100.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtThreads = 256;
constexpr int kRtMaxCluster = 8;
constexpr int kRtMaxStages = 8;
constexpr int kRtMaxExperts = 512;

struct RouterParams {
  int T, d, n_routed, top_k, renorm, bias_select_only;
  const float* bias;     // device (N_r) or null
  int cs;                // CTAs per cluster = K splits of one token tile
  int kb_per;            // 64-wide K blocks per CTA
  int num_kb;            // K blocks of d
  int own_rows;          // tokens each CTA routes (128 / cs)
  int n_chunks;          // ceil(T / 128): columns of tile_counts
  int n_acc;             // accumulators (1, or 2 when N_r > 256)
  int mma_n0, mma_n1;    // MMA N of each accumulator (multiples of 16)
  int ncols0, ncols1;    // exchanged columns of each accumulator (multiples of 32)
  int box_rows;          // rows of one W_g TMA box
  int nbox0, nbox1;      // W_g boxes per accumulator per stage
  int stages;
  int stage_bytes;       // A box + B boxes of one stage
  int b_acc1_off;        // offset of accumulator 1's B rows inside a stage
  int ring_bytes;        // the stage ring, reused as the exchange buffer
  int lds;               // row stride (floats) of the CTA's score buffer
  int tmem_cols;
  int fold_scan;         // 1: the grid's last cluster scans the chunk histogram
  int* idx;              // (T, top_k)
  float* gate;           // (T, top_k)
  int* tile_counts;      // [N_r][n_chunks] pairs per expert and tile (scanned in place)
  int* sub_base;         // [N_r][n_chunks * cs] an expert's pairs in the tile before each CTA's tokens
  int* counts;           // (N_r), written when fold_scan
  int* ticket;           // zero between forwards
  int* status;           // device status word
};

// Dynamic shared memory of a launch: ring, scores, histogram, barriers.
__host__ __device__ constexpr size_t router_smem_bytes(int ring_bytes, int own_rows, int lds,
                                                       int n_routed) {
  return 1024 + size_t(ring_bytes) + size_t(own_rows) * lds * 4 +
         size_t((n_routed + 3) / 4 * 4) * 4 + 256;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

template <int NPL>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWg, const RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* s_scores = reinterpret_cast<float*>(ring + P.ring_bytes);
  int* s_hist = reinterpret_cast<int*>(s_scores + size_t(P.own_rows) * P.lds);
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
  const int kb0 = static_cast<int>(rank) * P.kb_per;
  const int kb1 = min(P.num_kb, kb0 + P.kb_per);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;

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
        const int k0 = (kb0 + it) * kBK;
        mbar_arrive_expect_tx(fb, P.stage_bytes);
        tma_load_2d(a_dst, &tmX, fb, k0, row0);
        for (int j = 0; j < P.nbox0; ++j)
          tma_load_2d(a_dst + kATileBytes + j * box_bytes, &tmWg, fb, k0, j * P.box_rows);
        for (int j = 0; j < P.nbox1; ++j)
          tma_load_2d(a_dst + P.b_acc1_off + j * box_bytes, &tmWg, fb, k0, 256 + j * P.box_rows);
      }
      __syncwarp();
      issued_mask |= 1u << s;
      issued_par = (issued_par & ~(1u << s)) | (ph << s);
    }
    if (!ok && lane == 0) {
      // give the copies already issued a bounded chance to land before the
      // ring is reused or the CTA exits
      for (int i = 0; i < P.stages; ++i)
        if (issued_mask & (1u << i)) {
          int never = 0;
          mbar_wait(smem_u32(&full_bar[i]), (issued_par >> i) & 1u, &never);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc0 = idesc_bf16_f32(kBM, P.mma_n0);
    const uint32_t idesc1 = idesc_bf16_f32(kBM, P.n_acc > 1 ? P.mma_n1 : 16);
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
        const uint32_t b0 = a_base + kATileBytes;
        const uint32_t b1 = a_base + P.b_acc1_off;
#pragma unroll
        for (int k = 0; k < kBK / kUK; ++k)
          umma_bf16(tmem_base, sdesc_kmajor_sw128(a_base + k * kUK * 2),
                    sdesc_kmajor_sw128(b0 + k * kUK * 2), idesc0, (it > 0 || k > 0) ? 1u : 0u);
        if (P.n_acc > 1) {
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            umma_bf16(tmem_base + 256, sdesc_kmajor_sw128(a_base + k * kUK * 2),
                      sdesc_kmajor_sw128(b1 + k * kUK * 2), idesc1,
                      (it > 0 || k > 0) ? 1u : 0u);
        }
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
        umma_commit(smem_u32(tfull_bar));        // accumulators complete
      } else {
        mbar_arrive(smem_u32(tfull_bar));        // no K blocks: nothing to wait for
      }
    }
    __syncwarp();
  }
  if (warp >= 4) {
    bool ok = mbar_wait(smem_u32(tfull_bar), 0, s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) raise_timeout(s_abort, P.status);
    tc_fence_after_sync();
  }

  // ---------------------------------------------------------------- reduce
  // Round a exchanges accumulator a (experts 256a .. 256a + ncols - 1). Each
  // CTA first copies its 128 partial rows into its own exchange buffer (the
  // stage ring, free once every MMA of this CTA has completed: the first barrier
  // of round 0 follows the TMEM readers' wait; in round 1 it follows every
  // CTA's reads of round 0), then every CTA reads its own tokens' rows from all
  // CS buffers of the cluster and adds them in rank order.
  const int own = P.own_rows;
  for (int a = 0; a < P.n_acc; ++a) {
    const int ncols = a ? P.ncols1 : P.ncols0;
    const int xld = ncols + 4;      // row stride: 4 banks apart, conflict-free v4 stores
    tc_fence_before_sync();
    cluster_sync();
    tc_fence_after_sync();
    if (warp >= 4) {
      const int q = warp & 3;
      const int row = q * 32 + lane;                 // token row of the tile = TMEM lane
      float* dst = reinterpret_cast<float*>(ring) + row * xld;
      const bool have = nkb > 0 && *s_abort == 0;    // uniform over the CTA
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(a * 256);
      for (int c = 0; c < ncols; c += 32) {
        uint32_t v[32];
        if (have) {
          tmem_ld_32cols(taddr + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(dst + c + 4 * i) =
              make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
    cluster_sync();
    // this CTA's tokens: the same rows of every CTA's buffer, added in rank order
    const uint32_t xbase = smem_u32(ring);
    const int n4 = ncols / 4;
    for (int i = threadIdx.x; i < own * n4; i += kRtThreads) {
      const int r = i / n4;
      const int c = (i - r * n4) * 4;
      const uint32_t off =
          static_cast<uint32_t>(((static_cast<int>(rank) * own + r) * xld + c) * 4);
      float4 part[kRtMaxCluster];
#pragma unroll
      for (int s = 0; s < kRtMaxCluster; ++s)
        if (s < P.cs) part[s] = ld_cluster_f4(mapa_shared(xbase + off, static_cast<uint32_t>(s)));
      float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int s = 0; s < kRtMaxCluster; ++s)
        if (s < P.cs) {
          sum.x += part[s].x;
          sum.y += part[s].y;
          sum.z += part[s].z;
          sum.w += part[s].w;
        }
      *reinterpret_cast<float4*>(s_scores + r * P.lds + a * 256 + c) = sum;
    }
  }
  // every CTA has read the cluster's buffers: the ring may be reused, and no
  // CTA leaves while another can still read its shared memory
  cluster_sync();

  // ---------------------------------------------------------------- route
  const int tok0 = row0 + static_cast<int>(rank) * own;
  const int ntok = min(own, P.T - tok0);
  for (int tl = warp; tl < ntok; tl += kRtThreads / 32) {
    float v[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < P.n_routed ? s_scores[tl * P.lds + e] : 0.0f;
    }
    int my_e;
    float my_g;
    route_token<NPL>(v, P.bias, P.n_routed, P.top_k, P.renorm, P.bias_select_only, lane, my_e,
                     my_g);
    if (lane < P.top_k) {
      const long long o = static_cast<long long>(tok0 + tl) * P.top_k + lane;
      P.idx[o] = my_e;
      P.gate[o] = my_g;
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
                          : ld_cluster_s32(mapa_shared(hbase + static_cast<uint32_t>(e * 4),
                                                       static_cast<uint32_t>(s2)));
        pre += s2 < static_cast<int>(rank) ? h : 0;
        tot += h;
      }
      P.sub_base[static_cast<long long>(e) * n_sub + blockIdx.x] = pre;
      if (rank == 0) P.tile_counts[static_cast<long long>(e) * P.n_chunks + tile] = tot;
    }
  }
  // no CTA leaves while another can still read its histogram
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
        int* row = P.tile_counts + static_cast<long long>(e) * P.n_chunks;
        int run = 0;
        for (int c0 = 0; c0 < P.n_chunks; c0 += 8) {
          int v[8];
#pragma unroll
          for (int b = 0; b < 8; ++b) v[b] = c0 + b < P.n_chunks ? __ldcg(row + c0 + b) : 0;
#pragma unroll
          for (int b = 0; b < 8; ++b)
            if (c0 + b < P.n_chunks) {
              row[c0 + b] = run;
              run += v[b];
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
