// router_sm100.cuh - the fused router: for a tile of 128 tokens, the router
// scores s = x W_g^T on the 5th-generation tensor core, the softmax over the N_r
// experts, the top-k with ties to the lower expert index, the gates and the
// expert histogram, in one launch ("What is an "expert," really?", glossary:
// router / gate, top-k, softmax; panel 2: a linear scorer, softmax blend
// weights, keep the top k). With few tiles the last cluster of the grid also
// turns the histogram into per-tile bases and expert totals, so the
// permutation kernel can follow directly.
//
// Design (sm_100a, N_r <= 512, top_k <= 32):
//  * a cluster of CS CTAs (CS <= 8) owns one 128-token tile; CTA r computes the
//    scores of its slice of E = N_r/CS <= 64 experts over the whole K range
//    (one TMEM accumulator), so no partial sums are exchanged;
//  * warps 0 and 2 load A (x rows, one 128x64 box) and B (the slice's W_g rows)
//    per 64-wide K block through TMA (no multicast), on alternate stages of
//    the ring, so that their issue costs overlap; warp 1 issues tcgen05.mma
//    M=128, N=E;
//  * warps 0..15 copy the accumulator to shared memory; after a cluster
//    barrier every CTA routes its own 128/CS tokens of the tile: one warp per
//    token gathers the token's N_r scores from the CS slices through
//    distributed shared memory and runs the same selection as the two-kernel
//    router (route_token: softmax statistics, k rounds of warp reductions,
//    gates), so each token is selected once, by one warp;
//  * a shared histogram per CTA; reading the cluster's histograms, each CTA
//    writes its experts' offsets inside the tile and the first CTA the tile's
//    totals, one column of the tile histogram;
//  * every loop over tokens, columns or experts stays rolled: a CTA runs the
//    code about once, so its length (instruction fetch) would otherwise set
//    the time.
#pragma once

#include "gemm_sm100.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtThreads = 512;       // 16 warps
constexpr int kRtMaxCluster = 8;
constexpr int kRtMaxStages = 8;
constexpr int kRtMaxExperts = 512;
constexpr int kRtMaxTopK = 32;        // one selected expert per lane
constexpr int kRtMaxSliceCols = 64;   // accumulator columns of one slice

struct RouterParams {
  int T, d, n_routed, top_k, renorm, bias_select_only;
  const float* bias;     // device (N_r) or null
  int cs;                // CTAs per cluster = expert slices of one token tile
  int e_per;             // experts per slice (multiple of 16, <= 64): MMA N
  int ncols;             // accumulator columns read (e_per rounded up to 32)
  int num_kb;            // 64-wide K blocks of d
  int own_rows;          // tokens each CTA routes (128 / cs)
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

// Scratch laid over the ring once the scores are complete: the slice's scores
// [token][ncols + 1] in fp32 (odd row stride: a warp's 32 rows hit 32 banks).
__host__ __device__ constexpr size_t router_scratch_bytes() {
  return size_t(kBM) * (kRtMaxSliceCols + 1) * 4;
}

// Dynamic shared memory of a launch: ring, histogram, barriers.
__host__ __device__ constexpr size_t router_smem_bytes(int ring_bytes, int n_routed) {
  return 1024 + size_t(ring_bytes) + size_t((n_routed + 3) / 4 * 4) * 4 + 256;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// NPL: router scores each lane holds in the selection (N_r <= 32 * NPL).
template <int NPL>
__global__ void __launch_bounds__(kRtThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWg, const RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  int* s_hist = reinterpret_cast<int*>(ring + P.ring_bytes);
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

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ TMA producers
    // both walk the k-blocks; producer pid fills those with it % 2 == pid, i.e.
    // alternate stages of the ring, so that their issue costs overlap
    const int pid = warp == 0 ? 0 : 1;
    uint32_t issued_mask = 0, issued_par = 0;
    bool ok = true;
    for (int it = pid; it < nkb; it += 2) {
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
  // warps w, w+4, w+8, w+12 share TMEM lanes 32*(w%4).. (the tokens of that
  // quarter of the tile); each copies a quarter of the slice's columns into
  // the score rows [token][ncols + 1] laid over the ring (every MMA has
  // completed, so every stage has been read)
  float* s_score = reinterpret_cast<float*>(ring);
  const int lds = P.ncols + 1;
  {
    bool ok = mbar_wait(smem_u32(tfull_bar), 0, s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) raise_timeout(s_abort, P.status);
    tc_fence_after_sync();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int cpp = P.ncols / 4;                  // a multiple of 8
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    if (nkb > 0 && ok) {
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

  // ---------------------------------------------------------------- selection
  // after the cluster barrier every slice's scores are in its CTA's shared
  // memory; one warp per token of this CTA's 128/CS tokens gathers the
  // token's N_r scores (lane l: experts l + 32 i, read from the slice that
  // holds them) and selects its experts exactly as the two-kernel router does
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  tc_fence_after_sync();
  {
    const int own = P.own_rows;
    const int tok0 = row0 + static_cast<int>(rank) * own;
    const int ntok = max(0, min(own, P.T - tok0));
    // where lane l's experts live: the holding slice's score of token row 0
    uint32_t src[NPL];
    const uint32_t sbase = smem_u32(s_score);
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      const int sl = e < P.n_routed ? e / P.e_per : 0;
      const int c = e < P.n_routed ? e - sl * P.e_per : 0;
      src[i] = mapa_shared(sbase + static_cast<uint32_t>(c * 4), static_cast<uint32_t>(sl));
    }
#pragma unroll 1
    for (int tl = warp; tl < ntok; tl += kRtThreads / 32) {
      const uint32_t roff = static_cast<uint32_t>((static_cast<int>(rank) * own + tl) * lds * 4);
      float v[NPL];
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        v[i] = lane + 32 * i < P.n_routed ? __uint_as_float(ld_cluster_u32(src[i] + roff)) : 0.0f;
      int my_e;
      float my_g;
      route_token<NPL>(v, P.bias, P.n_routed, k, P.renorm, P.bias_select_only, lane, my_e, my_g);
      if (lane < k) {
        const long long o = static_cast<long long>(tok0 + tl) * k + lane;
        P.idx[o] = my_e;
        P.gate[o] = my_g;
        if (static_cast<unsigned>(my_e) < static_cast<unsigned>(P.n_routed))
          atomicAdd(&s_hist[my_e], 1);
      }
    }
  }

  // histograms: from the cluster's per-CTA counts, every CTA writes each
  // expert's pairs in lower-ranked CTAs of the tile (its offset inside the
  // tile) and the first CTA the tile's totals; the barrier also ends every
  // read of another CTA's scores
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
    // counts (in place) and the expert totals; then the ticket is reset for the
    // next forward (every cluster took exactly one)
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
