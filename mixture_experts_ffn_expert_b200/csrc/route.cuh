// route.cuh - routing and combine kernels of the MoE layer (CUDA cores,
// HBM/latency-bound work around the tensor-core GEMMs).
//
//  route_topk     sums the router-score partials of a split-K GEMM, adds the
//                 logit bias, softmax over the N_r scores of a token, top-k
//                 with ties to the lower expert index, raw or renormalised gates
//                 ("What is an "expert," really?", glossary: router / gate,
//                 top-k, softmax; panel 2), and a per-chunk expert histogram.
//  route_scan     one warp per expert: exclusive prefix over chunks of that
//                 expert's counts, and the expert's total.
//  route_scatter  every block derives the expert offsets (exclusive scan of the
//                 totals) itself; block 0 also publishes offsets and the prefix
//                 of 128-row m-tiles the grouped GEMM scheduler walks. Then the
//                 stable (token, slot) order inside each expert group, the
//                 permutation, and 16-byte-vector copies of each token row to
//                 its k grouped rows.
//  combine        out[t] = shared[t] + sum_j g[t,j] * Y[inv_pos[t,j]] in fp32,
//                 one bf16 rounding ("Shared Expert (DeepSeek-V3)", eq. (12)
//                 without the residual; shared term coefficient 1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include "ptx_sm100.cuh"

namespace moe {

constexpr int kRouteThreads = 256;             // 8 warps
constexpr int kMaxTopK = 32;
constexpr int kMaxRouted = 1024;

// One token's routing, computed by one warp from its N_r router scores (lane
// i holds the scores of experts lane + 32*j in v[j], the bias not yet added):
// softmax over all N_r experts, the top_k experts by the biased score with
// ties to the lower index, and the gates (raw probabilities, or renormalised
// over the selected set). Lane j < top_k receives the j-th selected expert in
// `my_e` and its gate in `my_g`.
template <int NPL>
__device__ __forceinline__ void route_token(float (&v)[NPL], const float* __restrict__ bias,
                                            int n_routed, int top_k, int renorm,
                                            int bias_select_only, int lane, int& my_e,
                                            float& my_g) {
  // The biased scores rank the experts; the gates are the softmax of the
  // biased scores (logit bias) or of the unbiased ones (selection-only bias).
  float m = -INFINITY;
  float key[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    const float b = (bias && e < n_routed) ? bias[e] : 0.0f;
    key[i] = e < n_routed ? v[i] + b : -INFINITY;
    v[i] = e < n_routed ? (bias_select_only ? v[i] : key[i]) : -INFINITY;
    m = fmaxf(m, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.0f;
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (lane + 32 * i < n_routed) sum += expf(v[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);

  // Selection keys: a NaN score (from NaN or infinite inputs) ranks as -inf,
  // so the order stays total and every lane agrees on each winner. Each key is
  // mapped to an unsigned integer with the same order (-0 and +0 equal); an
  // empty lane's 0 is below every real key (-inf maps to 0x007fffff).
  uint32_t okey[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    float kv = key[i] == key[i] ? key[i] : -INFINITY;
    kv = kv == 0.0f ? 0.0f : kv;
    const uint32_t b = __float_as_uint(kv);
    okey[i] = lane + 32 * i < n_routed ? ((b & 0x80000000u) ? ~b : (b | 0x80000000u)) : 0u;
  }
  // Each lane keeps its best untaken expert (largest key, lowest index among
  // equal keys) with its gate score. A round of the selection is two warp
  // reductions (redux.sync): the largest key, then the lowest expert index
  // holding it - ties go to the lower index; only the winning lane rescans.
  uint32_t taken = 0;
  uint32_t lk = 0u;
  int li = 0x7fffffff;
  float lv = 0.0f;
  auto rescan = [&]() {
    lk = 0u;
    li = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (!((taken >> i) & 1u) && okey[i] > lk) {   // ascending i: '>' keeps the lower index
        lk = okey[i];
        li = lane + 32 * i;
        lv = v[i];
      }
  };
  rescan();
  float my_gw = 0.0f;
  my_e = -1;
  for (int j = 0; j < top_k; ++j) {
    const uint32_t gmax = __reduce_max_sync(0xffffffffu, lk);
    const int be = static_cast<int>(
        __reduce_min_sync(0xffffffffu, static_cast<unsigned>(lk == gmax ? li : 0x7fffffff)));
    const float gw = __shfl_sync(0xffffffffu, lv, be & 31);   // the winner's gate score
    if (lane == j) { my_gw = gw; my_e = be; }
    if ((be & 31) == lane) {
      taken |= 1u << (be >> 5);
      rescan();
    }
  }
  // lane j < top_k: the probability of the j-th selected expert; the sum over
  // the selected ones for the renormalisation
  const float my_p = lane < top_k ? expf(my_gw - m) / sum : 0.0f;
  float sel_sum = my_p;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sel_sum += __shfl_xor_sync(0xffffffffu, sel_sum, o);
  my_g = renorm ? my_p / sel_sum : my_p;
}

// One warp per token; block = one chunk of `tpc` consecutive tokens.
// NPL = router scores held per lane (N_r <= 32 * NPL). The scores arrive as
// `splits` (<= MAXS) fp32 partial sums (split-K of the router GEMM),
// `split_stride` elements apart, and are added in split order; all partial
// loads of a lane are issued before the first add.
//
// The kernel starts early (programmatic dependent launch) while the router
// GEMM still runs, and each warp first runs its token body once on no data -
// score loads and stores switched off - before the dependency wait: the
// instructions (several KB, run once per warp) and the bias are then cached
// when the scores arrive. After an L2 flush, or another layer's weight stream,
// fetching them cold took longer than the selection itself (512-expert decode
// step: the kernel ended 4.6 us earlier with the warm-up). Both passes run the
// same code (the pass loop is not unrolled).
template <int NPL, int MAXS>
__global__ void __launch_bounds__(kRouteThreads)
    route_topk_kernel(const float* __restrict__ scores, int lds, int splits,
                      long long split_stride, const float* __restrict__ bias, int T,
                      int n_routed, int top_k, int renorm, int bias_select_only, int tpc,
                      int n_chunks,
                      int* __restrict__ idx, float* __restrict__ gate,
                      int* __restrict__ chunk_counts) {
  extern __shared__ int s_hist[];               // [n_routed]
  pdl_launch_dependents();
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x) s_hist[e] = 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int t_begin = chunk * tpc;
  const int t_end = min(T, t_begin + tpc);
  int warm = 0;                                 // the dry pass's (unused) selection
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const bool dry = pass == 0;
    if (!dry) {
      pdl_wait();                               // scores come from the router GEMM
      __syncthreads();
    }
    const int t_stop = dry ? min(t_end, t_begin + warp + 1) : t_end;   // dry: one token
    for (int t = t_begin + warp; t < t_stop; t += kRouteThreads / 32) {
      const float* row = scores + static_cast<long long>(t) * lds;
      float part[MAXS][NPL];
#pragma unroll
      for (int sp = 0; sp < MAXS; ++sp)
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int e = lane + 32 * i;
          part[sp][i] = (!dry && sp < splits && e < n_routed) ? row[sp * split_stride + e] : 0.0f;
        }
      float v[NPL];
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        float a = part[0][i];
#pragma unroll
        for (int sp = 1; sp < MAXS; ++sp) a += part[sp][i];
        v[i] = a;
      }
      int my_e;
      float my_g;
      route_token<NPL>(v, bias, n_routed, top_k, renorm, bias_select_only, lane, my_e, my_g);
      if (dry) {
        warm += my_e;
        continue;
      }
      if (lane < top_k) {
        const long long o = static_cast<long long>(t) * top_k + lane;
        idx[o] = my_e;
        gate[o] = my_g;
        atomicAdd(&s_hist[my_e], 1);
      }
    }
  }
  if (warm == INT_MIN) atomicAdd(&s_hist[0], 0);   // keeps the dry pass (never true; adds 0)
  __syncthreads();
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x)
    chunk_counts[static_cast<long long>(e) * n_chunks + chunk] = s_hist[e];
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// One warp scans one expert's row of chunk_counts [N_r][n_chunks]: the row
// becomes, in place, the exclusive prefix over chunks; returns the expert's
// total to every lane. The warp's loads for up to 32*kScanPrefetch chunks are
// issued before any scan. kL2 reads through L2 only (rows another block of the
// same grid wrote, made visible by a fence).
constexpr int kScanPrefetch = 16;

template <bool kL2>
__device__ __forceinline__ int scan_expert_chunks(int* row, int n_chunks, int lane) {
  int running = 0;
  for (int c0 = 0; c0 < n_chunks; c0 += 32 * kScanPrefetch) {
    int v[kScanPrefetch];
#pragma unroll
    for (int b = 0; b < kScanPrefetch; ++b) {
      const int c = c0 + b * 32 + lane;
      v[b] = c < n_chunks ? (kL2 ? __ldcg(row + c) : row[c]) : 0;
    }
    const int nb = min(kScanPrefetch, (n_chunks - c0 + 31) / 32);   // warp-uniform
#pragma unroll
    for (int b = 0; b < kScanPrefetch; ++b) {
      if (b >= nb) break;
      const int c = c0 + b * 32 + lane;
      const int incl = warp_inclusive_scan(v[b], lane);
      if (c < n_chunks) row[c] = running + incl - v[b];
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  return running;
}

// One warp per expert (8 experts per block): exclusive prefix over chunks of
// each expert's counts, in place, and the expert's total.
__global__ void __launch_bounds__(kRouteThreads)
    route_scan_kernel(int* __restrict__ chunk_counts, int n_chunks, int n_routed,
                      int* __restrict__ counts) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (kRouteThreads / 32) + (threadIdx.x >> 5);
  if (e >= n_routed) return;
  const int total =
      scan_expert_chunks<false>(chunk_counts + static_cast<long long>(e) * n_chunks, n_chunks, lane);
  if (lane == 0) counts[e] = total;
}

// Exclusive scan of n (<= kMaxRouted) ints in shared memory by a 256-thread
// block, in place; returns the total to every thread. `tmp` holds 8 ints.
__device__ __forceinline__ int block_exclusive_scan(int* s, int n, int* tmp) {
  constexpr int kPer = kMaxRouted / kRouteThreads;   // 4 consecutive items per thread
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int base = threadIdx.x * kPer;
  int loc[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    loc[i] = base + i < n ? s[base + i] : 0;
    sum += loc[i];
  }
  const int incl = warp_inclusive_scan(sum, lane);
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kRouteThreads / 32; ++w) {
    const int t = tmp[w];
    if (w < warp) wbase += t;
    total += t;
  }
  int run = wbase + incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (base + i < n) s[base + i] = run;
    run += loc[i];
  }
  __syncthreads();
  return total;
}

// Sum of one int per thread over a 256-thread block; every thread gets it.
// `tmp` holds 8 ints; the block must be converged.
__device__ __forceinline__ int block_sum(int v, int* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  int total = 0;
#pragma unroll
  for (int w = 0; w < kRouteThreads / 32; ++w) total += tmp[w];
  __syncthreads();
  return total;
}

// Block = one chunk. The chunk's expert ids and their bases inside each
// expert's group are staged in shared memory by all threads; warp 0 then ranks the (token, slot)
// entries in order with match-any, so rows inside an expert group follow
// ascending (t, j); every warp then copies token rows (d_vec 16-byte vectors
// each) to their k rows, four vectors in flight per lane. With a seat limit
// (capacity; INT_MAX when unlimited) an expert keeps its first `capacity` pairs
// in that order ("What is an expert, really?" glossary, capacity factor / token
// dropping): offsets and m-tiles count kept rows, a dropped pair gets inv_pos
// -1 and no row. Grid (n_chunks, column slices): every block ranks its chunk;
// the blocks of slice 0 write the permutation, block (0, 0) the offsets.
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kRouteThreads)
    route_scatter_kernel(const int* __restrict__ idx, const int* __restrict__ chunk_base,
                         int n_base, const int* __restrict__ sub_base, int subs_per_base,
                         int sub_tokens, const int* __restrict__ counts, int T, int top_k,
                         int n_routed, int tpc, int n_chunks, int tile_rows, int capacity,
                         const uint4* __restrict__ x,
                         int d_vec, uint4* __restrict__ xperm, int* __restrict__ perm_src,
                         int* __restrict__ inv_pos, int* __restrict__ offsets_out,
                         int* __restrict__ mtiles_out, int* __restrict__ mtiles2_out,
                         int* __restrict__ mtiles4_out, int* __restrict__ mt_hot_out,
                         int* __restrict__ mt_cold_out, int pass_mask,
                         int* __restrict__ status) {
  extern __shared__ int smem_i[];
  int* s_off = smem_i;                        // [kMaxRouted] expert offsets
  int* s_run = smem_i + kMaxRouted;           // [n_routed]
  int* s_e = s_run + n_routed;                // [tpc * top_k] expert of each entry
  int* s_pos = s_e + tpc * top_k;             // [tpc * top_k] chunk base, then row
  __shared__ int s_tmp[kRouteThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  const int chunk = blockIdx.x;
  const int t0 = chunk * tpc;
  const int ntok = max(0, min(tpc, T - t0));   // the last tile's chunks may hold no token
  const int n_ent = ntok * top_k;
  const long long ebase = static_cast<long long>(t0) * top_k;
  // The block's base inside each expert's group. The histogram it comes from
  // counts pairs per sub-chunk of sub_tokens tokens (a multiple of tpc):
  // chunk_base [N_r][n_base] holds the prefix at each group of subs_per_base
  // sub-chunks and, with two levels, sub_base [N_r][n_base * subs_per_base]
  // the pairs of the sub-chunks before it in its group; the pairs of the
  // sub-chunk's own tokens before this block are counted here.
  const int sub = t0 / sub_tokens;
  const int grp = sub / subs_per_base;
  const int pre_tokens = t0 - sub * sub_tokens;
  // (an expert index out of range - a router that gave up - gets a negative
  // place, so the entry is reported and dropped below)
  for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
    const int e = idx[ebase + i];
    const bool in_range = static_cast<unsigned>(e) < static_cast<unsigned>(n_routed);
    s_e[i] = in_range ? e : 0;
    int b = -(1 << 30);
    if (in_range) {
      b = chunk_base[static_cast<long long>(e) * n_base + grp];
      if (sub_base) b += sub_base[static_cast<long long>(e) * (n_base * subs_per_base) + sub];
    }
    s_pos[i] = b;
  }
  // an expert keeps at most `capacity` rows: its first pairs in (token, slot) order
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x) {
    s_off[e] = min(counts[e], capacity);
    s_run[e] = 0;
  }
  // consistency of the routing state: the expert totals must add up to the
  // T*top_k pairs and be non-negative. They always do unless the workspace was
  // overwritten during a forward; then every block of the grid sees the same
  // totals and the forward degrades to writing nothing out of range: no rows,
  // empty expert groups, every slot dropped, and the device status reports it.
  __syncthreads();
  const int pairs = T * top_k;
  int csum = 0, crange = 0;
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x) {
    const int c = counts[e];
    csum += c;
    crange |= c < 0 || c > pairs;
  }
  const int out_of_range = __syncthreads_or(crange);
  const bool bad = out_of_range || block_sum(csum, s_tmp) != pairs;
  if (bad)
    for (int e = threadIdx.x; e < n_routed; e += blockDim.x) s_off[e] = 0;
  __syncthreads();
  const int total = block_exclusive_scan(s_off, n_routed, s_tmp);
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    if (bad && threadIdx.x == 0) atomicExch(status, 7 /* MOE_DEVICE_INCONSISTENT */);
    // publish offsets and the m-tile prefix for the grouped GEMMs
    for (int e = threadIdx.x; e < n_routed; e += blockDim.x) offsets_out[e] = s_off[e];
    if (threadIdx.x == 0) offsets_out[n_routed] = total;
    // prefixes of m-tiles of tile_rows, 2*tile_rows (CTA-pair tiles) and
    // tile_rows/2 rows (the 64-row tiles of weight-streaming launches), and the
    // tile_rows prefix split in two classes: experts with at least two m-tiles
    // (their tiles reuse a weight tile through L2: tensor-heavy) and the others
    // (weight-streaming), which a launch may interleave; only the passes in
    // pass_mask (bit i: pass i) are written
    for (int pass = 0; pass < 5; ++pass) {
      if (!((pass_mask >> pass) & 1)) continue;        // uniform over the block
      const int rows = pass == 2 ? tile_rows / 2 : (pass == 1 ? tile_rows * 2 : tile_rows);
      int* dst = pass == 0 ? mtiles_out
               : pass == 1 ? mtiles2_out
               : pass == 2 ? mtiles4_out
               : pass == 3 ? mt_hot_out : mt_cold_out;
      __syncthreads();
      for (int e = threadIdx.x; e < n_routed; e += blockDim.x) {
        const int mt = bad ? 0 : (min(counts[e], capacity) + rows - 1) / rows;
        s_run[e] = pass == 3 ? (mt >= 2 ? mt : 0) : (pass == 4 ? (mt == 1 ? 1 : 0) : mt);
      }
      __syncthreads();
      const int total_mt = block_exclusive_scan(s_run, n_routed, s_tmp);
      for (int e = threadIdx.x; e < n_routed; e += blockDim.x) {
        dst[e] = s_run[e];
        s_run[e] = 0;
      }
      if (threadIdx.x == 0) dst[n_routed] = total_mt;
    }
    __syncthreads();
  }

  if (pre_tokens > 0 && !bad) {
    // pairs of this sub-chunk routed before this block's tokens, per expert
    const long long pbase = static_cast<long long>(t0 - pre_tokens) * top_k;
    __syncthreads();
    for (int i = threadIdx.x; i < pre_tokens * top_k; i += blockDim.x) {
      const int e = idx[pbase + i];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(n_routed)) atomicAdd(&s_run[e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) s_pos[i] += s_run[s_e[i]];
    __syncthreads();
    for (int e = threadIdx.x; e < n_routed; e += blockDim.x) s_run[e] = 0;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    for (int b = 0; b < n_ent; b += 32) {
      const int i = b + lane;
      const bool valid = i < n_ent;
      const int e = valid ? s_e[i] : -1;
      const uint32_t same = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(same & ((1u << lane) - 1u));
      if (valid) {
        const int r = s_pos[i] + s_run[e] + rank;   // place among the expert's pairs
        const bool ok = !bad && r >= 0 && r < counts[e];
        if (!ok && !bad) atomicExch(status, 7 /* MOE_DEVICE_INCONSISTENT */);
        s_pos[i] = ok && r < capacity ? s_off[e] + r : -1;  // -1: dropped, no seat left
      }
      __syncwarp();
      if (valid && lane == 31 - __clz(same)) s_run[e] += __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
  if (blockIdx.y == 0)
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
      const int pos = s_pos[i];
      inv_pos[ebase + i] = pos;
      if (pos >= 0) perm_src[pos] = t0 + i / top_k;
    }
  // blockIdx.y selects a column slice of the rows (several slices when the
  // batch has few chunks, so that the copy still spreads over the SMs)
  const int span = (d_vec + gridDim.y - 1) / gridDim.y;
  const int v_begin = blockIdx.y * span;
  const int v_end = min(d_vec, v_begin + span);
  // (no copies when the gate/up GEMM gathers the rows itself: xperm null)
  for (int tl = warp; xperm != nullptr && tl < ntok; tl += kRouteThreads / 32) {
    const uint4* src = x + static_cast<long long>(t0 + tl) * d_vec;
    const int* pos = s_pos + tl * top_k;
    for (int v0 = v_begin + lane; v0 < v_end; v0 += 32 * kCopyUnroll) {
      uint4 val[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u)
        if (v0 + 32 * u < v_end) val[u] = src[v0 + 32 * u];
      for (int j = 0; j < top_k; ++j) {
        if (pos[j] < 0) continue;
        uint4* dst = xperm + static_cast<long long>(pos[j]) * d_vec;
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u)
          if (v0 + 32 * u < v_end) dst[v0 + 32 * u] = val[u];
      }
    }
  }
}

__device__ __forceinline__ void bf16x8_fma(float (&acc)[8], uint4 v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] = fmaf(w, __uint_as_float(u[q] << 16), acc[2 * q]);
    acc[2 * q + 1] = fmaf(w, __uint_as_float(u[q] & 0xFFFF0000u), acc[2 * q + 1]);
  }
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

constexpr int kCombineThreads = 128;
constexpr int kCombineVec = 2;                 // 16-byte column vectors per thread
constexpr int kCombineBatch = 4;               // routed rows loaded before any FMA
constexpr int kCombineCols = kCombineThreads * kCombineVec;

// Grid (T, ceil(d_vec / 256)): block = one token and 256 16-byte column vectors,
// two per thread (strided by 128 so each load instruction is coalesced; two
// rather than four keeps registers low enough for eight resident blocks), all
// k routed rows of a vector loaded before its FMAs. shared (fp32, (T, d)) may
// be null when N_s = 0. The slots are added in order after the shared term; a
// dropped slot (inv_pos -1) adds nothing.
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint4* __restrict__ Y, const float* __restrict__ shared,
                   const int* __restrict__ inv_pos, const float* __restrict__ gate, int top_k,
                   int d_vec, uint4* __restrict__ out, int* __restrict__ router_ticket) {
  __shared__ int s_pos[kMaxTopK];
  __shared__ float s_w[kMaxTopK];
  pdl_launch_dependents();
  pdl_wait();
  // the fused router leaves its ticket at zero; resetting it here as well means
  // a ticket found corrupted in one forward cannot disturb the next
  if (router_ticket && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *router_ticket = 0;
  const long long t = blockIdx.x;
  if (threadIdx.x < top_k) {
    s_pos[threadIdx.x] = inv_pos[t * top_k + threadIdx.x];
    s_w[threadIdx.x] = gate[t * top_k + threadIdx.x];
  }
  __syncthreads();
  const int v0 = blockIdx.y * kCombineCols + threadIdx.x;
  float acc[kCombineVec][8];
#pragma unroll
  for (int u = 0; u < kCombineVec; ++u) {
    const int v = v0 + u * kCombineThreads;
    if (shared && v < d_vec) {
      const float4* s = reinterpret_cast<const float4*>(shared + (t * d_vec + v) * 8);
      const float4 a = s[0], b = s[1];
      acc[u][0] = a.x; acc[u][1] = a.y; acc[u][2] = a.z; acc[u][3] = a.w;
      acc[u][4] = b.x; acc[u][5] = b.y; acc[u][6] = b.z; acc[u][7] = b.w;
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
    }
  }
  for (int j0 = 0; j0 < top_k; j0 += kCombineBatch) {
    uint4 y[kCombineBatch][kCombineVec];
#pragma unroll
    for (int jj = 0; jj < kCombineBatch; ++jj)
#pragma unroll
      for (int u = 0; u < kCombineVec; ++u) {
        const int v = v0 + u * kCombineThreads;
        if (j0 + jj < top_k && v < d_vec && s_pos[j0 + jj] >= 0)
          y[jj][u] = Y[static_cast<long long>(s_pos[j0 + jj]) * d_vec + v];
      }
#pragma unroll
    for (int jj = 0; jj < kCombineBatch; ++jj)
#pragma unroll
      for (int u = 0; u < kCombineVec; ++u)
        if (j0 + jj < top_k && s_pos[j0 + jj] >= 0) bf16x8_fma(acc[u], y[jj][u], s_w[j0 + jj]);
  }
#pragma unroll
  for (int u = 0; u < kCombineVec; ++u) {
    const int v = v0 + u * kCombineThreads;
    if (v < d_vec)
      out[t * d_vec + v] =
          make_uint4(pack2_bf16(acc[u][0], acc[u][1]), pack2_bf16(acc[u][2], acc[u][3]),
                     pack2_bf16(acc[u][4], acc[u][5]), pack2_bf16(acc[u][6], acc[u][7]));
  }
}

}  // namespace moe
