/*
 * moe_ffn.h - C ABI of libmoe_ffn.so: forward pass of a mixture-of-experts
 * feed-forward layer with fine-grained routed experts and an always-on shared
 * expert, on one NVIDIA B200 (sm_100a).
 *
 * What the library computes (one call of moe_forward, T tokens of width d):
 *
 *   s[t,e]  = x[t,:] . W_g[e,:] + bias[e]                 router scores
 *   p[t,:]  = softmax(s[t,:]) over all N_r routed experts
 *   S_t     = the top_k experts by p, ties to the lower expert index
 *   g[t,i]  = p[t,i]            (renorm = 0), or
 *             p[t,i] / sum_{j in S_t} p[t,j]   (renorm = 1), for i in S_t
 *   out[t]  = FFN_shared(x[t]) + sum_{i in S_t} g[t,i] * FFN_i(x[t])
 *   FFN(u)  = W2 ( SiLU(W1 u) * (W3 u) ),   SiLU(z) = z / (1 + exp(-z))
 *
 * Sources: "Shared Expert (DeepSeek-V3)" (ai-engineer-exhaustive), "How it
 * works": eq. (12) without its residual term u_t (the caller adds the residual
 * at block level), the SwiGLU definition, and "Official code" (N_s shared
 * experts fused into one SwiGLU of inner width N_s*f, computed on the whole
 * packed batch and added with coefficient 1, never gated, never in the top-k
 * pool). The router (linear scorer, softmax blend weights, keep the top-k) is
 * "What is an "expert," really?" (svac-llc), glossary and panel 2; the
 * selected-set sum is "Shared and fine-grained experts", Researcher "Why
 * segmentation helps".
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    16-byte aligned. bf16 tensors are passed as uint16_t bit patterns.
 *  - Layouts: x (T, d); W_g (N_r, d); W1, W3 (N_r, f, d); W2 (N_r, d, f);
 *    W1s, W3s (N_s*f, d); W2s (d, N_s*f); bias (N_r) fp32; out (T, d).
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream. Calls that take a stream only enqueue work: they never
 *    synchronise the host and never allocate device memory.
 *  - Every call returns a moe_status (0 = OK). On failure, moe_last_error()
 *    returns a message for the calling thread.
 *  - A plan is not thread-safe: do not run two forwards of one plan at the
 *    same time. Distinct plans are independent.
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t;               /* bf16 bit pattern */
typedef struct moe_plan* moe_plan_t;      /* opaque, owned by the library */

typedef enum {
  MOE_OK = 0,
  MOE_INVALID_CONFIG = 1,   /* layer shape rejected (see moe_plan_create) */
  MOE_INVALID_ARG = 2,      /* null or misaligned pointer, negative T, ... */
  MOE_WORKSPACE_TOO_SMALL = 3,
  MOE_CUDA_ERROR = 4,       /* a CUDA runtime/driver call or launch failed */
  MOE_UNSUPPORTED = 5,      /* valid layer the kernels do not cover */
  MOE_DEVICE_TIMEOUT = 6,   /* a kernel gave up a bounded wait (see moe_plan_device_status) */
  MOE_DEVICE_INCONSISTENT = 7 /* the permutation kernel found routing totals that do not add
                                 up (scratch overwritten during a forward); that forward wrote
                                 no grouped rows and dropped every routed slot */
} moe_status;

/* Create a plan for one layer shape.
 * d: model width; f: inner width of one routed expert; n_routed: N_r;
 * top_k: experts kept per token; n_shared: N_s (shared inner width N_s*f);
 * renorm: 1 to renormalise the selected probabilities to sum 1, 0 for raw.
 * Rejected with MOE_INVALID_CONFIG (returns NULL) when any of d, f, N_r, top_k
 * is below 1, N_s is negative or top_k exceeds N_r - the budget rules of
 * "MoE：细粒度专家与共享专家（shared expert）" (cooking-agi), budget section.
 * Returns NULL with MOE_UNSUPPORTED when d or f is not a multiple of 8
 * (16-byte rows), N_r > 1024, top_k > 32 or N_s*f > 2^24.
 * The plan is bound to the CUDA device current at creation. */
moe_plan_t moe_plan_create(int d, int f, int n_routed, int top_k, int n_shared,
                           int renorm);

/* Status of the last moe_plan_create on this thread (MOE_OK if it succeeded). */
int moe_last_status(void);

/* Tuning options (moe_plan_set_option). Results do not depend on them.
 * MOE_OPTION_PAIR_MIN_ROWS: a GEMM whose expected rows per expert group
 *   (T*top_k/N_r for the routed experts, T for the shared expert) reach this
 *   value runs as CTA pairs (tcgen05 cta_group::2, 256-row tiles, two SMs per
 *   tile); smaller groups run one CTA per 128-row tile. By default only the
 *   routed down projection uses pairs, from 256 rows per expert; setting the
 *   option applies the value to every GEMM (0 always uses pairs, a value above
 *   any T*top_k never does).
 * MOE_OPTION_WIDE_TILES: CTA-pair tiles of 512 accumulator columns instead of
 *   256 (fewer operand bytes per FLOP, fewer tiles). -1 (default) chooses per
 *   GEMM (wide for reductions of at least 4096 with at least 3 waves of
 *   tiles), 0 never, 1 always.
 * MOE_OPTION_MERGE_SHARED: when a routed GEMM runs one CTA per tile, compute
 *   the matching shared GEMM as extra tiles of that same launch, spread evenly
 *   among the routed tiles. -1 (the default): automatic - merged when the shared
 *   expert is small (at most half the SMs' worth of 128 x 128 tiles, the decode
 *   regime) and the routed tile options are at their defaults; a larger shared
 *   expert runs as its own launches (merged, it measured slower on B200 for the
 *   DeepSeek-V3 layer shape). 0: never (a small shared expert then runs on the
 *   plan's side stream beside the routing). 1: whenever possible (a merged
 *   launch uses the default routed tile shape). Results are the same bits
 *   either way.
 * MOE_OPTION_EXPERT_CAPACITY: seats per expert per forward ("What is an
 *   'expert,' really?", glossary: capacity factor / token dropping, each expert
 *   has a seat limit per batch and overflow tokens are skipped). 0 (default):
 *   unlimited, the layer is dropless. C > 0: expert e keeps the first
 *   min(count_e, C) of the (token, slot) pairs routed to it, in ascending
 *   (token, slot) order; a dropped pair adds nothing to its token's output, the
 *   kept gates are not renormalised and the shared expert still applies. This
 *   option changes results; the others do not (setting it turns the capacity
 *   factor below off).
 * MOE_OPTION_CAPACITY_FACTOR_PERMILLE: the same token dropping stated as the
 *   glossary's capacity factor cf, passed in thousandths (1000 = 1.0; 0, the
 *   default, turns it off). A forward over T tokens then gives each expert
 *   C = max(1, ceil(cf * T * top_k / N_r)) seats - the factor times an
 *   expert's even share of the batch's T*top_k routed pairs (the glossary
 *   names the factor without a formula; this is the conventional one). Setting
 *   it turns MOE_OPTION_EXPERT_CAPACITY off. moe_plan_capacity_seats reports C.
 * MOE_OPTION_BIAS_SELECTION_ONLY: 0 (default): the logit bias set with
 *   moe_plan_set_logit_bias is added to the router scores for both the top-k
 *   selection and the gates. 1: it only chooses the experts (the selection-only
 *   load-balance bias "Shared Expert (DeepSeek-V3)" mentions for the routed
 *   centroids); the gates are the softmax of the unbiased scores over all N_r
 *   experts, renormalised over the selected ones when the plan renormalises.
 * MOE_OPTION_FUSED_ROUTER: 1 computes the router in one kernel (scores on
 *   the tensor core, softmax, top-k, gates and the expert histogram of each
 *   128-token tile, its experts split over a cluster of up to 8 CTAs, and with
 *   few tiles the histogram scan) whenever N_r <= 512 and top_k <= 16; 0 and
 *   -1 (default, measured faster on B200 for every tested shape) use the
 *   two-kernel router (a split-K scores GEMM, then softmax + top-k, then the
 *   histogram scan). Both give the same selection up to fp32 rounding of the
 *   scores.
 * MOE_OPTION_SWIGLU_TILE_COLS: output columns of one tile of the routed
 *   gate/up GEMM when it runs one CTA per tile: 0 (default) is 128 (N=256
 *   MMAs: on B200 an MMA instruction costs about the same time at any size, so
 *   the widest moves the most weight bytes, also in the weight-streaming
 *   decode regime); 32 or 64 (more, narrower tiles) or 128 force it.
 * MOE_OPTION_DOWN_TILE_COLS: output columns of one tile of the routed down
 *   GEMM when it runs one CTA per tile: 0 (default) is 256; 128 or 256.
 * MOE_OPTION_TILE_ROWS: rows of one tile of the routed GEMMs when they run
 *   one CTA per tile: 0 (default) is 128; 64 (M=64 MMAs and 64-row boxes of the
 *   grouped rows: smaller pipeline stages, so more of them) or 128 force it.
 * MOE_OPTION_INTERLEAVE: order of the tiles of the routed GEMMs when they run
 *   one CTA per 128-row tile. 1: the tiles of experts with at least two
 *   m-blocks (tensor-heavy, their weight tiles reused through L2) are spread
 *   evenly among the other experts' tiles (weight streaming), so that tensor
 *   and HBM work overlap; 0: expert order; -1 (default): 1 when the expected
 *   rows per expert (T*top_k/N_r) are from 32 to 191.
 * MOE_OPTION_SHARED_CONCURRENT: where a shared expert too large for the
 *   routing phase runs. 1: beside the routed GEMMs, on a second stream and a
 *   few SMs (the routed GEMMs keep the rest); -1 (default) and 0: after them on
 *   the caller's stream (measured faster on B200 for the DeepSeek-V3 layer
 *   shape). Small shared experts always run beside the routing kernels.
 * MOE_OPTION_CTAS_PER_SM: CTAs per SM of the routed GEMMs when they run one
 *   CTA per tile. 2: two resident CTAs per SM, each with half the pipeline
 *   ring and half the tensor memory (two independent pipelines per SM; measured
 *   no faster on B200, where the SM's MMA issue rate, shared by both, is the
 *   limit); 1 and 0 (default): one CTA per SM with the whole ring.
 * MOE_OPTION_GATHER_ROWS: 1 lets the routed gate/up GEMM, when it runs one CTA
 *   per tile, gather its rows from x through the permutation (its producer
 *   warps copy them into the pipeline with cp.async), so that the permutation
 *   kernel writes no permuted row copies; 0 keeps the copies and the
 *   tensor-map loads of them; -1 (default) gathers when the expected rows per
 *   expert (T*top_k/N_r) are below 32 (decode). The same results bit for bit.
 * MOE_OPTION_TEST_WAIT_TIMEOUT: test hook for the failure path, not for normal
 *   use. Value 1 arms it for the next forward only: if that forward runs the
 *   routed gate/up GEMM on the one-CTA-per-tile kernel, one CTA withholds the
 *   loads of its first pipeline stage, its MMA warp's bounded wait (2 s) expires,
 *   and the kernel sets the device status to MOE_DEVICE_TIMEOUT, drains its
 *   copies, frees its tensor memory and returns; that forward's output is
 *   invalid, the context stays usable. No fault, trap or unbounded wait. */
enum {
  MOE_OPTION_PAIR_MIN_ROWS = 1,
  MOE_OPTION_WIDE_TILES = 2,
  MOE_OPTION_MERGE_SHARED = 3,
  MOE_OPTION_EXPERT_CAPACITY = 4,
  MOE_OPTION_BIAS_SELECTION_ONLY = 5,
  MOE_OPTION_CAPACITY_FACTOR_PERMILLE = 6,
  MOE_OPTION_FUSED_ROUTER = 7,
  MOE_OPTION_SWIGLU_TILE_COLS = 8,
  MOE_OPTION_SHARED_CONCURRENT = 9,
  MOE_OPTION_TILE_ROWS = 10,
  MOE_OPTION_INTERLEAVE = 11,
  MOE_OPTION_CTAS_PER_SM = 12,
  MOE_OPTION_DOWN_TILE_COLS = 13,
  MOE_OPTION_GATHER_ROWS = 14,
  MOE_OPTION_TEST_WAIT_TIMEOUT = 100
};
int moe_plan_set_option(moe_plan_t plan, int option, int64_t value);

/* Optional per-expert logit bias: device pointer to N_r fp32 values added to
 * the router scores before the softmax (affects both selection and gates).
 * NULL removes it. The pointer must stay valid while forwards use it. */
int moe_plan_set_logit_bias(moe_plan_t plan, const float* bias);

/* Bytes of device workspace one forward over T tokens needs (T >= 0). */
size_t moe_workspace_bytes(moe_plan_t plan, int64_t T);

/* Hand the plan a caller-owned device workspace (256-byte aligned). The plan
 * keeps the pointer; forwards over T tokens need moe_workspace_bytes(T).
 * The workspace also holds the routing of the last forward. */
int moe_plan_set_workspace(moe_plan_t plan, void* workspace, size_t bytes);

/* Forward over T tokens (T = 0 is a no-op returning MOE_OK). x, W_g, W1, W3,
 * W2 and out must be non-NULL; W1s, W3s, W2s must be NULL exactly when N_s = 0.
 * Enqueues the whole layer on `stream`: router GEMM, softmax + top-k, expert
 * histogram + scan + stable permutation, grouped gate/up + SiLU GEMM, grouped
 * down GEMM, shared SwiGLU GEMMs, weighted combine. No host synchronisation,
 * no device allocation. Errors: MOE_INVALID_ARG, MOE_WORKSPACE_TOO_SMALL,
 * MOE_CUDA_ERROR (launch failures are reported, in-kernel faults surface at the
 * next synchronising CUDA call). */
int moe_forward(moe_plan_t plan, int64_t T, const moe_bf16_t* x,
                const moe_bf16_t* W_g, const moe_bf16_t* W1, const moe_bf16_t* W3,
                const moe_bf16_t* W2, const moe_bf16_t* W1s,
                const moe_bf16_t* W3s, const moe_bf16_t* W2s, moe_bf16_t* out,
                void* stream);

/* Copy the routing of the last forward (device to device, enqueued on
 * `stream`): idx (T, top_k) int32 expert ids in slot order (descending
 * probability, ties to the lower index); w (T, top_k) fp32 gates; counts (N_r)
 * int32 (token, slot) pairs routed to each expert; offsets (N_r+1) int32
 * exclusive prefix of the rows each expert kept (of counts, unless an expert
 * capacity dropped pairs). Any output may be NULL. T must equal the last
 * forward's T. */
int moe_get_routing(moe_plan_t plan, int64_t T, int32_t* idx, float* w,
                    int32_t* counts, int32_t* offsets, void* stream);

/* Copy the stable permutation of the last forward (device to device):
 * perm_src (T*top_k) int32 token of each grouped row (rows of expert e are
 * offsets[e]..offsets[e+1]-1, in ascending (token, slot) order; entries past
 * offsets[N_r] are unspecified when pairs were dropped);
 * inv_pos (T, top_k) int32 grouped row of each (token, slot), -1 for a pair
 * dropped by the expert capacity. NULL skips. */
int moe_get_permutation(moe_plan_t plan, int64_t T, int32_t* perm_src,
                        int32_t* inv_pos, void* stream);

/* Read (synchronously) and clear the plan's device status: MOE_OK, or
 * MOE_DEVICE_TIMEOUT if a kernel abandoned a bounded wait since the last read
 * (MOE_DEVICE_INCONSISTENT if the permutation kernel found inconsistent routing
 * state).
 * It covers the forwards that ran on the plan's workspace and, when this plan
 * has run moe_forward_noalloc since the last read, the status word of the
 * static scratch those forwards share (one word for every plan of the
 * process: a read through any plan that used it clears it). Kernels never spin
 * without a bound; a timeout means that forward's output is invalid. */
int moe_plan_device_status(moe_plan_t plan);

/* Timing: when enabled, moe_forward records a CUDA event on its stream before
 * every kernel launch and after the last one, into one of 4 event sets used in
 * turn, so the host can read forward i-1 while forward i is still queued.
 * moe_plan_kernel_times waits for the final event of the timed forward `back`
 * steps before the latest one (0 = latest, at most 3) and writes up to `cap`
 * per-kernel durations in milliseconds; it returns how many kernels that
 * forward launched, or a negative moe_status. moe_plan_kernel_name gives the
 * name of kernel i of the last forward, with "[pair]" or "[pair512]" appended
 * for the CTA-pair GEMM variants (owned by the plan, valid until the next
 * forward; NULL when out of range). */
int moe_plan_enable_timing(moe_plan_t plan, int enable);
int moe_plan_kernel_times(moe_plan_t plan, int back, float* ms, int cap);
const char* moe_plan_kernel_name(moe_plan_t plan, int i);

/* Forward for callers that cannot allocate device memory - for instance a
 * plugin whose host application owns the whole device-memory budget through
 * its own pool, or a latency-critical loop where cudaMalloc would synchronise
 * the device. The pages have no counterpart of this call; it is a deployment
 * convenience. Same arguments and result as moe_forward, but the scratch the
 * layer needs lives in one static device array of 32 MiB inside the library
 * (held on every GPU that loads the library until the process exits) instead
 * of the plan's workspace; the caller passes only inputs and outputs, and the
 * call allocates nothing. T whose scratch would exceed 32 MiB is rejected with
 * MOE_WORKSPACE_TOO_SMALL before anything is enqueued (the 512-expert decode
 * shape d=2048, f=512, N_r=512, k=10, N_s=1 needs about 13 MiB at T=128).
 * moe_plan_create looks up the array's device address (with the plan's device
 * current), so the call itself makes no lookup. All calls share the one array
 * and it keeps the last call's contents: two calls that overlap on the GPU
 * (different streams, plans or threads) race, so keep them on one stream.
 * Timing events are not recorded. The plan's routing, permutation, launch
 * count and kernel-name getters keep describing the last moe_forward; a
 * bounded-wait timeout is reported by moe_plan_device_status. */
int moe_forward_noalloc(moe_plan_t plan, int64_t T, const moe_bf16_t* x,
                        const moe_bf16_t* W_g, const moe_bf16_t* W1,
                        const moe_bf16_t* W3, const moe_bf16_t* W2,
                        const moe_bf16_t* W1s, const moe_bf16_t* W3s,
                        const moe_bf16_t* W2s, moe_bf16_t* out, void* stream);

/* Number of kernels the last forward of this plan launched. */
int moe_plan_last_launch_count(moe_plan_t plan);

/* Seats per expert a forward over T tokens gives each expert under the plan's
 * capacity options (0: unlimited, the layer is dropless); a negative
 * moe_status on a NULL plan or negative T. Host only, enqueues nothing. */
int64_t moe_plan_capacity_seats(moe_plan_t plan, int64_t T);

void moe_plan_destroy(moe_plan_t plan);

const char* moe_strerror(int status);
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FFN_H */
