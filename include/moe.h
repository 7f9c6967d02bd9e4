/*
 * moe.h -- C-ABI of the DeepSeekMoE layer forward pass for NVIDIA B200 (sm_100a).
 *
 * What is computed (per token t, hidden vector u_t of width d):
 *   logit[t,i] = u_t . e_i + b_i                 for the N_r routed experts
 *   s[t,:]     = softmax(logit[t,:])              over the routed experts only
 *   sel[t]     = the top_k largest logits, lower expert index first on equal logits
 *   g[t,i]     = s[t,i] if i in sel[t] else 0     (not renormalised)
 *   h_t        = u_t + sum_{j shared} FFN_j(u_t) + sum_{i in sel[t]} g[t,i] FFN_i(u_t)
 *   FFN(x)     = W_down (SiLU(W_gate x) * (W_up x)),  SiLU(z) = z / (1 + exp(-z))
 *   count_i    = #{t : i in sel[t]},  P_i = (1/T) sum_t s[t,i],
 *   aux_loss   = alpha1 * sum_i (count_i / T) * P_i
 * Sources: "DeepSeekMoE: Towards Ultimate Expert Specialization in Mixture-of-Experts
 * Language Models" (deepforge.srivtx.xyz article): section "Routing in a classic MoE
 * layer" (routing equation with residual), "Top-k routing, from affinities to gates"
 * (softmax before the top-k cut, no renormalisation, stable ranking), "Where this sits"
 * (fine-grained segmentation mN/mK and K_s shared experts that every token uses),
 * "Expert-level balance loss" (L_ExpBal = alpha_1 sum_i f_i P_i).  The SwiGLU form of the
 * expert FFN follows the GLU-variants paper cited by the observer.broadside.tech card.
 *
 * Conventions for every entry point:
 *   - Status codes are returned; nothing throws across the ABI.  On failure
 *     moe_last_error() returns a thread-local, NUL-terminated description.
 *   - "device" pointers are CUDA global-memory pointers of the current device; "host"
 *     pointers are ordinary (pageable or pinned) host memory.
 *   - All row-major, no padding between rows.  bf16 is IEEE-like bfloat16 (16-bit).
 *   - stream: a cudaStream_t (NULL = the legacy default stream).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes            */
  MOE_ERR_UNSUPPORTED = 2,  /* a valid layer this build does not handle (see create)  */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                      */
  MOE_ERR_OOM = 4,          /* device allocation failed                               */
  MOE_ERR_DEVICE_CHECK = 5  /* a kernel recorded an error (bounded wait ran out, ...) */
} moe_status;

/* MOE_BF16_E4M3_GATEUP: a bf16 layer (bf16 inputs, weights and outputs) whose gate/up
 * GEMM runs on e4m3 operands -- a reduced-precision variant this library adds (the
 * DeepSeekMoE pages define the layer only in full precision).  Every token row and
 * every gate/up weight row (one output channel, d values) is quantised with its own
 * fp32 scale: a = max |x_i|; a = 0 gives q = 0 and scale 0; otherwise
 * q_i = e4m3(fp32(x_i * fp32(448 / a))) (round to nearest even, saturating at 448) and
 * scale = fp32(a / 448).  The gate/up products are computed on q with fp32 accumulation
 * and multiplied by the two row scales; the router, the down projection, the residual and
 * the combine are those of MOE_BF16.  Needs d % 128 == 0. */
typedef enum { MOE_FP32 = 0, MOE_BF16 = 1, MOE_BF16_E4M3_GATEUP = 2 } moe_dtype;

/* Layer description.  All weight pointers are DEVICE pointers in `dtype`, read only
 * during moe_create (the library keeps its own re-laid-out copy; the caller may free
 * them when moe_create returns).
 *   T          tokens per forward call (fixed per handle; decode and prefill use
 *              separate handles), 1 <= T <= 2^24
 *   d          hidden width;  inter = I, intermediate width of every expert
 *   n_routed   N_r = mN routed experts (1..256);  n_shared = K_s always-on experts
 *   top_k      K' = mK - K_s routed experts per token (1..min(16, N_r))
 *   alpha1     balance-loss factor alpha_1
 *   centroids  [n_routed, d]
 *   logit_bias [n_routed] fp32 added to the logits before the softmax, or NULL
 *   w_gate     [n_shared + n_routed, inter, d]   shared experts first
 *   w_up       [n_shared + n_routed, inter, d]
 *   w_down     [n_shared + n_routed, d, inter]
 * bf16 layers need d % 64 == 0 and inter % 64 == 0 (MOE_ERR_UNSUPPORTED otherwise);
 * MOE_BF16_E4M3_GATEUP layers also d % 128 == 0; fp32 layers need d % 4 == 0.  The
 * weights of MOE_BF16_E4M3_GATEUP layers are given in bf16 and quantised by moe_create. */
typedef struct {
  int32_t T;
  int32_t d;
  int32_t n_routed;
  int32_t n_shared;
  int32_t top_k;
  int32_t inter;
  int32_t dtype; /* moe_dtype */
  float alpha1;
  const void* centroids;
  const float* logit_bias;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} moe_cfg;

typedef struct moe_handle moe_handle;

/* Validate cfg, allocate the handle's device workspace (sized for cfg->T), copy and
 * re-lay-out the weights.  Synchronous (returns after the copies finished) on the
 * current device.  *out is set to NULL on failure. */
moe_status moe_create(const moe_cfg* cfg, moe_handle** out);

/* One forward pass of the layer over cfg->T tokens, enqueued on `stream`; no host
 * synchronisation and no allocation.  All pointers are DEVICE pointers owned by the
 * caller:
 *   u             [T, d] in dtype, 16-byte aligned (input)
 *   h             [T, d] in dtype, 16-byte aligned (output)
 *   topk_idx      [T, top_k] int32 routed expert ids in [0, n_routed), descending logit
 *   topk_w        [T, top_k] fp32 gates g = s at those experts
 *   expert_counts [n_routed] int32
 *   aux_loss      [1] fp32
 * Deterministic: identical inputs give bit-identical outputs.  Calls on one handle must
 * not overlap in time (they share the handle's workspace).  A device-side failure is
 * reported by moe_device_status(). */
moe_status moe_forward(moe_handle* handle, const void* u, void* h, int32_t* topk_idx,
                       float* topk_w, int32_t* expert_counts, float* aux_loss,
                       moe_stream_t stream);

/* moe_forward on HOST buffers: copies u host->device, runs the forward, copies every
 * output device->host and synchronises `stream` before returning.  Sizes as in
 * moe_forward; any output pointer except h_host may be NULL (not copied back). */
moe_status moe_forward_host(moe_handle* handle, const void* u_host, void* h_host,
                            int32_t* topk_idx_host, float* topk_w_host,
                            int32_t* expert_counts_host, float* aux_loss_host,
                            moe_stream_t stream);

/* Pipelined moe_forward on HOST buffers, for a caller that streams batch after batch
 * through one layer.  Enqueues the host->device copy of u, the forward and the
 * device->host copies of the outputs on the handle's own copy-in, forward and copy-out
 * streams and returns without waiting.  The handle double-buffers its device staging, so
 * two calls can be in flight and the copies of one overlap the forward of its neighbours
 * (the two copy directions use separate copy engines).  Ordering: a call's copy-in
 * starts after the work enqueued on `stream` before the call, and after the forward two
 * calls earlier (which read the same staging slot); its forward runs after the copy-out two
 * calls earlier.  Host buffers must be pinned; u_host must stay unchanged and the output
 * buffers unread until moe_pipeline_wait(handle, stream) has been called and `stream`
 * synchronised.  The first call creates the streams and allocates the staging (twice the
 * input and output sizes).  Sizes as in moe_forward; any output except h_host may be NULL.
 * Calls must come from one host thread at a time and must not overlap moe_forward or
 * moe_forward_host calls on the same handle (they share its workspace). */
moe_status moe_forward_host_pipelined(moe_handle* handle, const void* u_host, void* h_host,
                                      int32_t* topk_idx_host, float* topk_w_host,
                                      int32_t* expert_counts_host, float* aux_loss_host,
                                      moe_stream_t stream);

/* Make `stream` wait for every moe_forward_host_pipelined call issued so far (their
 * device->host copies included).  Does not block the host. */
moe_status moe_pipeline_wait(moe_handle* handle, moe_stream_t stream);

/* Synchronise `stream`, then read and clear the handle's device error word.
 * Returns MOE_DEVICE_CHECK (with the kernel's code in moe_last_error()) if any kernel
 * of an earlier forward recorded an error, else MOE_OK. */
moe_status moe_device_status(moe_handle* handle, moe_stream_t stream);

/* Per-expert affinity sums sum_t s[t,i] (fp32, [n_routed], DEVICE) of the most recent
 * forward on this handle, copied on `stream`.  Data-parallel callers all-reduce these
 * together with expert_counts and then call moe_balance_loss with the global T. */
moe_status moe_expert_psum(moe_handle* handle, float* psum, moe_stream_t stream);

/* aux_loss = alpha1 * sum_i (counts[i] / n_tokens) * (psum[i] / n_tokens), one kernel on
 * `stream`, fixed summation order.  counts, psum, aux_loss are DEVICE pointers. */
moe_status moe_balance_loss(const int32_t* counts, const float* psum, int32_t n_routed,
                            int64_t n_tokens, float alpha1, float* aux_loss,
                            moe_stream_t stream);

/* Per-kernel timing.  After moe_timing_begin(handle, n), each of the next n calls of
 * moe_forward on this handle records a CUDA event on its stream before each of its
 * kernels and after the last one (host-side event creation happens here, not in
 * moe_forward).  moe_timing_end synchronises those events, writes the summed elapsed
 * milliseconds of kernel i over the recorded calls to kernel_ms[i] (i < 6: router, scan,
 * permute, gate/up GEMM, down GEMM, combine), the number of recorded calls to
 * *n_forwards, and switches recording off. */
moe_status moe_timing_begin(moe_handle* handle, int32_t max_forwards);
moe_status moe_timing_end(moe_handle* handle, double* kernel_ms, int32_t* n_forwards);

/* ---------------------------------------------------------------------------------
 * Allocation-free router step.  (The DeepSeekMoE pages have no counterpart: this is a
 * deployment convenience of this library.)
 *
 * Some callers cannot call cudaMalloc: code whose GPU memory is owned by another
 * allocator (a framework's caching allocator or a serving engine's arena that has
 * reserved the device's memory and forbids allocations behind its back), and code on a
 * latency-critical path where cudaMalloc/cudaFree would implicitly synchronise the
 * device.  For them moe_route_noalloc runs the routing part of the layer -- the same
 * bf16 tcgen05 router and scan kernels moe_forward uses -- without a handle and without
 * allocating: the kernels' scratch (per-tile expert histograms, within-tile ranks,
 * per-tile affinity sums, tile tables, an error word) lives in one file-scope device
 * array of MOE_NOALLOC_SCRATCH_BYTES, which every GPU that loads this library holds
 * until the process exits.
 *
 * Inputs (DEVICE, 16-byte aligned): u [T, d] bf16; centroids [n_routed, d] bf16;
 * logit_bias [n_routed] fp32 or NULL.  Outputs (DEVICE): topk_idx [T, top_k] int32,
 * topk_w [T, top_k] fp32, expert_counts [n_routed] int32, aux_loss [1] fp32 and, if not
 * NULL, device_error [1] int32 (0, or the code a kernel recorded, e.g. a bounded wait that
 * ran out).  For T > 128 (or d % 128 != 0) these are bit for bit the values moe_forward
 * returns for that layer (the same kernels run).  For decode-sized batches (T <= 128,
 * d % 128 == 0) moe_forward routes with a SIMT kernel that sums each logit in another
 * order: the gates then agree to within fp32 rounding and the routed sets wherever the
 * K'-th and (K'+1)-th affinities are further apart than that rounding.
 * Limits: 1 <= T <= MOE_NOALLOC_MAX_TOKENS, 1 <= n_routed <= MOE_NOALLOC_MAX_ROUTED,
 * 1 <= top_k <= min(MOE_NOALLOC_MAX_TOP_K, n_routed), d a multiple of 64; anything
 * larger returns MOE_ERR_UNSUPPORTED before touching the GPU.
 * The first call on a device does a one-time set-up with that device current (it looks
 * up the array's device address with cudaGetSymbolAddress and reads the compute
 * capability); make that first call before any stream capture.  No call allocates:
 * no cudaMalloc/cudaFree and no allocating library routine.
 * All calls share the one array and each call overwrites it (the error word is cleared
 * at the start of every call), so calls that overlap on the GPU -- on different streams,
 * or from several host threads -- race and give wrong results: serialise them. */
#define MOE_NOALLOC_MAX_TOKENS 16384
#define MOE_NOALLOC_MAX_ROUTED 256
#define MOE_NOALLOC_MAX_TOP_K 16
#define MOE_NOALLOC_SCRATCH_BYTES (2048u * 1024u)
moe_status moe_route_noalloc(const void* u, const void* centroids, const float* logit_bias,
                             int32_t T, int32_t d, int32_t n_routed, int32_t top_k, float alpha1,
                             int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                             float* aux_loss, int32_t* device_error, moe_stream_t stream);

/* Diagnostic (no counterpart on the DeepSeekMoE pages): checks, on the current device,
 * that the library's bounded waits give up.  Runs one one-block kernel whose thread waits,
 * for at most limit_ns nanoseconds (1e6 .. 2e9), on something nothing will complete --
 * kind 0: an mbarrier phase (the wait of the GEMM/router pipelines), kind 1: a global
 * counter (the wait of the fused row copy) -- then synchronises the current stream of the
 * device and stores the error code the kernel recorded in *device_code (HOST pointer):
 * 0x102 for kind 0, 0x105 for kind 1 when the wait ran out as designed.  The kernel
 * returns normally, so the context stays usable.  Allocates a 4-byte word. */
moe_status moe_selftest_wait_timeout(int32_t kind, int64_t limit_ns, int32_t* device_code);

/* Diagnostic (for per-kernel tests): copy one of the handle's workspace buffers, as the
 * most recent forward left it, to DEVICE memory `dst` on `stream` (bytes <= its size), or
 * with dst == NULL only report its size in *size.  which:
 *   0 slot_row [T, top_k] int32   destination row of each (token, slot) in the buffers below
 *   1 xp  [rows_cap, d]    expert-contiguous token rows (layer dtype; e4m3 bytes for
 *                          MOE_BF16_E4M3_GATEUP; unused padding rows are unspecified)
 *   2 hr  [rows_cap, inter] routed experts' SwiGLU activations (bf16 / fp32)
 *   3 yr  [rows_cap, d]    routed experts' outputs before the gates
 *   4 hs  [T_pad, n_shared*inter]  shared experts' activations, experts side by side
 *   5 ys  [T_pad, d]       sum of the shared experts' outputs
 *   6 grp_row [G] int32    first row of each group (shared group first when n_shared > 0)
 * Buffers 4 and 5 are empty (size 0) when n_shared == 0. */
moe_status moe_debug_copy(const moe_handle* handle, int32_t which, void* dst, size_t bytes,
                          size_t* size, moe_stream_t stream);

/* Number of kernels one moe_forward launches on this handle. */
int32_t moe_kernels_per_forward(const moe_handle* handle);

/* Bytes of device memory the handle owns (weights copy + workspace). */
size_t moe_device_bytes(const moe_handle* handle);

/* Free everything the handle owns.  NULL-safe.  Synchronises the device first. */
void moe_destroy(moe_handle* handle);

/* Thread-local description of the last failure on this thread ("" if none). */
const char* moe_last_error(void);

int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
