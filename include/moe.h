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
  MOE_ERR_UNSUPPORTED = 2,  /* a valid layer the library does not handle (see create) */
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
/* MOE_BF16_E4M3: MOE_BF16_E4M3_GATEUP whose down projection runs on e4m3 operands too, with
 * the same per-row rule: each row of the SwiGLU activations (as the layer stores them, in
 * bf16) and each W_down row (one output channel) gets its own scale; the K_s shared
 * experts, which run as one group, quantise the concatenation of their activations and of
 * their W_down rows (one scale per concatenated row).  Needs d % 128 == 0 and
 * inter % 128 == 0. */
typedef enum { MOE_FP32 = 0, MOE_BF16 = 1, MOE_BF16_E4M3_GATEUP = 2, MOE_BF16_E4M3 = 3 } moe_dtype;

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
 * MOE_BF16_E4M3_GATEUP layers also d % 128 == 0, MOE_BF16_E4M3 layers d % 128 == 0 and
 * inter % 128 == 0; fp32 layers need d % 4 == 0.  The weights of the e4m3 variants are
 * given in bf16 and quantised by moe_create. */
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

/* ---------------------------------------------------------------------------------
 * Backward pass of the layer (for training).  The pages give the forward only; the
 * gradients are those of L = sum_t dh_t . h_t + d_aux * aux for the layer above, with the
 * top-k choice (and with it f_i = count_i / T) held fixed: the chosen gates g = s carry
 * the gradient into the affinities and through the softmax ("Routing in a classic MoE
 * layer", "Top-k routing, from affinities to gates"); the balance loss reaches them through
 * P_i ("Expert-level balance loss"); shared experts pass dh to their FFN with gate 1.
 *
 * moe_backward_prepare: once per handle, synchronous; allocates the backward's workspace and
 * transposed copies of the down, gate/up and centroid weights, and makes every later
 * moe_forward on the handle also keep its logits.  bf16 layers on the paired-GEMM path only
 * (MOE_ERR_UNSUPPORTED for fp32 layers, MOE_BF16_E4M3_GATEUP and T <= 128 with
 * d % 128 == 0).
 *
 * moe_backward, on `stream`, after a moe_forward of the same handle on the same u (it reuses
 * that forward's routing, grouped rows and expert outputs, so no other forward may run on the
 * handle in between).  DEVICE pointers: u [T, d] bf16 and topk_idx, topk_w, expert_counts:
 * that forward's input and outputs; dh [T, d] bf16, the incoming gradient of h; d_aux the
 * weight of the balance loss in L.  Outputs: du [T, d] bf16; d_centroids [n_routed, d]
 * fp32; d_bias [n_routed] fp32 (the gradient of a per-expert logit bias) or NULL; and
 * either all or none (NULL) of the weight gradients, fp32 in the layouts of moe_cfg's
 * weights: d_w_gate, d_w_up [n_shared + n_routed, inter, d], d_w_down [n_shared + n_routed,
 * d, inter] (an expert without tokens gets zeros).  Rows of u, dh and du and the weight
 * gradients 16-byte aligned.  Deterministic (fixed-order sums, no atomics). */
moe_status moe_backward_prepare(moe_handle* handle);
moe_status moe_backward(moe_handle* handle, const void* u, const int32_t* topk_idx,
                        const float* topk_w, const int32_t* expert_counts, const void* dh,
                        float d_aux, void* du, float* d_centroids, float* d_bias,
                        float* d_w_gate, float* d_w_up, float* d_w_down, moe_stream_t stream);

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
 * Expert-parallel layer: the routed experts are split over `world` ranks (one GPU each),
 * the tokens stay data-parallel.  Source: the deepforge.srivtx.xyz article, section "Where
 * this sits" (experts spread over devices, whose computation the device-level balance loss
 * keeps even); the arithmetic is the layer's above, and a token's output does not depend
 * on the split.
 *
 * Rank r holds the n_shared shared experts and the routed experts [e0, e0 + n_local),
 * n_local = n_routed / world, e0 = r * n_local.  One forward of T tokens on every rank:
 *   1. moe_ep_dispatch(u) -> topk_idx, topk_w, expert_counts (this rank's tokens),
 *      aux_loss (of this rank's batch), send_rows: the token row of every (token, slot),
 *      T * top_k rows ordered by expert, tokens ascending within an expert -- i.e. the rows
 *      for rank q are the contiguous block of q's experts.
 *   2. caller: all-to-all the per-expert counts (n_local per rank), then the rows, so that
 *      rank q receives from every source s the rows s routed to q's experts, in the order s
 *      sent them: blocks (s, e) for s = 0..world-1, e = 0..n_local-1.
 *   3. moe_ep_experts(recv_rows, recv_counts [world, n_local], n_recv) -> out_rows: each
 *      received row through its expert's SwiGLU FFN, same row order.
 *   4. caller: the reverse all-to-all (each rank gets back its send_rows' outputs).
 *   5. moe_ep_combine(u, back_rows, topk_w) -> h = u + sum_shared FFN_j(u) +
 *      sum_k g_k * back_rows[row of (t, k)].
 * The global balance loss: all-reduce expert_counts and moe_ep_expert_psum's sums over
 * the ranks, then moe_balance_loss with the global token count.
 */
typedef struct moe_ep_handle moe_ep_handle;

/* cfg as for moe_create (bf16 layers only; n_routed % world == 0), except that w_gate,
 * w_up and w_down hold [n_shared + n_local, ...] experts: the shared ones, then this rank's
 * routed experts e0 .. e0 + n_local - 1; centroids and logit_bias cover all n_routed
 * experts.  recv_capacity: the most rows moe_ep_experts will be given (0 = world * T *
 * top_k: every rank's rows when all ranks route T tokens; pass the sum over the ranks of
 * T_rank * top_k when their token counts differ).  Synchronous; *out = NULL on failure. */
moe_status moe_ep_create(const moe_cfg* cfg, int32_t rank, int32_t world, int64_t recv_capacity,
                         moe_ep_handle** out);

/* Step 1 on `stream`.  DEVICE pointers: u [T, d] bf16 (16-byte aligned); outputs topk_idx,
 * topk_w [T, top_k], expert_counts [n_routed] int32, aux_loss [1], send_rows [T * top_k, d]
 * bf16 (16-byte aligned).  Row j of send_rows belongs to (token, slot) pairs in the order
 * described above. */
moe_status moe_ep_dispatch(moe_ep_handle* handle, const void* u, int32_t* topk_idx,
                           float* topk_w, int32_t* expert_counts, float* aux_loss,
                           void* send_rows, moe_stream_t stream);

/* Step 3 on `stream`.  recv_rows [n_recv, d] bf16 and recv_counts [world, n_local] int32
 * (DEVICE; sum = n_recv, which the caller also passes on the host), out_rows [n_recv, d]
 * bf16 (DEVICE).  n_recv <= the handle's recv capacity (MOE_ERR_INVALID_ARG otherwise). */
moe_status moe_ep_experts(moe_ep_handle* handle, const void* recv_rows,
                          const int32_t* recv_counts, int64_t n_recv, void* out_rows,
                          moe_stream_t stream);

/* Step 5 on `stream`.  u [T, d] (the dispatch's input), back_rows [T * top_k, d] (step 4's
 * result, in send_rows' order), topk_w [T, top_k] (the dispatch's gates), h [T, d]; all
 * DEVICE, bf16 rows 16-byte aligned.  Uses the row order of the most recent dispatch. */
moe_status moe_ep_combine(moe_ep_handle* handle, const void* u, const void* back_rows,
                          const float* topk_w, void* h, moe_stream_t stream);

/* Per-expert affinity sums [n_routed] (fp32, DEVICE) of the most recent dispatch. */
moe_status moe_ep_expert_psum(moe_ep_handle* handle, float* psum, moe_stream_t stream);

/* As moe_device_status, for the expert-parallel handle. */
moe_status moe_ep_device_status(moe_ep_handle* handle, moe_stream_t stream);

/* The received-row capacity fixed at create (0 for NULL). */
int64_t moe_ep_recv_capacity(const moe_ep_handle* handle);

/* Free everything the handle owns.  NULL-safe.  Synchronises the device first. */
void moe_ep_destroy(moe_ep_handle* handle);

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
 *   7 row_tok [rows_cap] int32  token of each routed row (decode-sized path: T <= 128
 *                          bf16 layers with d % 128 == 0; else empty)
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
