// moe_api.cu -- the C-ABI (include/moe.h): validation, weight re-layout, workspace,
// TMA descriptors and the launch sequence of one DeepSeekMoE layer forward pass.
//
// Launch sequence of moe_forward (one stream, no host synchronisation, every launch with
// programmatic dependent launch):
//   1. router      logits -> softmax -> top-k, gates, per-tile histograms / ranks / sums
//                  (tensor-core kernel; a SIMT kernel for decode-sized batches and fp32)
//   2. scan        per-expert counts, padded offsets, tile tables, balance loss
//   3. quantise    (e4m3 gate/up layers only) e4m3 token rows + per-row scales
//   4. permute     token rows -> expert-contiguous rows (top_k copies per token); on bf16
//                  layers with shared experts this copy runs inside step 5 instead
//   5. gate/up     grouped GEMM + SwiGLU (shared group reads the token rows directly)
//   6. down        grouped GEMM
//   7. combine     h = u + shared + sum_k g_k * routed_k (fp32, fixed order)
#include <algorithm>
#include <cstring>
#include <string>
#include <vector>

#include "moe.h"
#include "api_common.cuh"
#include "backward.cuh"
#include "combine.cuh"
#include "gemm_simt.cuh"
#include "gemm_small.cuh"
#include "gemm_tc.cuh"
#include "router.cuh"
#include "quant.cuh"
#include "scan_permute.cuh"

using namespace moe;

namespace {

thread_local std::string g_last_error;

// Quantise `rows` bf16 rows of `cols` values to e4m3 with per-row scales, on `st`.
cudaError_t launch_quant(const void* src, int64_t rows, int cols, void* dst, float* scale,
                         int n_sms, cudaStream_t st) {
  int64_t blocks = (rows + kQuantWarps - 1) / kQuantWarps;
  if (blocks > (int64_t)n_sms * 16) blocks = (int64_t)n_sms * 16;
  QuantArgs qa{static_cast<const __nv_bfloat16*>(src), rows, cols, static_cast<uint8_t*>(dst), scale};
  return launch_pdl(quant_rows_e4m3_kernel, dim3((unsigned)blocks), dim3(kQuantWarps * 32), 0, st, qa);
}

__device__ int g_never_set = 0;   // a counter no kernel writes (bounded-wait self-test)

__global__ void wait_selftest_kernel(int kind, uint64_t limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);   // expects one arrival, which never comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (kind == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, kErrWaitMma, limit_ns);
    else counter_wait(&g_never_set, 1, &abort_flag, err, kErrWaitCopy, limit_ns);
  }
}

__global__ void balance_loss_kernel(const int32_t* counts, const float* psum, int n, double inv_t,
                                    float alpha1, float* out) {
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += ((double)counts[i] * inv_t) * ((double)psum[i] * inv_t);
    *out = (float)((double)alpha1 * acc);
  }
}

constexpr int kKernelsPerForward = 6;
// counters of the fused row copy and of the decode FFN kernel's groups (1 + G <= 2 + kMaxRouted)
constexpr size_t kSyncBytes = 2048;
static_assert(kSyncBytes >= 4 * (2 + kMaxRouted), "per-group counters");

}  // namespace

namespace moe {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace moe

struct moe_handle {
  moe_cfg cfg;
  int device = 0, n_sms = 0;
  bool bf16 = true;        // bf16 storage (MOE_BF16 and MOE_BF16_E4M3_GATEUP)
  bool e4m3 = false;       // gate/up GEMM on e4m3 operands (MOE_BF16_E4M3_GATEUP, MOE_BF16_E4M3)
  bool e4m3_down = false;  // down GEMM on e4m3 operands too (MOE_BF16_E4M3)
  int es = 2;              // element size
  int G = 0, has_shared = 0, inter_shared = 0;
  int n_tiles = 0;         // router tiles
  int router_cluster = 1;  // CTAs per token of the decode-sized router
  int router_rows = 0;     // tokens per router tile
  int64_t T_pad = 0, rows_cap = 0;   // padded to bm, the GEMM row tile
  int bm = 0, tile_rows = 0;
  int gemm_grid = 0;                  // CTAs of the paired-SM GEMMs (2 per cluster)
  int gemm_grid_f8 = 0;               // same, e4m3 gate/up GEMM
  // small-batch (decode) path: token counts <= n_tok, weights on the MMA's M dimension
  bool small = false;
  int n_tok = 0, small_stages = 0;
  size_t small_smem = 0;
  int n_pad = 0, maxk = 16, maxc = 32;
  int router_stages = 0, router_kps = 1;
  uint32_t router_tmem_cols = 0;
  size_t router_smem = 0, simt_router_smem = 0;
  // weights (library-owned, re-laid-out)
  void* centroids = nullptr;
  float* bias = nullptr;
  void* w_gu_s = nullptr;  // bf16 [2*inter_shared, d], gate/up interleaved by 64 rows
  void* w_gu_r = nullptr;  // bf16 [n_routed, 2*inter, d]
  void* w_g = nullptr;     // fp32 [G, inter, d]
  void* w_u = nullptr;     // fp32 [G, inter, d]
  void* w_d_s = nullptr;   // [d, inter_shared]
  void* w_d_r = nullptr;   // [n_routed, d, inter]
  // workspace
  int32_t *topk_rank = nullptr, *slot_row = nullptr, *tile_hist = nullptr, *tile_base = nullptr;
  int32_t *grp_row = nullptr, *ts1 = nullptr, *ts2 = nullptr;
  float *tile_psum = nullptr, *psum_total = nullptr;
  void *xp = nullptr, *hs = nullptr, *hr = nullptr, *ys = nullptr, *yr = nullptr;
  int* err = nullptr;
  int* copy_done = nullptr;   // counters of the fused row copy (paired bf16 path with a shared
                              // group; decode FFN kernel: also one per group, see SmallGemmArgs)
  int32_t* row_tok = nullptr; // [rows_cap] token of each routed row (decode-sized path: the
                              // scan places the rows, the decode FFN kernel's epilogue warps copy them)
  // e4m3 gate/up: quantised weights (interleaved rows), per-row scales, quantised tokens
  void *w8_gu_s = nullptr, *w8_gu_r = nullptr, *u8 = nullptr;
  float *sw_s = nullptr, *sw_r = nullptr, *su = nullptr, *su_p = nullptr;
  CUtensorMap tmU8, tmXp8, tmW8guS, tmW8guR;
  // e4m3 down projection: quantised W_down rows and activation rows, their scales
  void *w8_d_s = nullptr, *w8_d_r = nullptr, *h8s = nullptr, *h8r = nullptr;
  float *sw_d_s = nullptr, *sw_d_r = nullptr, *sh_s = nullptr, *sh_r = nullptr;
  CUtensorMap tmH8s, tmH8r, tmW8dS, tmW8dR;
  bool fuse_permute = false;
  // staging for moe_forward_host
  void *u_dev = nullptr, *h_dev = nullptr;
  int32_t *idx_dev = nullptr, *cnt_dev = nullptr;
  float *w_dev = nullptr, *aux_dev = nullptr;
  CUtensorMap tmE, tmXp, tmWguS, tmWguR, tmHs, tmHr, tmWdS, tmWdR;
  CUtensorMap tmXpN, tmHsN, tmHrN;   // token operands of the decode FFN kernel (n_tok rows)
  CUtensorMap tmWguS64, tmWguR64;    // gate/up weights in 64-row boxes (decode FFN kernel)
  // moe_forward_host_pipelined: copy-in / forward / copy-out streams, two staging slots
  struct PipeSlot {
    void *u = nullptr, *h = nullptr;
    int32_t *idx = nullptr, *cnt = nullptr;
    float *w = nullptr, *aux = nullptr;
    cudaEvent_t in_done = nullptr, comp_done = nullptr, out_done = nullptr;
    bool used = false;
  };
  cudaStream_t p_in = nullptr, p_c = nullptr, p_out = nullptr;
  cudaEvent_t p_entry = nullptr;
  PipeSlot pslot[2];
  int64_t p_calls = 0;
  bool p_ready = false;
  // backward (moe_backward_prepare): the forward's logits, transposed weight copies and the
  // backward's workspace
  bool bwd = false;
  bool bwd_forward = false;                // a forward ran since moe_backward_prepare
  int kpad = 0;                            // n_pad rounded up to 64: K of the e-product GEMM
  float* logits = nullptr;                 // [T, n_routed]
  int32_t* ts3 = nullptr;                  // [G + 1] dHmid GEMM tiles (N = I at 256 per tile)
  void *w_dT_s = nullptr, *w_dT_r = nullptr;     // [Is, d], [n_routed, I, d]
  void *w_guT_s = nullptr, *w_guT_r = nullptr;   // [d, 2 Is], [n_routed, d, 2 I] (interleaved K)
  void* e_T = nullptr;                            // [d, kpad] centroids transposed (zero-padded)
  void *dyr = nullptr, *dhr = nullptr, *dhs = nullptr, *dabr = nullptr, *dabs = nullptr;
  void *dxr = nullptr, *dxs = nullptr, *dur = nullptr, *dlb = nullptr;
  float *dg = nullptr, *dl = nullptr, *cen_part = nullptr;
  int32_t *r_grp = nullptr, *r_ts = nullptr;      // one-group tables of the e-product GEMM
  // weight gradients: transposed activations [width, rows] (padding rows zero) and the
  // (static) tile tables of the dW_gate/up and dW_down GEMMs
  void *xpT = nullptr, *dyrT = nullptr, *hrT = nullptr, *dabrT = nullptr;
  void *uT = nullptr, *dhT = nullptr, *hsT = nullptr, *dabsT = nullptr;
  int32_t *wts1 = nullptr, *wts2 = nullptr;
  CUtensorMap tmXpT, tmDyrT, tmHrT, tmDabrT, tmUT, tmDhT, tmHsT, tmDabsT;
  int cen_chunks = 0;
  CUtensorMap tmDyr, tmWdTs, tmWdTr, tmDabs, tmDabr, tmWguTs, tmWguTr, tmDlb, tmEt;
  // per-kernel timing (moe_timing_begin / moe_timing_end)
  std::vector<cudaEvent_t> events;   // kKernelsPerForward + 1 per recorded call
  int timing_cap = 0, timing_used = 0;
  std::vector<void*> allocs;
  size_t bytes = 0;
};

namespace {

moe_status dalloc(moe_handle* H, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return MOE_OK;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(MOE_ERR_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  H->allocs.push_back(*p);
  H->bytes += bytes;
  return MOE_OK;
}

void free_handle(moe_handle* H) {
  if (!H) return;
  for (cudaEvent_t e : H->events) cudaEventDestroy(e);
  for (auto& P : H->pslot)
    for (cudaEvent_t e : {P.in_done, P.comp_done, P.out_done})
      if (e) cudaEventDestroy(e);
  if (H->p_entry) cudaEventDestroy(H->p_entry);
  for (cudaStream_t st : {H->p_in, H->p_c, H->p_out})
    if (st) cudaStreamDestroy(st);
  for (void* p : H->allocs) cudaFree(p);
  delete H;
}

moe_status validate(const moe_cfg* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->T < 1 || c->T > (1 << 24)) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [1, 2^24]", c->T);
  if (c->d < 1 || c->inter < 1) return fail(MOE_ERR_INVALID_ARG, "d and inter must be positive");
  if (c->n_routed < 1 || c->n_routed > kMaxRouted)
    return fail(MOE_ERR_UNSUPPORTED, "n_routed=%d outside [1, %d]", c->n_routed, kMaxRouted);
  if (c->n_shared < 0 || c->n_shared > 64)
    return fail(MOE_ERR_INVALID_ARG, "n_shared=%d outside [0, 64]", c->n_shared);
  if (c->top_k < 1 || c->top_k > c->n_routed)
    return fail(MOE_ERR_INVALID_ARG, "top_k=%d outside [1, n_routed=%d]", c->top_k, c->n_routed);
  if (c->top_k > kMaxTopK)
    return fail(MOE_ERR_UNSUPPORTED, "top_k=%d above %d", c->top_k, kMaxTopK);
  if (c->dtype != MOE_FP32 && c->dtype != MOE_BF16 && c->dtype != MOE_BF16_E4M3_GATEUP &&
      c->dtype != MOE_BF16_E4M3)
    return fail(MOE_ERR_INVALID_ARG,
                "dtype=%d is not MOE_FP32, MOE_BF16, MOE_BF16_E4M3_GATEUP or MOE_BF16_E4M3", c->dtype);
  if (!c->centroids || !c->w_gate || !c->w_up || !c->w_down)
    return fail(MOE_ERR_INVALID_ARG, "a weight pointer is NULL");
  if ((c->dtype == MOE_BF16_E4M3_GATEUP || c->dtype == MOE_BF16_E4M3) && c->d % 128)
    return fail(MOE_ERR_UNSUPPORTED, "e4m3 layers need d %% 128 == 0 (d=%d)", c->d);
  if (c->dtype == MOE_BF16_E4M3 && c->inter % 128)
    return fail(MOE_ERR_UNSUPPORTED, "e4m3 down projections need inter %% 128 == 0 (inter=%d)", c->inter);
  if (c->dtype != MOE_FP32) {
    if (c->d % 64 || c->inter % 64)
      return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need d %% 64 == 0 and inter %% 64 == 0 (d=%d inter=%d)",
                  c->d, c->inter);
  } else {
    if (c->d % 4 || c->inter % 4)
      return fail(MOE_ERR_UNSUPPORTED, "fp32 layers need d %% 4 == 0 and inter %% 4 == 0 (d=%d inter=%d)",
                  c->d, c->inter);
  }
  const int64_t rows_cap = (int64_t)c->T * c->top_k + (int64_t)c->n_routed * (kPairBM - 1);
  if (rows_cap >= (int64_t(1) << 30)) return fail(MOE_ERR_UNSUPPORTED, "T * top_k too large");
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_last_error(void) { return g_last_error.c_str(); }

int32_t moe_kernels_per_forward(const moe_handle* handle) {
  // six timing slots; the permute has no kernel when the gate/up GEMM copies the rows, and
  // decode-sized layers run both GEMMs (and the row copy, after the scan has placed the
  // rows) in one kernel; e4m3 layers add the token quantisation
  return handle ? kKernelsPerForward - (handle->small ? 2 : handle->fuse_permute ? 1 : 0) +
                      (handle->e4m3 ? 1 : 0) +
                      (handle->e4m3_down ? 1 + handle->has_shared : 0)
                : 0;
}

size_t moe_device_bytes(const moe_handle* handle) { return handle ? handle->bytes : 0; }

static moe_status create_impl(const moe_cfg* cfg, moe_handle* H) {
  const moe_cfg& c = *cfg;
  MOE_CUDA(cudaGetDevice(&H->device));
  int major = 0, minor = 0;
  MOE_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, H->device));
  MOE_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, H->device));
  if (major != 10 || minor != 0)
    return fail(MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device is sm_%d%d",
                major, minor);
  MOE_CUDA(cudaDeviceGetAttribute(&H->n_sms, cudaDevAttrMultiProcessorCount, H->device));

  H->cfg = c;
  H->cfg.centroids = H->cfg.w_gate = H->cfg.w_up = H->cfg.w_down = nullptr;
  H->cfg.logit_bias = nullptr;
  H->bf16 = c.dtype != MOE_FP32;
  H->e4m3 = c.dtype == MOE_BF16_E4M3_GATEUP || c.dtype == MOE_BF16_E4M3;
  H->e4m3_down = c.dtype == MOE_BF16_E4M3;
  H->es = H->bf16 ? 2 : 4;
  H->has_shared = c.n_shared > 0 ? 1 : 0;
  H->inter_shared = c.n_shared * c.inter;
  H->G = H->has_shared + c.n_routed;
  // (the small-batch path, decided below, takes one token per router CTA)
  H->router_rows = H->bf16 ? router_tile_rows(c.T, H->n_sms) : kRouterPass;
  H->n_tiles = (c.T + H->router_rows - 1) / H->router_rows;
  H->small = H->bf16 && !H->e4m3 && c.T <= kSmallMaxTok && c.d % kSmallBM == 0;
  if (H->small) {
    H->router_rows = 1;
    H->n_tiles = c.T;
    H->router_cluster = router_small_cluster(c.T, H->n_sms);
  }
  H->n_tok = (c.T + 15) / 16 * 16;
  H->bm = H->small ? 1 : (H->bf16 ? kPairBM : kSimtBM);
  H->tile_rows = H->small ? 0 : H->bm;
  // the paired GEMM copies the routed rows itself while the shared group's tiles run
  H->fuse_permute = H->bf16 && !H->small && H->has_shared;
  H->T_pad = H->small ? H->n_tok : ((int64_t)c.T + H->bm - 1) / H->bm * H->bm;
  H->rows_cap = ((int64_t)c.T * c.top_k + (int64_t)c.n_routed * (H->bm - 1) + H->bm - 1) /
                H->bm * H->bm;
  if (H->small) H->rows_cap = ((int64_t)c.T * c.top_k + 15) / 16 * 16;
  H->n_pad = (c.n_routed + 15) / 16 * 16;
  H->maxk = combine_maxk(c.top_k);
  H->maxc = router_maxc(H->n_pad);
  const size_t es = H->es;
  const size_t d = c.d, I = c.inter, Is = H->inter_shared, nr = c.n_routed, ks = c.n_shared;

  // ---- weights
  cudaStream_t st;
  MOE_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  struct StreamGuard {
    cudaStream_t s;
    ~StreamGuard() { cudaStreamDestroy(s); }
  } guard{st};

  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->bias), (size_t)H->n_pad * 4));
  MOE_CUDA(cudaMemsetAsync(H->bias, 0, (size_t)H->n_pad * 4, st));
  if (c.logit_bias)
    MOE_CUDA(cudaMemcpyAsync(H->bias, c.logit_bias, nr * 4, cudaMemcpyDeviceToDevice, st));
  const size_t cen_rows = H->bf16 ? (size_t)H->n_pad : nr;
  MOE_TRY(dalloc(H, &H->centroids, cen_rows * d * es));
  MOE_CUDA(cudaMemsetAsync(H->centroids, 0, cen_rows * d * es, st));
  MOE_CUDA(cudaMemcpyAsync(H->centroids, c.centroids, nr * d * es, cudaMemcpyDeviceToDevice, st));

  const char* wg = static_cast<const char*>(c.w_gate);
  const char* wu = static_cast<const char*>(c.w_up);
  const char* wd = static_cast<const char*>(c.w_down);
  if (H->bf16) {
    // gate/up interleaved in blocks of 64 rows: [g0..63, u0..63, g64..127, u64..127, ...]
    const size_t blk = 64 * d * es;
    if (ks) {
      MOE_TRY(dalloc(H, &H->w_gu_s, 2 * Is * d * es));
      MOE_CUDA(cudaMemcpy2DAsync(H->w_gu_s, 2 * blk, wg, blk, blk, Is / 64, cudaMemcpyDeviceToDevice, st));
      MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_gu_s) + blk, 2 * blk, wu, blk, blk, Is / 64,
                                 cudaMemcpyDeviceToDevice, st));
    }
    MOE_TRY(dalloc(H, &H->w_gu_r, 2 * nr * I * d * es));
    MOE_CUDA(cudaMemcpy2DAsync(H->w_gu_r, 2 * blk, wg + ks * I * d * es, blk, blk, nr * I / 64,
                               cudaMemcpyDeviceToDevice, st));
    MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_gu_r) + blk, 2 * blk, wu + ks * I * d * es, blk,
                               blk, nr * I / 64, cudaMemcpyDeviceToDevice, st));
  } else {
    MOE_TRY(dalloc(H, &H->w_g, (ks + nr) * I * d * es));
    MOE_TRY(dalloc(H, &H->w_u, (ks + nr) * I * d * es));
    MOE_CUDA(cudaMemcpyAsync(H->w_g, wg, (ks + nr) * I * d * es, cudaMemcpyDeviceToDevice, st));
    MOE_CUDA(cudaMemcpyAsync(H->w_u, wu, (ks + nr) * I * d * es, cudaMemcpyDeviceToDevice, st));
  }
  // down projection: shared experts side by side along the intermediate axis [d, ks*I]
  if (ks) {
    MOE_TRY(dalloc(H, &H->w_d_s, d * Is * es));
    for (size_t j = 0; j < ks; ++j)
      MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_d_s) + j * I * es, Is * es, wd + j * d * I * es,
                                 I * es, I * es, d, cudaMemcpyDeviceToDevice, st));
  }
  MOE_TRY(dalloc(H, &H->w_d_r, nr * d * I * es));
  MOE_CUDA(cudaMemcpyAsync(H->w_d_r, wd + ks * d * I * es, nr * d * I * es, cudaMemcpyDeviceToDevice, st));
  if (H->e4m3) {
    // e4m3 copies of the interleaved gate/up rows, one fp32 scale per row
    if (ks) {
      MOE_TRY(dalloc(H, &H->w8_gu_s, 2 * Is * d));
      MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sw_s), 2 * Is * 4));
      MOE_CUDA(launch_quant(H->w_gu_s, (int64_t)(2 * Is), (int)d, H->w8_gu_s, H->sw_s, H->n_sms, st));
    }
    MOE_TRY(dalloc(H, &H->w8_gu_r, 2 * nr * I * d));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sw_r), 2 * nr * I * 4));
    MOE_CUDA(launch_quant(H->w_gu_r, (int64_t)(2 * nr * I), (int)d, H->w8_gu_r, H->sw_r, H->n_sms, st));
  }
  if (H->e4m3_down) {
    // e4m3 copies of the W_down rows (output channels), one fp32 scale per row; the shared
    // group's rows are the K_s experts' rows side by side
    if (ks) {
      MOE_TRY(dalloc(H, &H->w8_d_s, d * Is));
      MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sw_d_s), d * 4));
      MOE_CUDA(launch_quant(H->w_d_s, (int64_t)d, (int)Is, H->w8_d_s, H->sw_d_s, H->n_sms, st));
    }
    MOE_TRY(dalloc(H, &H->w8_d_r, nr * d * I));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sw_d_r), nr * d * 4));
    MOE_CUDA(launch_quant(H->w_d_r, (int64_t)(nr * d), (int)I, H->w8_d_r, H->sw_d_r, H->n_sms, st));
  }

  // ---- workspace
  const size_t T = c.T, K = c.top_k, nt = H->n_tiles;
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->topk_rank), T * K * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->slot_row), T * K * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->tile_hist), nt * nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->tile_base), nt * nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->tile_psum), nt * nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->psum_total), nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->grp_row), (size_t)H->G * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->ts1), (size_t)(H->G + 1) * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->ts2), (size_t)(H->G + 1) * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->err), 256));
  MOE_CUDA(cudaMemsetAsync(H->err, 0, 256, st));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->copy_done), kSyncBytes));
  MOE_CUDA(cudaMemsetAsync(H->copy_done, 0, kSyncBytes, st));
  const size_t rc = (size_t)H->rows_cap, tp = (size_t)H->T_pad;
  MOE_TRY(dalloc(H, &H->xp, rc * d * (H->e4m3 ? 1 : es)));   // e4m3 rows on that path
  if (H->small) MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->row_tok), rc * 4));
  if (H->e4m3) {
    MOE_TRY(dalloc(H, &H->u8, tp * d));
    MOE_CUDA(cudaMemsetAsync(H->u8, 0, tp * d, st));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->su), tp * 4));
    MOE_CUDA(cudaMemsetAsync(H->su, 0, tp * 4, st));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->su_p), rc * 4));
    MOE_CUDA(cudaMemsetAsync(H->su_p, 0, rc * 4, st));
  }
  MOE_TRY(dalloc(H, &H->hr, rc * I * es));
  MOE_TRY(dalloc(H, &H->yr, rc * d * es));
  if (H->e4m3_down) {
    MOE_TRY(dalloc(H, &H->h8r, rc * I));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sh_r), rc * 4));
    if (ks) {
      MOE_TRY(dalloc(H, &H->h8s, tp * Is));
      MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->sh_s), tp * 4));
    }
  }
  if (ks) {
    MOE_TRY(dalloc(H, &H->hs, tp * Is * es));
    MOE_TRY(dalloc(H, &H->ys, tp * d * es));
  }
  MOE_TRY(dalloc(H, &H->u_dev, T * d * es));
  MOE_TRY(dalloc(H, &H->h_dev, T * d * es));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->idx_dev), T * K * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->w_dev), T * K * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->cnt_dev), nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->aux_dev), 4));
  MOE_CUDA(cudaStreamSynchronize(st));

  // ---- kernels' launch attributes and TMA descriptors
  if (H->bf16) {
    const RouterStages rs = router_stages(H->n_pad, H->router_rows);
    if (rs.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "router stages do not fit in shared memory");
    H->router_kps = rs.kps;
    H->router_stages = rs.stages;
    H->router_smem = router_smem_bytes(H->n_pad, rs.kps, H->router_rows, rs.stages);
    H->router_tmem_cols = router_tmem_cols(H->n_pad);
    const void* rk = with_maxc(H->maxc, [](auto m) { return (const void*)router_tc_kernel<m()>; });
    MOE_CUDA(cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H->router_smem));
    MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
    MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kDown>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
    // persistent grid: as many CTA pairs as can be resident at once
    {
      cudaLaunchConfig_t lc = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      lc.gridDim = dim3(2 * (H->n_sms / 2), 1, 1);
      lc.blockDim = dim3(kGemmThreads, 1, 1);
      lc.dynamicSmemBytes = kGemmSmemBytes;
      lc.attrs = attr;
      lc.numAttrs = 1;
      int clusters = 0;
      MOE_CUDA(cudaOccupancyMaxActiveClusters(
          &clusters, (const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU>, &lc));
      if (clusters < 1) return fail(MOE_ERR_UNSUPPORTED, "no CTA pair of the GEMM kernel fits on this device");
      H->gemm_grid = 2 * clusters;
      if (H->e4m3) {
        MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
        MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kDown, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
        lc.blockDim = dim3(gemm_threads(true), 1, 1);
        MOE_CUDA(cudaOccupancyMaxActiveClusters(
            &clusters, (const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU, true>, &lc));
        if (clusters < 1) return fail(MOE_ERR_UNSUPPORTED, "no CTA pair of the e4m3 GEMM fits on this device");
        H->gemm_grid_f8 = 2 * clusters;
      }
    }

    bool ok = encode_2d(&H->tmE, H->centroids, d, (uint64_t)H->n_pad, (uint32_t)H->n_pad) &&
              (H->e4m3 || encode_2d(&H->tmXp, H->xp, d, rc, 128)) &&
              encode_3d(&H->tmWguR, H->w_gu_r, d, 2 * I, nr, kGemmBN / 2) &&
              encode_2d(&H->tmHr, H->hr, I, rc, 128) &&
              encode_3d(&H->tmWdR, H->w_d_r, I, d, nr, kGemmBN / 2);
    if (ks)
      ok = ok && encode_2d(&H->tmWguS, H->w_gu_s, d, 2 * Is, kGemmBN / 2) &&
           encode_2d(&H->tmHs, H->hs, Is, tp, 128) &&
           encode_2d(&H->tmWdS, H->w_d_s, Is, d, kGemmBN / 2);
    else {
      H->tmWguS = H->tmWguR;
      H->tmHs = H->tmHr;
      H->tmWdS = H->tmWdR;
    }
    if (H->e4m3) {
      ok = ok && encode_2d_e4m3(&H->tmU8, H->u8, d, tp, 128) &&
           encode_2d_e4m3(&H->tmXp8, H->xp, d, rc, 128) &&
           encode_3d_e4m3(&H->tmW8guR, H->w8_gu_r, d, 2 * I, nr, kGemmBN / 2);
      if (ks) ok = ok && encode_2d_e4m3(&H->tmW8guS, H->w8_gu_s, d, 2 * Is, kGemmBN / 2);
      else H->tmW8guS = H->tmW8guR;
    }
    if (H->e4m3_down) {
      ok = ok && encode_2d_e4m3(&H->tmH8r, H->h8r, I, rc, 128) &&
           encode_3d_e4m3(&H->tmW8dR, H->w8_d_r, I, d, nr, kGemmBN / 2);
      if (ks)
        ok = ok && encode_2d_e4m3(&H->tmH8s, H->h8s, Is, tp, 128) &&
             encode_2d_e4m3(&H->tmW8dS, H->w8_d_s, Is, d, kGemmBN / 2);
      else {
        H->tmH8s = H->tmH8r;
        H->tmW8dS = H->tmW8dR;
      }
    }
    if (!ok) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight/workspace tensor");
    if (H->small) {
      H->simt_router_smem = router_epi_bytes(H->n_pad);
      const void* rk = with_maxc(H->maxc, [](auto m) { return (const void*)router_small_kernel<m()>; });
      MOE_CUDA(cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)H->simt_router_smem));
      const int stages = small_stages(H->n_tok);
      H->small_stages = stages;
      H->small_smem = small_smem_bytes(H->n_tok, stages);
      MOE_CUDA(cudaFuncSetAttribute((const void*)decode_ffn_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H->small_smem));
      // the kernel's grid-wide waits need every CTA resident at once: one CTA per SM
      int per_sm = 0;
      MOE_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void*)decode_ffn_kernel,
                                                             kSmallThreads, H->small_smem));
      if (per_sm < 1) return fail(MOE_ERR_UNSUPPORTED, "the decode FFN kernel does not fit on an SM");
      bool okn = encode_2d(&H->tmXpN, H->xp, d, rc, (uint32_t)H->n_tok) &&
           encode_2d(&H->tmHrN, H->hr, I, rc, (uint32_t)H->n_tok) &&
           encode_3d(&H->tmWguR64, H->w_gu_r, d, 2 * I, nr, 64);
      if (ks)
        okn = okn && encode_2d(&H->tmHsN, H->hs, Is, tp, (uint32_t)H->n_tok) &&
              encode_2d(&H->tmWguS64, H->w_gu_s, d, 2 * Is, 64);
      else {
        H->tmHsN = H->tmHrN;
        H->tmWguS64 = H->tmWguR64;
      }
      if (!okn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a small-batch operand");
    }
  } else {
    H->simt_router_smem = router_epi_bytes(H->n_pad);
    const void* rk = with_maxc(H->maxc, [](auto m) { return (const void*)router_simt_kernel<m()>; });
    MOE_CUDA(cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)H->simt_router_smem));
  }
  return MOE_OK;
}

moe_status moe_create(const moe_cfg* cfg, moe_handle** out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  MOE_TRY(validate(cfg));
  moe_handle* H = new (std::nothrow) moe_handle();
  if (!H) return fail(MOE_ERR_OOM, "host allocation failed");
  moe_status s = create_impl(cfg, H);
  if (s != MOE_OK) {
    cudaDeviceSynchronize();
    free_handle(H);
    return s;
  }
  *out = H;
  return MOE_OK;
}

// Record timing event `slot` of the current call (no-op unless timing is on).
static inline void tick(moe_handle* H, cudaStream_t s, int slot) {
  if (H->timing_used < H->timing_cap)
    cudaEventRecord(H->events[(size_t)H->timing_used * (kKernelsPerForward + 1) + slot], s);
}

moe_status moe_forward(moe_handle* H, const void* u, void* h, int32_t* topk_idx, float* topk_w,
                       int32_t* expert_counts, float* aux_loss, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!u || !h || !topk_idx || !topk_w || !expert_counts || !aux_loss)
    return fail(MOE_ERR_INVALID_ARG, "an input/output pointer is NULL");
  if (!aligned16(u) || !aligned16(h)) return fail(MOE_ERR_INVALID_ARG, "u and h must be 16-byte aligned");
  int dev = -1;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev != H->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the handle's device %d", dev, H->device);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const int T = c.T, d = c.d, K = c.top_k, nr = c.n_routed;

  const int bn1 = H->small ? kSmallBM : (H->bf16 ? kGemmBN / 2 : kSimtBN);
  const int bn2 = H->small ? 2 * kSmallBM : (H->bf16 ? kGemmBN : kSimtBN);
  ScanArgs sa{H->tile_hist, H->tile_psum, H->n_tiles, nr, T, H->has_shared, H->inter_shared,
              c.inter, d, H->bm, H->tile_rows, bn1, bn2, c.alpha1, expert_counts, aux_loss,
              H->psum_total,
              H->tile_base, H->grp_row, H->ts1, H->ts2,
              H->fuse_permute || H->small ? H->copy_done : nullptr, H->bwd ? H->ts3 : nullptr};
  if (H->small) sa.n_sync = 1 + H->G;   // the decode FFN kernel's per-group counters too
  if (H->small) {   // the scan places the routed rows; the decode FFN kernel copies them
    sa.topk_idx = topk_idx; sa.topk_rank = H->topk_rank;
    sa.slot_row = H->slot_row; sa.row_tok = H->row_tok;
    sa.top_k = K; sa.router_rows = H->router_rows; sa.rows_cap = (int)H->rows_cap; sa.err = H->err;
  }
  RouterOut ro{topk_idx, topk_w, H->topk_rank, H->tile_hist, H->tile_psum, H->err,
               H->bwd ? H->logits : nullptr};
  CUtensorMap tmU, tmUr;
  tick(H, stream, 0);
  if (H->small) {
    RouterSmallArgs ra{static_cast<const __nv_bfloat16*>(u),
                       static_cast<const __nv_bfloat16*>(H->centroids), H->bias, T, d, nr, K,
                       H->router_rows, ro};
    with_maxc(H->maxc, [&](auto m) {
      launch_pdl_cluster(router_small_kernel<m()>, dim3(H->n_tiles * H->router_cluster), dim3(kRouterEpiThreads),
                         H->simt_router_smem, stream, (unsigned)H->router_cluster, ra);
      return 0;
    });
  } else if (H->bf16) {
    if (!encode_2d(&tmU, u, d, T, 128) || !encode_2d(&tmUr, u, d, T, (uint32_t)H->router_rows))
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for u");
    RouterTcArgs ra{T, d, nr, H->n_pad, K, H->router_kps, H->router_stages, H->router_rows, H->n_tiles,
                    H->router_tmem_cols, H->bias, ro};
    const int rgrid = H->n_tiles < H->n_sms ? H->n_tiles : H->n_sms;
    with_maxc(H->maxc, [&](auto m) {
      launch_pdl(router_tc_kernel<m()>, dim3(rgrid), dim3(kRouterThreads), H->router_smem, stream, tmUr, H->tmE, ra);
      return 0;
    });
  } else {
    RouterSimtArgs ra{static_cast<const float*>(u), static_cast<const float*>(H->centroids), H->bias,
                      T, d, nr, K, ro};
    with_maxc(H->maxc, [&](auto m) {
      launch_pdl(router_simt_kernel<m()>, dim3(H->n_tiles), dim3(kRouterEpiThreads), H->simt_router_smem, stream, ra);
      return 0;
    });
  }
  MOE_CUDA(cudaGetLastError());

  tick(H, stream, 1);
  launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, stream, sa);
  MOE_CUDA(cudaGetLastError());

  PermuteArgs pa{static_cast<const uint8_t*>(u), topk_idx, H->topk_rank, H->tile_base, H->slot_row,
                 static_cast<uint8_t*>(H->xp), T, K, nr, (int)H->rows_cap, H->router_rows,
                 d * H->es, H->err};
  tick(H, stream, 2);
  if (H->e4m3) {
    // e4m3 token rows and scales; the row copy then moves those
    MOE_CUDA(launch_quant(u, T, d, H->u8, H->su, H->n_sms, stream));
    pa.u = static_cast<const uint8_t*>(H->u8);
    pa.row_bytes = d;
    pa.scale_src = H->su;
    pa.scale_dst = H->su_p;
  }
  if (!H->fuse_permute && !H->small) {
    launch_pdl(permute_kernel, dim3((T + kPermuteWarps - 1) / kPermuteWarps), dim3(kPermuteWarps * 32), 0, stream, pa);
    MOE_CUDA(cudaGetLastError());
  }

  const int I = c.inter, Is = H->inter_shared;
  if (H->small) {
    CUtensorMap tmUN;   // token rows of the shared group, n_tok per tile
    if (!encode_2d(&tmUN, u, d, T, (uint32_t)H->n_tok))
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for u");
    SmallGemmArgs s{};
    s.grp_row = H->grp_row; s.counts = expert_counts; s.G = H->G;
    s.has_shared = H->has_shared; s.T = T; s.n_tok = H->n_tok; s.stages = H->small_stages;
    s.ph[0] = SmallPhase{H->ts1, d / 64, d / 64, Is, I, static_cast<__nv_bfloat16*>(H->hs), Is,
                         static_cast<__nv_bfloat16*>(H->hr), I};
    s.ph[1] = SmallPhase{H->ts2, Is / 64, I / 64, d, d, static_cast<__nv_bfloat16*>(H->ys), d,
                         static_cast<__nv_bfloat16*>(H->yr), d};
    s.err = H->err;
    // the routed rows (placed by the scan) are copied by the kernel's epilogue warps
    s.row_tok = H->row_tok; s.u = static_cast<const __nv_bfloat16*>(u);
    s.xp = static_cast<__nv_bfloat16*>(H->xp); s.n_rows = T * K; s.copy_vecs = d / 8;
    s.sync = H->copy_done;
    tick(H, stream, 3);
    launch_pdl(decode_ffn_kernel, dim3(H->n_sms), dim3(kSmallThreads), H->small_smem, stream, H->tmWguS64,
               H->tmWguR64, tmUN, H->tmXpN, H->tmWdS, H->tmWdR, H->tmHsN, H->tmHrN, s);
    MOE_CUDA(cudaGetLastError());
    tick(H, stream, 4);   // (the down GEMM runs inside the same kernel)
  } else if (H->bf16) {
    GemmArgs g1{};
    g1.grp_row = H->grp_row; g1.ts = H->ts1; g1.G = H->G; g1.has_shared = H->has_shared;
    g1.kb_shared = d / kGemmBK; g1.kb_routed = d / kGemmBK;
    g1.nt_shared = (Is + bn1 - 1) / bn1; g1.nt_routed = (I + bn1 - 1) / bn1;
    g1.out_shared = static_cast<__nv_bfloat16*>(H->hs); g1.ld_shared = Is; g1.rows_shared = H->T_pad;
    g1.cols_shared = Is;
    g1.out_routed = static_cast<__nv_bfloat16*>(H->hr); g1.ld_routed = I; g1.rows_routed = H->rows_cap;
    g1.cols_routed = I;
    g1.err = H->err;
    if (H->fuse_permute) {
      g1.perm = pa;
      g1.copy_done = H->copy_done;
    }
    tick(H, stream, 3);
    if (H->e4m3) {
      g1.kb_shared = d / (2 * kGemmBK);   // k-blocks of 128 e4m3 values
      g1.kb_routed = d / (2 * kGemmBK);
      g1.sa_shared = H->su;
      g1.sa_routed = H->su_p;
      g1.sb_shared = H->sw_s;
      g1.sb_routed = H->sw_r;
      g1.sb_routed_stride = 2 * (int64_t)I;
      launch_pdl(grouped_gemm_tc_kernel<kGateUpSwiGLU, true>, dim3(H->gemm_grid_f8), dim3(gemm_threads(true)),
                 kGemmSmemBytes, stream, H->tmU8, H->tmXp8, H->tmW8guS, H->tmW8guR, g1);
    } else {
      launch_pdl(grouped_gemm_tc_kernel<kGateUpSwiGLU>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,  tmU, H->tmXp, H->tmWguS, H->tmWguR, g1);
    }
    MOE_CUDA(cudaGetLastError());

    GemmArgs g2{};
    g2.grp_row = H->grp_row; g2.ts = H->ts2; g2.G = H->G; g2.has_shared = H->has_shared;
    g2.kb_shared = Is / kGemmBK; g2.kb_routed = I / kGemmBK;
    g2.nt_shared = (d + bn2 - 1) / bn2; g2.nt_routed = (d + bn2 - 1) / bn2;
    g2.out_shared = static_cast<__nv_bfloat16*>(H->ys); g2.ld_shared = d; g2.rows_shared = H->T_pad;
    g2.cols_shared = d;
    g2.out_routed = static_cast<__nv_bfloat16*>(H->yr); g2.ld_routed = d; g2.rows_routed = H->rows_cap;
    g2.cols_routed = d;
    g2.err = H->err;
    tick(H, stream, 4);
    if (H->e4m3_down) {
      // the activations' rows to e4m3 (the shared group's rows span its K_s experts), then the
      // down GEMM on e4m3 operands with the row scales applied in its epilogue
      if (H->has_shared)
        MOE_CUDA(launch_quant(H->hs, H->T_pad, Is, H->h8s, H->sh_s, H->n_sms, stream));
      MOE_CUDA(launch_quant(H->hr, H->rows_cap, I, H->h8r, H->sh_r, H->n_sms, stream));
      g2.kb_shared = Is / (2 * kGemmBK);   // k-blocks of 128 e4m3 values
      g2.kb_routed = I / (2 * kGemmBK);
      g2.sa_shared = H->sh_s;
      g2.sa_routed = H->sh_r;
      g2.sb_shared = H->sw_d_s;
      g2.sb_routed = H->sw_d_r;
      g2.sb_routed_stride = d;
      launch_pdl(grouped_gemm_tc_kernel<kDown, true>, dim3(H->gemm_grid_f8), dim3(gemm_threads(true)),
                 kGemmSmemBytes, stream, H->tmH8s, H->tmH8r, H->tmW8dS, H->tmW8dR, g2);
    } else {
      launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes,
                 stream, H->tmHs, H->tmHr, H->tmWdS, H->tmWdR, g2);
    }
    MOE_CUDA(cudaGetLastError());
  } else {
    const size_t ks = c.n_shared;
    const float* wg = static_cast<const float*>(H->w_g);
    const float* wu = static_cast<const float*>(H->w_u);
    const int grid = H->n_sms * 4;
    SimtGemmArgs s1{};
    s1.grp_row = H->grp_row; s1.ts = H->ts1; s1.G = H->G; s1.has_shared = H->has_shared;
    s1.a_shared = static_cast<const float*>(u); s1.a_rows_shared = T;
    s1.a_routed = static_cast<const float*>(H->xp); s1.a_rows_routed = H->rows_cap;
    s1.K_shared = d; s1.K_routed = d;
    s1.b0_shared = wg; s1.b1_shared = wu;
    s1.b0_routed = wg + ks * I * (size_t)d; s1.b1_routed = wu + ks * I * (size_t)d;
    s1.b_expert_stride = (int64_t)I * d;
    s1.N_shared = Is; s1.N_routed = I;
    s1.nt_shared = (Is + bn1 - 1) / bn1; s1.nt_routed = (I + bn1 - 1) / bn1;
    s1.out_shared = static_cast<float*>(H->hs); s1.out_rows_shared = H->T_pad;
    s1.out_routed = static_cast<float*>(H->hr); s1.out_rows_routed = H->rows_cap;
    s1.err = H->err;
    tick(H, stream, 3);
    launch_pdl(grouped_gemm_simt_kernel<kGateUpSwiGLU>, dim3(grid), dim3(kSimtThreads), 0, stream, s1);
    MOE_CUDA(cudaGetLastError());

    SimtGemmArgs s2{};
    s2.grp_row = H->grp_row; s2.ts = H->ts2; s2.G = H->G; s2.has_shared = H->has_shared;
    s2.a_shared = static_cast<const float*>(H->hs); s2.a_rows_shared = H->T_pad;
    s2.a_routed = static_cast<const float*>(H->hr); s2.a_rows_routed = H->rows_cap;
    s2.K_shared = Is; s2.K_routed = I;
    s2.b0_shared = static_cast<const float*>(H->w_d_s); s2.b1_shared = nullptr;
    s2.b0_routed = static_cast<const float*>(H->w_d_r); s2.b1_routed = nullptr;
    s2.b_expert_stride = (int64_t)d * I;
    s2.N_shared = d; s2.N_routed = d;
    s2.nt_shared = (d + bn2 - 1) / bn2; s2.nt_routed = (d + bn2 - 1) / bn2;
    s2.out_shared = static_cast<float*>(H->ys); s2.out_rows_shared = H->T_pad;
    s2.out_routed = static_cast<float*>(H->yr); s2.out_rows_routed = H->rows_cap;
    s2.err = H->err;
    tick(H, stream, 4);
    launch_pdl(grouped_gemm_simt_kernel<kDown>, dim3(grid), dim3(kSimtThreads), 0, stream, s2);
    MOE_CUDA(cudaGetLastError());

    const int parts = combine_parts(T, d / 4, H->n_sms);
    CombineArgs<float> ca{static_cast<const float*>(u), static_cast<const float*>(H->ys),
                          static_cast<const float*>(H->yr), H->slot_row, topk_w,
                          static_cast<float*>(h), T, d, K, parts};
    tick(H, stream, 5);
    const int cgrid = (int)(((int64_t)T * parts + kCombineWarps - 1) / kCombineWarps);
    launch_pdl(combine_f32_kernel, dim3(cgrid), dim3(kCombineWarps * 32), 0, stream, ca);
    MOE_CUDA(cudaGetLastError());
  }
  if (H->bf16) {
    const int parts = combine_parts(T, d / 8, H->n_sms);
    CombineArgs<__nv_bfloat16> ca{static_cast<const __nv_bfloat16*>(u),
                                  static_cast<const __nv_bfloat16*>(H->ys),
                                  static_cast<const __nv_bfloat16*>(H->yr), H->slot_row, topk_w,
                                  static_cast<__nv_bfloat16*>(h), T, d, K, parts};
    tick(H, stream, 5);
    const int cgrid = (int)(((int64_t)T * parts + kCombineWarps - 1) / kCombineWarps);
    with_maxk(H->maxk, [&](auto m) {
      launch_pdl(combine_bf16_kernel<m()>, dim3(cgrid), dim3(kCombineWarps * 32), 0, stream, ca);
      return 0;
    });
    MOE_CUDA(cudaGetLastError());
  }
  if (H->timing_used < H->timing_cap) {
    tick(H, stream, kKernelsPerForward);
    ++H->timing_used;
  }
  if (H->bwd) H->bwd_forward = true;
  return MOE_OK;
}


moe_status moe_backward_prepare(moe_handle* H) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (H->bwd) return MOE_OK;
  if (!H->bf16 || H->e4m3 || H->small)
    return fail(MOE_ERR_UNSUPPORTED, "the backward runs bf16 layers on the paired-GEMM path "
                                     "(not fp32, not e4m3 gate/up, not T <= 128 decode-sized)");
  int dev = -1;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev != H->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the handle's device %d", dev, H->device);
  const moe_cfg& c = H->cfg;
  const size_t d = c.d, I = c.inter, Is = H->inter_shared, nr = c.n_routed, T = c.T, K = c.top_k;
  const size_t rc = (size_t)H->rows_cap, tp = (size_t)H->T_pad, np = (size_t)H->n_pad, es = 2;
  const bool ks = H->has_shared;
  cudaStream_t st;
  MOE_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  struct StreamGuard {
    cudaStream_t s;
    ~StreamGuard() { cudaStreamDestroy(s); }
  } guard{st};
  H->kpad = (H->n_pad + 63) / 64 * 64;
  const size_t kp = (size_t)H->kpad;
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->logits), T * nr * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->ts3), (size_t)(H->G + 1) * 4));
  MOE_CUDA(cudaMemsetAsync(H->ts3, 0, (size_t)(H->G + 1) * 4, st));   // no tiles before a forward
  // transposed weights: down [d, I] -> [I, d]; interleaved gate/up [2I, d] -> [d, 2I]
  MOE_TRY(dalloc(H, &H->w_dT_r, nr * I * d * es));
  MOE_TRY(dalloc(H, &H->w_guT_r, nr * 2 * I * d * es));
  MOE_TRY(dalloc(H, &H->e_T, d * kp * es));
  void* e_pad = nullptr;   // the centroids with zero rows up to kpad, transposed below
  MOE_TRY(dalloc(H, &e_pad, kp * d * es));
  MOE_CUDA(cudaMemsetAsync(e_pad, 0, kp * d * es, st));
  MOE_CUDA(cudaMemcpyAsync(e_pad, H->centroids, np * d * es, cudaMemcpyDeviceToDevice, st));
  auto tr = [&](const void* src, void* dst, size_t R, size_t C, size_t batch) {
    transpose_bf16_kernel<<<dim3((unsigned)((C + kTrTile - 1) / kTrTile), (unsigned)((R + kTrTile - 1) / kTrTile),
                              (unsigned)batch), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                              static_cast<__nv_bfloat16*>(dst), (int)R, (int)C);
    return cudaGetLastError();
  };
  MOE_CUDA(tr(H->w_d_r, H->w_dT_r, d, I, nr));
  MOE_CUDA(tr(H->w_gu_r, H->w_guT_r, 2 * I, d, nr));
  MOE_CUDA(tr(e_pad, H->e_T, kp, d, 1));
  if (ks) {
    MOE_TRY(dalloc(H, &H->w_dT_s, Is * d * es));
    MOE_TRY(dalloc(H, &H->w_guT_s, 2 * Is * d * es));
    MOE_CUDA(tr(H->w_d_s, H->w_dT_s, d, Is, 1));
    MOE_CUDA(tr(H->w_gu_s, H->w_guT_s, 2 * Is, d, 1));
    MOE_TRY(dalloc(H, &H->dhs, tp * Is * es));
    MOE_TRY(dalloc(H, &H->dabs, tp * 2 * Is * es));
    MOE_TRY(dalloc(H, &H->dxs, tp * d * es));
  }
  MOE_TRY(dalloc(H, &H->dyr, rc * d * es));
  MOE_TRY(dalloc(H, &H->dhr, rc * I * es));
  MOE_TRY(dalloc(H, &H->dabr, rc * 2 * I * es));
  MOE_TRY(dalloc(H, &H->dxr, rc * d * es));
  MOE_TRY(dalloc(H, &H->dur, tp * d * es));
  MOE_TRY(dalloc(H, &H->dlb, tp * kp * es));
  MOE_CUDA(cudaMemsetAsync(H->dlb, 0, tp * kp * es, st));   // rows past T, columns past n_pad: 0
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->dg), T * K * 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->dl), T * np * 4));
  H->cen_chunks = (int)((T + kCenChunk - 1) / kCenChunk);
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->cen_part), (size_t)H->cen_chunks * nr * (d + 1) * 4));
  MOE_TRY(dalloc(H, &H->xpT, d * rc * es));
  MOE_TRY(dalloc(H, &H->dyrT, d * rc * es));
  MOE_TRY(dalloc(H, &H->hrT, I * rc * es));
  MOE_TRY(dalloc(H, &H->dabrT, 2 * I * rc * es));
  if (ks) {
    MOE_TRY(dalloc(H, &H->uT, d * tp * es));
    MOE_TRY(dalloc(H, &H->dhT, d * tp * es));
    MOE_TRY(dalloc(H, &H->hsT, Is * tp * es));
    MOE_TRY(dalloc(H, &H->dabsT, 2 * Is * tp * es));
  }
  {
    // static tile tables: group g of dW_gate/up has (2 I_g / 256) x (d / 256) tiles, of
    // dW_down (d / 256) x ceil(I_g / 256), I_g = K_s I for the shared group
    std::vector<int32_t> w1(H->G + 1, 0), w2(H->G + 1, 0);
    for (int g = 0; g < H->G; ++g) {
      const size_t Ig = (H->has_shared && g == 0) ? Is : I;
      w1[g + 1] = w1[g] + (int)((2 * Ig + kPairBM - 1) / kPairBM) * (int)((d + kGemmBN - 1) / kGemmBN);
      w2[g + 1] = w2[g] + (int)((d + kPairBM - 1) / kPairBM) * (int)((Ig + kGemmBN - 1) / kGemmBN);
    }
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->wts1), (size_t)(H->G + 1) * 4));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->wts2), (size_t)(H->G + 1) * 4));
    MOE_CUDA(cudaMemcpyAsync(H->wts1, w1.data(), w1.size() * 4, cudaMemcpyHostToDevice, st));
    MOE_CUDA(cudaMemcpyAsync(H->wts2, w2.data(), w2.size() * 4, cudaMemcpyHostToDevice, st));
    MOE_CUDA(cudaStreamSynchronize(st));   // the host tables above go out of scope
  }
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->r_grp), 4));
  MOE_TRY(dalloc(H, reinterpret_cast<void**>(&H->r_ts), 8));
  const int32_t grp0 = 0;
  const int32_t rts[2] = {0, (int)(tp / kPairBM) * (int)((d + kGemmBN - 1) / kGemmBN)};
  MOE_CUDA(cudaMemcpyAsync(H->r_grp, &grp0, 4, cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaMemcpyAsync(H->r_ts, rts, 8, cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  bool ok = encode_2d(&H->tmDyr, H->dyr, d, rc, 128) &&
            encode_3d(&H->tmWdTr, H->w_dT_r, d, I, nr, kGemmBN / 2) &&
            encode_2d(&H->tmDabr, H->dabr, 2 * I, rc, 128) &&
            encode_3d(&H->tmWguTr, H->w_guT_r, 2 * I, d, nr, kGemmBN / 2) &&
            encode_2d(&H->tmDlb, H->dlb, kp, tp, 128) && encode_2d(&H->tmEt, H->e_T, kp, d, kGemmBN / 2);
  if (ks)
    ok = ok && encode_2d(&H->tmWdTs, H->w_dT_s, d, Is, kGemmBN / 2) &&
         encode_2d(&H->tmDabs, H->dabs, 2 * Is, tp, 128) &&
         encode_2d(&H->tmWguTs, H->w_guT_s, 2 * Is, d, kGemmBN / 2);
  else {
    H->tmWdTs = H->tmWdTr;
    H->tmDabs = H->tmDabr;
    H->tmWguTs = H->tmWguTr;
  }
  ok = ok && encode_2d(&H->tmXpT, H->xpT, rc, d, 128) && encode_2d(&H->tmDyrT, H->dyrT, rc, d, 128) &&
       encode_2d(&H->tmHrT, H->hrT, rc, I, 128) && encode_2d(&H->tmDabrT, H->dabrT, rc, 2 * I, 128);
  if (ks)
    ok = ok && encode_2d(&H->tmUT, H->uT, tp, d, 128) && encode_2d(&H->tmDhT, H->dhT, tp, d, 128) &&
         encode_2d(&H->tmHsT, H->hsT, tp, Is, 128) && encode_2d(&H->tmDabsT, H->dabsT, tp, 2 * Is, 128);
  else {
    H->tmUT = H->tmXpT;
    H->tmDhT = H->tmDyrT;
    H->tmHsT = H->tmHrT;
    H->tmDabsT = H->tmDabrT;
  }
  if (!ok) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a backward operand");
  MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kWgrad>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
  MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kGateUpBwd>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
  H->bwd = true;
  H->bwd_forward = false;
  return MOE_OK;
}

moe_status moe_backward(moe_handle* H, const void* u, const int32_t* topk_idx, const float* topk_w,
                        const int32_t* expert_counts, const void* dh, float d_aux, void* du,
                        float* d_centroids, float* d_bias, float* d_w_gate, float* d_w_up,
                        float* d_w_down, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!H->bwd || !H->bwd_forward)
    return fail(MOE_ERR_INVALID_ARG, "call moe_backward_prepare and then moe_forward first");
  if (!u || !topk_idx || !topk_w || !expert_counts || !dh || !du || !d_centroids)
    return fail(MOE_ERR_INVALID_ARG, "an input/output pointer is NULL");
  if (!aligned16(u) || !aligned16(dh) || !aligned16(du))
    return fail(MOE_ERR_INVALID_ARG, "u, dh and du must be 16-byte aligned");
  const bool wgrad = d_w_gate || d_w_up || d_w_down;
  if (wgrad && !(d_w_gate && d_w_up && d_w_down))
    return fail(MOE_ERR_INVALID_ARG, "d_w_gate, d_w_up and d_w_down are all given or all NULL");
  if (wgrad && (!aligned16(d_w_gate) || !aligned16(d_w_up) || !aligned16(d_w_down)))
    return fail(MOE_ERR_INVALID_ARG, "the weight gradients must be 16-byte aligned");
  int dev = -1;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev != H->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the handle's device %d", dev, H->device);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const int T = c.T, d = c.d, K = c.top_k, nr = c.n_routed, I = c.inter, Is = H->inter_shared;
  // 1. dY rows of the routed experts (g dh) and the gates' gradients (dh . Y)
  BwdRowsArgs ba{static_cast<const __nv_bfloat16*>(dh), topk_w, H->slot_row,
                 static_cast<const __nv_bfloat16*>(H->yr), static_cast<__nv_bfloat16*>(H->dyr), H->dg,
                 T, d, K, H->rows_cap, H->err};
  launch_pdl(bwd_rows_kernel, dim3((T + kBwdWarps - 1) / kBwdWarps), dim3(kBwdWarps * 32), 0, stream, ba);
  MOE_CUDA(cudaGetLastError());
  CUtensorMap tmDh, tmU;
  if (!encode_2d(&tmDh, dh, d, T, 128) || !encode_2d(&tmU, u, d, T, 128))
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for u or dh");
  // 2. dHmid = dY W_down (shared group: dY = dh)
  GemmArgs g{};
  g.grp_row = H->grp_row; g.ts = H->ts3; g.G = H->G; g.has_shared = H->has_shared;
  g.kb_shared = d / kGemmBK; g.kb_routed = d / kGemmBK;
  g.nt_shared = (Is + kGemmBN - 1) / kGemmBN; g.nt_routed = (I + kGemmBN - 1) / kGemmBN;
  g.out_shared = static_cast<__nv_bfloat16*>(H->dhs); g.ld_shared = Is; g.rows_shared = H->T_pad;
  g.cols_shared = Is;
  g.out_routed = static_cast<__nv_bfloat16*>(H->dhr); g.ld_routed = I; g.rows_routed = H->rows_cap;
  g.cols_routed = I;
  g.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             tmDh, H->tmDyr, H->tmWdTs, H->tmWdTr, g);
  MOE_CUDA(cudaGetLastError());
  // 3. gate/up recomputed with the SwiGLU backward: (da, db) interleaved like W_gu's rows
  GemmArgs g1{};
  g1.grp_row = H->grp_row; g1.ts = H->ts1; g1.G = H->G; g1.has_shared = H->has_shared;
  g1.kb_shared = d / kGemmBK; g1.kb_routed = d / kGemmBK;
  g1.nt_shared = (Is + kGemmBN / 2 - 1) / (kGemmBN / 2); g1.nt_routed = (I + kGemmBN / 2 - 1) / (kGemmBN / 2);
  g1.out_shared = static_cast<__nv_bfloat16*>(H->dabs); g1.ld_shared = 2 * (int64_t)Is;
  g1.rows_shared = H->T_pad; g1.cols_shared = Is;
  g1.out_routed = static_cast<__nv_bfloat16*>(H->dabr); g1.ld_routed = 2 * (int64_t)I;
  g1.rows_routed = H->rows_cap; g1.cols_routed = I;
  g1.dh_shared = static_cast<const __nv_bfloat16*>(H->dhs); g1.ld_dh_shared = Is;
  g1.dh_routed = static_cast<const __nv_bfloat16*>(H->dhr); g1.ld_dh_routed = I;
  g1.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kGateUpBwd>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes,
             stream, tmU, H->tmXp, H->tmWguS, H->tmWguR, g1);
  MOE_CUDA(cudaGetLastError());
  // 4. dX = [da db] [W_gate; W_up]
  GemmArgs g2{};
  g2.grp_row = H->grp_row; g2.ts = H->ts2; g2.G = H->G; g2.has_shared = H->has_shared;
  g2.kb_shared = 2 * Is / kGemmBK; g2.kb_routed = 2 * I / kGemmBK;
  g2.nt_shared = g2.nt_routed = (d + kGemmBN - 1) / kGemmBN;
  g2.out_shared = static_cast<__nv_bfloat16*>(H->dxs); g2.ld_shared = d; g2.rows_shared = H->T_pad;
  g2.cols_shared = d;
  g2.out_routed = static_cast<__nv_bfloat16*>(H->dxr); g2.ld_routed = d; g2.rows_routed = H->rows_cap;
  g2.cols_routed = d;
  g2.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             H->tmDabs, H->tmDabr, H->tmWguTs, H->tmWguTr, g2);
  MOE_CUDA(cudaGetLastError());
  // 5. router: dl = s (ds - sum s ds), then dl e (one-group GEMM, K = n_pad)
  BwdRouterArgs ra{H->logits, topk_idx, H->dg, expert_counts, T, nr, K, H->n_pad, H->kpad,
                   (float)((double)d_aux * (double)c.alpha1 / ((double)T * (double)T)), H->dl,
                   static_cast<__nv_bfloat16*>(H->dlb)};
  with_maxc(H->maxc, [&](auto m) {
    launch_pdl(bwd_router_kernel<m()>, dim3((T + kBwdWarps - 1) / kBwdWarps), dim3(kBwdWarps * 32), 0, stream, ra);
    return 0;
  });
  MOE_CUDA(cudaGetLastError());
  GemmArgs g3{};
  g3.grp_row = H->r_grp; g3.ts = H->r_ts; g3.G = 1; g3.has_shared = 1;
  g3.kb_shared = g3.kb_routed = H->kpad / kGemmBK;
  g3.nt_shared = g3.nt_routed = (d + kGemmBN - 1) / kGemmBN;
  g3.out_shared = g3.out_routed = static_cast<__nv_bfloat16*>(H->dur);
  g3.ld_shared = g3.ld_routed = d;
  g3.rows_shared = g3.rows_routed = H->T_pad;
  g3.cols_shared = g3.cols_routed = d;
  g3.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             H->tmDlb, H->tmDlb, H->tmEt, H->tmEt, g3);
  MOE_CUDA(cudaGetLastError());
  // 6. du = dh + dX_shared + sum_k dX_k + dl e (fixed order, one rounding)
  const int parts = combine_parts(T, d / 8, H->n_sms);
  CombineArgs<__nv_bfloat16> ca{static_cast<const __nv_bfloat16*>(dh),
                                H->has_shared ? static_cast<const __nv_bfloat16*>(H->dxs) : nullptr,
                                static_cast<const __nv_bfloat16*>(H->dxr), H->slot_row, nullptr,
                                static_cast<__nv_bfloat16*>(du), T, d, K, parts,
                                static_cast<const __nv_bfloat16*>(H->dur)};
  const int cgrid = (int)(((int64_t)T * parts + kCombineWarps - 1) / kCombineWarps);
  with_maxk(H->maxk, [&](auto m) {
    launch_pdl(combine_bf16_kernel<m()>, dim3(cgrid), dim3(kCombineWarps * 32), 0, stream, ca);
    return 0;
  });
  MOE_CUDA(cudaGetLastError());
  // 7. centroid and bias gradients: chunk partials, then their fixed-order sum
  BwdCentroidArgs cp{H->dl, static_cast<const __nv_bfloat16*>(u), T, d, nr, H->n_pad, H->cen_chunks,
                     H->cen_part};
  {
    const dim3 cg((d + kCenCols - 1) / kCenCols, H->cen_chunks);
    switch (centroid_maxper(nr)) {
      case 1: launch_pdl(bwd_centroid_partial_kernel<1>, cg, dim3(256), 0, stream, cp); break;
      case 2: launch_pdl(bwd_centroid_partial_kernel<2>, cg, dim3(256), 0, stream, cp); break;
      case 4: launch_pdl(bwd_centroid_partial_kernel<4>, cg, dim3(256), 0, stream, cp); break;
      case 8: launch_pdl(bwd_centroid_partial_kernel<8>, cg, dim3(256), 0, stream, cp); break;
      default: launch_pdl(bwd_centroid_partial_kernel<16>, cg, dim3(256), 0, stream, cp); break;
    }
  }
  MOE_CUDA(cudaGetLastError());
  const int rgrid = (int)(((size_t)nr * (d + 1) + 255) / 256);
  launch_pdl(bwd_centroid_reduce_kernel, dim3(rgrid < 4 * H->n_sms ? rgrid : 4 * H->n_sms), dim3(256), 0,
             stream, (const float*)H->cen_part, H->cen_chunks, nr, d, d_centroids, d_bias);
  MOE_CUDA(cudaGetLastError());
  if (!wgrad) return MOE_OK;
  // 8. weight gradients: transposed activations (padding rows zero), then per group
  //    dW_gate/up = [da db]^T X (rows interleaved like W_gu, split on the way out) and
  //    dW_down = dY^T Hmid, K = the group's rows
  const int64_t rc = H->rows_cap, tp = H->T_pad;
  auto mtr = [&](const void* src, void* dst, int64_t rows, int C, int64_t ld_src, int64_t ld_dst,
                 bool routed) {
    MaskedTransposeArgs ma{static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), rows, C,
                           ld_src, ld_dst, routed ? H->grp_row + H->has_shared : nullptr, expert_counts,
                           nr, 0, T, routed ? rows : (int64_t)T};
    launch_pdl(masked_transpose_kernel, dim3((unsigned)((C + kMtTile * kMtColTiles - 1) / (kMtTile * kMtColTiles)),
                                             (unsigned)((rows + kMtTile - 1) / kMtTile)),
               dim3(256), 0, stream, ma);
    return cudaGetLastError();
  };
  MOE_CUDA(mtr(H->xp, H->xpT, rc, d, d, rc, true));
  MOE_CUDA(mtr(H->dyr, H->dyrT, rc, d, d, rc, true));
  MOE_CUDA(mtr(H->hr, H->hrT, rc, I, I, rc, true));
  MOE_CUDA(mtr(H->dabr, H->dabrT, rc, 2 * I, 2 * I, rc, true));
  if (H->has_shared) {
    MOE_CUDA(mtr(u, H->uT, tp, d, d, tp, false));
    MOE_CUDA(mtr(dh, H->dhT, tp, d, d, tp, false));
    MOE_CUDA(mtr(H->hs, H->hsT, tp, Is, Is, tp, false));
    MOE_CUDA(mtr(H->dabs, H->dabsT, tp, 2 * Is, 2 * Is, tp, false));
  }
  const size_t ks = c.n_shared;
  GemmArgs w1{};
  w1.grp_row = H->grp_row; w1.ts = H->wts1; w1.G = H->G; w1.has_shared = H->has_shared;
  w1.kb_shared = (int)(tp / kGemmBK); w1.kb_routed = 0;
  w1.nt_shared = w1.nt_routed = (d + kGemmBN - 1) / kGemmBN;
  w1.rows_shared = 2 * (int64_t)Is; w1.rows_routed = 2 * (int64_t)I;
  w1.cols_shared = w1.cols_routed = d;
  w1.err = H->err;
  w1.wg_counts = expert_counts; w1.wg_bm = H->bm; w1.wg_split = 1;
  w1.wg_out0_shared = d_w_gate; w1.wg_out1_shared = d_w_up;
  w1.wg_out0_routed = d_w_gate + ks * (size_t)I * d; w1.wg_out1_routed = d_w_up + ks * (size_t)I * d;
  w1.wg_stride = (int64_t)I * d;
  // 32-byte stores when the caller's gradient buffers allow them (16-byte alignment is
  // all the interface requires)
  const bool al32 = ((reinterpret_cast<uintptr_t>(d_w_gate) | reinterpret_cast<uintptr_t>(d_w_up) |
                      reinterpret_cast<uintptr_t>(d_w_down)) & 31u) == 0;
  w1.wg_v8 = al32;
  launch_pdl(grouped_gemm_tc_kernel<kWgrad>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             H->tmDabsT, H->tmDabrT, H->tmUT, H->tmXpT, w1);
  MOE_CUDA(cudaGetLastError());
  GemmArgs w2{};
  w2.grp_row = H->grp_row; w2.ts = H->wts2; w2.G = H->G; w2.has_shared = H->has_shared;
  w2.kb_shared = (int)(tp / kGemmBK); w2.kb_routed = 0;
  w2.nt_shared = (Is + kGemmBN - 1) / kGemmBN; w2.nt_routed = (I + kGemmBN - 1) / kGemmBN;
  w2.rows_shared = w2.rows_routed = d;
  w2.cols_shared = Is; w2.cols_routed = I;
  w2.err = H->err;
  w2.wg_counts = expert_counts; w2.wg_bm = H->bm; w2.wg_split = 0;
  w2.wg_out0_shared = d_w_down; w2.wg_out0_routed = d_w_down + ks * (size_t)d * I;
  w2.wg_stride = (int64_t)d * I;
  w2.wg_v8 = al32;
  w2.wg_colsplit = I;   // the shared group's K_s experts sit side by side along I
  launch_pdl(grouped_gemm_tc_kernel<kWgrad>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             H->tmDhT, H->tmDyrT, H->tmHsT, H->tmHrT, w2);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status moe_timing_begin(moe_handle* H, int32_t max_forwards) {
  if (!H || max_forwards < 1) return fail(MOE_ERR_INVALID_ARG, "handle is NULL or max_forwards < 1");
  const size_t need = (size_t)max_forwards * (kKernelsPerForward + 1);
  while (H->events.size() < need) {
    cudaEvent_t e;
    MOE_CUDA(cudaEventCreate(&e));
    H->events.push_back(e);
  }
  H->timing_cap = max_forwards;
  H->timing_used = 0;
  return MOE_OK;
}

moe_status moe_timing_end(moe_handle* H, double* kernel_ms, int32_t* n_forwards) {
  if (!H || !kernel_ms || !n_forwards) return fail(MOE_ERR_INVALID_ARG, "a pointer is NULL");
  for (int k = 0; k < kKernelsPerForward; ++k) kernel_ms[k] = 0.0;
  const int n = H->timing_used;
  H->timing_cap = 0;
  H->timing_used = 0;
  for (int f = 0; f < n; ++f) {
    const cudaEvent_t* ev = &H->events[(size_t)f * (kKernelsPerForward + 1)];
    MOE_CUDA(cudaEventSynchronize(ev[kKernelsPerForward]));
    for (int k = 0; k < kKernelsPerForward; ++k) {
      float ms = 0.f;
      MOE_CUDA(cudaEventElapsedTime(&ms, ev[k], ev[k + 1]));
      kernel_ms[k] += ms;
    }
  }
  *n_forwards = n;
  return MOE_OK;
}

moe_status moe_forward_host(moe_handle* H, const void* u_host, void* h_host, int32_t* topk_idx_host,
                            float* topk_w_host, int32_t* expert_counts_host, float* aux_loss_host,
                            moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!u_host || !h_host) return fail(MOE_ERR_INVALID_ARG, "u_host and h_host must not be NULL");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const size_t row = (size_t)c.T * c.d * H->es, tk = (size_t)c.T * c.top_k;
  MOE_CUDA(cudaMemcpyAsync(H->u_dev, u_host, row, cudaMemcpyHostToDevice, stream));
  MOE_TRY(moe_forward(H, H->u_dev, H->h_dev, H->idx_dev, H->w_dev, H->cnt_dev, H->aux_dev, stream_));
  MOE_CUDA(cudaMemcpyAsync(h_host, H->h_dev, row, cudaMemcpyDeviceToHost, stream));
  if (topk_idx_host)
    MOE_CUDA(cudaMemcpyAsync(topk_idx_host, H->idx_dev, tk * 4, cudaMemcpyDeviceToHost, stream));
  if (topk_w_host)
    MOE_CUDA(cudaMemcpyAsync(topk_w_host, H->w_dev, tk * 4, cudaMemcpyDeviceToHost, stream));
  if (expert_counts_host)
    MOE_CUDA(cudaMemcpyAsync(expert_counts_host, H->cnt_dev, (size_t)c.n_routed * 4,
                             cudaMemcpyDeviceToHost, stream));
  if (aux_loss_host)
    MOE_CUDA(cudaMemcpyAsync(aux_loss_host, H->aux_dev, 4, cudaMemcpyDeviceToHost, stream));
  MOE_CUDA(cudaStreamSynchronize(stream));
  return MOE_OK;
}

namespace {
moe_status pipe_init(moe_handle* H) {
  const moe_cfg& c = H->cfg;
  const size_t row = (size_t)c.T * c.d * H->es, tk = (size_t)c.T * c.top_k;
  for (cudaStream_t* st : {&H->p_in, &H->p_c, &H->p_out})
    MOE_CUDA(cudaStreamCreateWithFlags(st, cudaStreamNonBlocking));
  MOE_CUDA(cudaEventCreateWithFlags(&H->p_entry, cudaEventDisableTiming));
  for (auto& P : H->pslot) {
    MOE_TRY(dalloc(H, &P.u, row));
    MOE_TRY(dalloc(H, &P.h, row));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&P.idx), tk * 4));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&P.w), tk * 4));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&P.cnt), (size_t)c.n_routed * 4));
    MOE_TRY(dalloc(H, reinterpret_cast<void**>(&P.aux), 4));
    for (cudaEvent_t* e : {&P.in_done, &P.comp_done, &P.out_done})
      MOE_CUDA(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
  }
  H->p_ready = true;
  return MOE_OK;
}
}  // namespace

moe_status moe_forward_host_pipelined(moe_handle* H, const void* u_host, void* h_host,
                                      int32_t* topk_idx_host, float* topk_w_host,
                                      int32_t* expert_counts_host, float* aux_loss_host,
                                      moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!u_host || !h_host) return fail(MOE_ERR_INVALID_ARG, "u_host and h_host must not be NULL");
  int dev = -1;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev != H->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the handle's device %d", dev, H->device);
  if (!H->p_ready) MOE_TRY(pipe_init(H));
  cudaStream_t us = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const size_t row = (size_t)c.T * c.d * H->es, tk = (size_t)c.T * c.top_k;
  moe_handle::PipeSlot& P = H->pslot[H->p_calls & 1];
  // copy-in: after the caller's earlier work and after the forward that last read the slot
  MOE_CUDA(cudaEventRecord(H->p_entry, us));
  MOE_CUDA(cudaStreamWaitEvent(H->p_in, H->p_entry, 0));
  if (P.used) MOE_CUDA(cudaStreamWaitEvent(H->p_in, P.comp_done, 0));
  MOE_CUDA(cudaMemcpyAsync(P.u, u_host, row, cudaMemcpyHostToDevice, H->p_in));
  MOE_CUDA(cudaEventRecord(P.in_done, H->p_in));
  // forward: after its input and after the copy-out that last read the slot's outputs
  MOE_CUDA(cudaStreamWaitEvent(H->p_c, P.in_done, 0));
  if (P.used) MOE_CUDA(cudaStreamWaitEvent(H->p_c, P.out_done, 0));
  MOE_TRY(moe_forward(H, P.u, P.h, P.idx, P.w, P.cnt, P.aux,
                      reinterpret_cast<moe_stream_t>(H->p_c)));
  MOE_CUDA(cudaEventRecord(P.comp_done, H->p_c));
  // copy-out
  MOE_CUDA(cudaStreamWaitEvent(H->p_out, P.comp_done, 0));
  MOE_CUDA(cudaMemcpyAsync(h_host, P.h, row, cudaMemcpyDeviceToHost, H->p_out));
  if (topk_idx_host)
    MOE_CUDA(cudaMemcpyAsync(topk_idx_host, P.idx, tk * 4, cudaMemcpyDeviceToHost, H->p_out));
  if (topk_w_host)
    MOE_CUDA(cudaMemcpyAsync(topk_w_host, P.w, tk * 4, cudaMemcpyDeviceToHost, H->p_out));
  if (expert_counts_host)
    MOE_CUDA(cudaMemcpyAsync(expert_counts_host, P.cnt, (size_t)c.n_routed * 4,
                             cudaMemcpyDeviceToHost, H->p_out));
  if (aux_loss_host)
    MOE_CUDA(cudaMemcpyAsync(aux_loss_host, P.aux, 4, cudaMemcpyDeviceToHost, H->p_out));
  MOE_CUDA(cudaEventRecord(P.out_done, H->p_out));
  P.used = true;
  ++H->p_calls;
  return MOE_OK;
}

moe_status moe_pipeline_wait(moe_handle* H, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (H->p_calls == 0) return MOE_OK;
  // copy-outs run in issue order on one stream: the last one covers all earlier ones
  const moe_handle::PipeSlot& P = H->pslot[(H->p_calls - 1) & 1];
  MOE_CUDA(cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(stream_), P.out_done, 0));
  return MOE_OK;
}

moe_status moe_device_status(moe_handle* H, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  MOE_CUDA(cudaStreamSynchronize(stream));
  int code = 0;
  MOE_CUDA(cudaMemcpy(&code, H->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code != 0) {
    MOE_CUDA(cudaMemset(H->err, 0, sizeof(int)));
    return fail(MOE_ERR_DEVICE_CHECK, "a kernel recorded device error 0x%x", code);
  }
  return MOE_OK;
}

moe_status moe_expert_psum(moe_handle* H, float* psum, moe_stream_t stream_) {
  if (!H || !psum) return fail(MOE_ERR_INVALID_ARG, "handle or psum is NULL");
  MOE_CUDA(cudaMemcpyAsync(psum, H->psum_total, (size_t)H->cfg.n_routed * 4, cudaMemcpyDeviceToDevice,
                           reinterpret_cast<cudaStream_t>(stream_)));
  return MOE_OK;
}

moe_status moe_balance_loss(const int32_t* counts, const float* psum, int32_t n_routed,
                            int64_t n_tokens, float alpha1, float* aux_loss, moe_stream_t stream_) {
  if (!counts || !psum || !aux_loss) return fail(MOE_ERR_INVALID_ARG, "a pointer is NULL");
  if (n_routed < 1 || n_tokens < 1) return fail(MOE_ERR_INVALID_ARG, "n_routed and n_tokens must be positive");
  launch_pdl(balance_loss_kernel, dim3(1), dim3(32), 0, reinterpret_cast<cudaStream_t>(stream_),  counts, psum, n_routed, 1.0 / (double)n_tokens, alpha1, aux_loss);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status moe_debug_copy(const moe_handle* H, int32_t which, void* dst, size_t bytes,
                          size_t* size, moe_stream_t stream_) {
  if (!H || !size) return fail(MOE_ERR_INVALID_ARG, "handle and size must not be NULL");
  const moe_cfg& c = H->cfg;
  const size_t rc = (size_t)H->rows_cap, tp = (size_t)H->T_pad, d = c.d, I = c.inter;
  const size_t es = H->es, xes = H->e4m3 ? 1 : es;
  const void* src = nullptr;
  size_t n = 0;
  switch (which) {
    case 0: src = H->slot_row; n = (size_t)c.T * c.top_k * 4; break;
    case 1: src = H->xp; n = rc * d * xes; break;
    case 2: src = H->hr; n = rc * I * es; break;
    case 3: src = H->yr; n = rc * d * es; break;
    case 4: src = H->hs; n = H->hs ? tp * (size_t)H->inter_shared * es : 0; break;
    case 5: src = H->ys; n = H->ys ? tp * d * es : 0; break;
    case 6: src = H->grp_row; n = (size_t)H->G * 4; break;
    case 7: src = H->row_tok; n = H->row_tok ? rc * 4 : 0; break;
    default: return fail(MOE_ERR_INVALID_ARG, "which=%d outside [0, 7]", which);
  }
  *size = n;
  if (!dst) return MOE_OK;
  if (bytes > n) return fail(MOE_ERR_INVALID_ARG, "bytes=%zu above the buffer's %zu", bytes, n);
  if (bytes)
    MOE_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice,
                             reinterpret_cast<cudaStream_t>(stream_)));
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(int32_t kind, int64_t limit_ns, int32_t* device_code) {
  if (!device_code) return fail(MOE_ERR_INVALID_ARG, "device_code is NULL");
  if (kind != 0 && kind != 1) return fail(MOE_ERR_INVALID_ARG, "kind must be 0 or 1");
  if (limit_ns < 1000000 || limit_ns > 2000000000)
    return fail(MOE_ERR_INVALID_ARG, "limit_ns outside [1e6, 2e9]");
  int* err = nullptr;
  MOE_CUDA(cudaMalloc(&err, sizeof(int)));
  cudaError_t e = cudaMemset(err, 0, sizeof(int));
  if (e == cudaSuccess) {
    wait_selftest_kernel<<<1, 32>>>(kind, (uint64_t)limit_ns, err);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int code = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&code, err, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(err);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "self-test kernel: %s", cudaGetErrorString(e));
  *device_code = code;
  return MOE_OK;
}

void moe_destroy(moe_handle* H) {
  if (!H) return;
  cudaDeviceSynchronize();
  free_handle(H);
}

}  // extern "C"
