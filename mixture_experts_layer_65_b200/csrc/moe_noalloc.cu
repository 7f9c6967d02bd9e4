// moe_noalloc.cu -- moe_route_noalloc: the router step (routing, gates, expert counts,
// balance loss) for callers that cannot allocate device memory.
//
// It launches the same bf16 tcgen05 router kernel and scan kernel as moe_forward; the
// per-tile histograms, ranks and affinity sums and the scan's tables live in one fixed
// file-scope device array instead of a handle's workspace.  The array exists once per
// GPU that loads this library and stays there until the process exits.
#include <mutex>

#include "moe.h"
#include "router.cuh"

using namespace moe;

namespace {

// router tiles the scratch holds (moe_forward's tiling needs at most one per SM per round of
// 128-token tiles: 148 at T = 16384 on a B200)
constexpr int kNoAllocTiles = 320;
// byte offsets inside the scratch array
constexpr size_t kOffRank = 0;                                                      // [T, top_k] i32
constexpr size_t kOffHist = kOffRank + (size_t)MOE_NOALLOC_MAX_TOKENS * kMaxTopK * 4;  // [tiles, N_r] i32
constexpr size_t kOffPsum = kOffHist + (size_t)kNoAllocTiles * kMaxRouted * 4;         // [tiles, N_r] f32
constexpr size_t kOffBase = kOffPsum + (size_t)kNoAllocTiles * kMaxRouted * 4;         // [tiles, N_r] i32
constexpr size_t kOffPsumTot = kOffBase + (size_t)kNoAllocTiles * kMaxRouted * 4;      // [N_r] f32
constexpr size_t kOffGrp = kOffPsumTot + kMaxRouted * 4;                               // [N_r] i32
constexpr size_t kOffTs1 = kOffGrp + (kMaxRouted + 64) * 4;                             // [N_r + 1] i32
constexpr size_t kOffTs2 = kOffTs1 + (kMaxRouted + 64) * 4;                             // [N_r + 1] i32
constexpr size_t kOffErr = kOffTs2 + (kMaxRouted + 64) * 4;                             // error word
constexpr size_t kOffZeroBias = kOffErr + 256;                                         // [N_r] f32 zeros
constexpr size_t kScratchBytes = kOffZeroBias + kMaxRouted * 4;
static_assert(kScratchBytes <= MOE_NOALLOC_SCRATCH_BYTES, "scratch layout exceeds the stated size");

}  // namespace

// The scratch itself.  In host code this name is only a host-side stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace moe {
void set_last_error(const char* msg);   // moe_api.cu: the text moe_last_error() returns
}

namespace {

moe_status nfail(moe_status st, const char* msg) {
  moe::set_last_error(msg);
  return st;
}

struct DeviceSetup {
  std::once_flag once;
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  cudaError_t status = cudaSuccess;
  int sm_major = 0, sm_minor = 0, n_sms = 0;
};
DeviceSetup g_setup[64];

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                             CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                             CUtensorMapFloatOOBfill);

bool encode_rows(CUtensorMap* m, const void* ptr, uint64_t d, uint64_t rows, uint32_t box_rows) {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  cuuint64_t dims[2] = {d, rows};
  cuuint64_t strides[1] = {d * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MAXC>
cudaError_t launch_router(const CUtensorMap& tmU, const CUtensorMap& tmE, const RouterTcArgs& ra,
                          int grid, size_t smem, cudaStream_t st) {
  launch_pdl(router_tc_kernel<MAXC>, dim3(grid), dim3(kRouterThreads), smem, st, tmU, tmE, ra);
  return cudaGetLastError();
}

// The router instantiations may use up to the opt-in shared-memory budget: set once per
// device, in the one-time set-up.
cudaError_t set_router_smem_limits() {
  const void* k[] = {(const void*)router_tc_kernel<2>, (const void*)router_tc_kernel<4>,
                     (const void*)router_tc_kernel<8>, (const void*)router_tc_kernel<16>,
                     (const void*)router_tc_kernel<32>};
  for (const void* f : k) {
    const cudaError_t e =
        cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRouterSmemBudget);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* u, const void* centroids, const float* logit_bias,
                                        int32_t T, int32_t d, int32_t n_routed, int32_t top_k,
                                        float alpha1, int32_t* topk_idx, float* topk_w,
                                        int32_t* expert_counts, float* aux_loss,
                                        int32_t* device_error, moe_stream_t stream_) {
  if (!u || !centroids || !topk_idx || !topk_w || !expert_counts || !aux_loss)
    return nfail(MOE_ERR_INVALID_ARG, "moe_route_noalloc: a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(centroids)) & 15u)
    return nfail(MOE_ERR_INVALID_ARG, "moe_route_noalloc: u and centroids must be 16-byte aligned");
  if (T < 1 || T > MOE_NOALLOC_MAX_TOKENS)
    return nfail(MOE_ERR_UNSUPPORTED,
                 "moe_route_noalloc: T must be in [1, MOE_NOALLOC_MAX_TOKENS = 16384]");
  if (n_routed < 1 || n_routed > MOE_NOALLOC_MAX_ROUTED)
    return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: n_routed must be in [1, 256]");
  if (top_k < 1 || top_k > n_routed || top_k > MOE_NOALLOC_MAX_TOP_K)
    return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: top_k must be in [1, min(16, n_routed)]");
  if (d < 64 || d % 64)
    return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: d must be a positive multiple of 64");

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return nfail(MOE_ERR_CUDA, "moe_route_noalloc: cudaGetDevice failed");
  DeviceSetup& S = g_setup[dev];
  // once per device, with that device current: find the scratch array's device address
  std::call_once(S.once, [&S, dev] {
    S.status = cudaDeviceGetAttribute(&S.sm_major, cudaDevAttrComputeCapabilityMajor, dev);
    if (S.status == cudaSuccess)
      S.status = cudaDeviceGetAttribute(&S.sm_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (S.status == cudaSuccess)
      S.status = cudaDeviceGetAttribute(&S.n_sms, cudaDevAttrMultiProcessorCount, dev);
    if (S.status == cudaSuccess)
      S.status = cudaGetSymbolAddress(reinterpret_cast<void**>(&S.scratch), g_noalloc_scratch);
    if (S.status == cudaSuccess && S.sm_major == 10 && S.sm_minor == 0)
      S.status = set_router_smem_limits();
  });
  if (S.status != cudaSuccess || !S.scratch)
    return nfail(MOE_ERR_CUDA, "moe_route_noalloc: one-time set-up (scratch address, kernel attributes) failed");
  if (S.sm_major != 10 || S.sm_minor != 0)
    return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: needs an sm_100a (B200) device");

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
  unsigned char* sc = S.scratch;
  int32_t* err = reinterpret_cast<int32_t*>(sc + kOffErr);
  float* zero_bias = reinterpret_cast<float*>(sc + kOffZeroBias);
  // the array keeps the previous call's contents: clear what must start at zero
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), st) != cudaSuccess ||
      (!logit_bias && cudaMemsetAsync(zero_bias, 0, (size_t)n_routed * 4, st) != cudaSuccess))
    return nfail(MOE_ERR_CUDA, "moe_route_noalloc: cudaMemsetAsync on the scratch failed");

  const int n_pad = (n_routed + 15) / 16 * 16;
  // moe_forward's tiling: one tile of <= 128 tokens per SM and round, so the tile count is at
  // most max(SMs, T / 128 + SMs), far below the scratch's capacity on a 148-SM part
  const int rows = router_tile_rows(T, S.n_sms);
  const int n_tiles = (T + rows - 1) / rows;
  if (n_tiles > kNoAllocTiles)
    return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: more router tiles than the scratch holds");
  CUtensorMap tmU, tmE;
  if (!encode_rows(&tmU, u, d, T, (uint32_t)rows) || !encode_rows(&tmE, centroids, d, n_routed, n_pad))
    return nfail(MOE_ERR_CUDA, "moe_route_noalloc: cuTensorMapEncodeTiled failed");
  const RouterStages rs = router_stages(n_pad, rows);
  if (rs.stages < 2) return nfail(MOE_ERR_UNSUPPORTED, "moe_route_noalloc: router stages do not fit");
  const size_t smem = router_smem_bytes(n_pad, rs.kps, rows, rs.stages);
  const uint32_t cols = router_tmem_cols(n_pad);

  ScanArgs sa{reinterpret_cast<int32_t*>(sc + kOffHist), reinterpret_cast<float*>(sc + kOffPsum),
              n_tiles, n_routed, T, /*has_shared=*/0,
              /*inter_shared=*/0, /*inter=*/64, d, /*bm=*/128, /*tile_rows=*/128, /*bn1=*/128,
              /*bn2=*/256, alpha1,
              expert_counts,
              aux_loss, reinterpret_cast<float*>(sc + kOffPsumTot),
              reinterpret_cast<int32_t*>(sc + kOffBase), reinterpret_cast<int32_t*>(sc + kOffGrp),
              reinterpret_cast<int32_t*>(sc + kOffTs1), reinterpret_cast<int32_t*>(sc + kOffTs2),
              /*copy_done=*/nullptr};
  RouterOut ro{topk_idx, topk_w, reinterpret_cast<int32_t*>(sc + kOffRank),
               reinterpret_cast<int32_t*>(sc + kOffHist), reinterpret_cast<float*>(sc + kOffPsum), err};
  RouterTcArgs ra{T, d, n_routed, n_pad, top_k, rs.kps, rs.stages, rows, n_tiles, cols,
                  logit_bias ? logit_bias : zero_bias, ro};
  const int grid = n_tiles < S.n_sms ? n_tiles : S.n_sms;
  const int mc = router_maxc(n_pad);
  cudaError_t e = mc == 2 ? launch_router<2>(tmU, tmE, ra, grid, smem, st)
                 : mc == 4 ? launch_router<4>(tmU, tmE, ra, grid, smem, st)
                 : mc == 8 ? launch_router<8>(tmU, tmE, ra, grid, smem, st)
                 : mc == 16 ? launch_router<16>(tmU, tmE, ra, grid, smem, st)
                            : launch_router<32>(tmU, tmE, ra, grid, smem, st);
  if (e != cudaSuccess) return nfail(MOE_ERR_CUDA, "moe_route_noalloc: router launch failed");
  launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, st, sa);
  if (cudaGetLastError() != cudaSuccess) return nfail(MOE_ERR_CUDA, "moe_route_noalloc: scan launch failed");
  if (device_error &&
      cudaMemcpyAsync(device_error, err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return nfail(MOE_ERR_CUDA, "moe_route_noalloc: copying the device error word failed");
  return MOE_OK;
}
