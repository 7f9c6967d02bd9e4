// moe_ep.cu -- the expert-parallel layer of the C-ABI (include/moe.h, moe_ep_*).
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Where this sits": the experts of a layer are
// spread over devices (the device-level balance loss keeps their computation even).  Each
// rank holds all shared experts and a contiguous range of the routed experts, and routes its
// own tokens; between the calls below the caller moves the routed rows with two all-to-alls
// (NCCL).  The arithmetic is the layer's: the same router, grouped GEMMs and combine
// kernels as moe_forward, so a token's output does not depend on how the experts are split.
//
//   moe_ep_dispatch  router and scan (unpadded expert offsets), then the row copy: every (token, slot) row in expert order = destination-rank
//                    order, which is what the caller's all-to-all sends
//   moe_ep_experts   layout scan of the received blocks, rows into padded expert groups,
//                    gate/up + SwiGLU and down GEMMs of the local experts, rows back into the
//                    received order
//   moe_ep_combine   the shared experts on this rank's tokens, then the combine with the
//                    returned rows
#include <cstring>
#include <vector>

#include "api_common.cuh"
#include "combine.cuh"
#include "ep.cuh"
#include "gemm_small.cuh"
#include "gemm_tc.cuh"
#include "router.cuh"
#include "scan_permute.cuh"

using namespace moe;

struct moe_ep_handle {
  moe_cfg cfg;
  int rank = 0, world = 1, e0 = 0, n_local = 0;
  int device = 0, n_sms = 0;
  int64_t recv_cap = 0, rows_cap = 0, T_pad = 0;
  int n_pad = 0, maxc = 32, maxk = 16, has_shared = 0, inter_shared = 0;
  bool small_router = false;
  int router_rows = 0, n_tiles = 0, router_stages = 0, router_kps = 1, gemm_grid = 0;
  int router_cluster = 1;   // CTAs per token of the decode-sized router
  uint32_t router_tmem_cols = 0;
  size_t router_smem = 0, simt_router_smem = 0;
  // weights: all centroids (padded), this rank's routed experts and the shared group
  void* centroids = nullptr;
  float* bias = nullptr;
  void *w_gu_s = nullptr, *w_gu_r = nullptr, *w_d_s = nullptr, *w_d_r = nullptr;
  // dispatch
  int32_t *topk_rank = nullptr, *slot_row = nullptr, *tile_hist = nullptr, *tile_base = nullptr;
  int32_t *disp_grp = nullptr, *disp_ts1 = nullptr, *disp_ts2 = nullptr;
  int* err = nullptr;
  float *tile_psum = nullptr, *psum_total = nullptr;
  // local experts
  int32_t *recv_off = nullptr, *block_dst = nullptr, *row_map = nullptr, *grp_row = nullptr;
  int32_t *ts1 = nullptr, *ts2 = nullptr, *local_counts = nullptr;
  void *xp = nullptr, *hr = nullptr, *yr = nullptr;
  // shared group (static one-group tile tables)
  int32_t *sh_grp = nullptr, *sh_ts1 = nullptr, *sh_ts2 = nullptr;
  void *hs = nullptr, *ys = nullptr;
  CUtensorMap tmE, tmXp, tmHr, tmWguR, tmWdR, tmHs, tmWguS, tmWdS;
  DeviceArena mem;
};

namespace {

moe_status ep_validate(const moe_cfg* c, int32_t rank, int32_t world, int64_t recv_capacity) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (world < 1 || rank < 0 || rank >= world)
    return fail(MOE_ERR_INVALID_ARG, "rank=%d outside [0, world=%d)", rank, world);
  if (c->dtype != MOE_BF16)
    return fail(MOE_ERR_UNSUPPORTED, "the expert-parallel layer runs bf16 layers (MOE_BF16) only");
  if (c->T < 1 || c->T > (1 << 24)) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [1, 2^24]", c->T);
  if (c->n_routed < 1 || c->n_routed > kMaxRouted)
    return fail(MOE_ERR_UNSUPPORTED, "n_routed=%d outside [1, %d]", c->n_routed, kMaxRouted);
  if (c->n_routed % world)
    return fail(MOE_ERR_INVALID_ARG, "n_routed=%d is not a multiple of world=%d", c->n_routed, world);
  if (c->n_shared < 0 || c->n_shared > 64)
    return fail(MOE_ERR_INVALID_ARG, "n_shared=%d outside [0, 64]", c->n_shared);
  if (c->top_k < 1 || c->top_k > c->n_routed || c->top_k > kMaxTopK)
    return fail(MOE_ERR_INVALID_ARG, "top_k=%d outside [1, min(16, n_routed)]", c->top_k);
  if (c->d < 64 || c->d % 64 || c->inter < 64 || c->inter % 64)
    return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need d %% 64 == 0 and inter %% 64 == 0");
  if (!c->centroids || !c->w_gate || !c->w_up || !c->w_down)
    return fail(MOE_ERR_INVALID_ARG, "a weight pointer is NULL");
  if (recv_capacity < 0) return fail(MOE_ERR_INVALID_ARG, "recv_capacity < 0");
  const int64_t cap = recv_capacity ? recv_capacity : (int64_t)world * c->T * c->top_k;
  if (cap + (int64_t)c->n_routed * kPairBM >= (int64_t(1) << 30))
    return fail(MOE_ERR_UNSUPPORTED, "received-row capacity %lld too large", (long long)cap);
  return MOE_OK;
}

moe_status ep_create_impl(const moe_cfg& c, int32_t rank, int32_t world, int64_t recv_capacity,
                          moe_ep_handle* H) {
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
  H->rank = rank;
  H->world = world;
  H->n_local = c.n_routed / world;
  H->e0 = rank * H->n_local;
  H->recv_cap = recv_capacity ? recv_capacity : (int64_t)world * c.T * c.top_k;
  H->rows_cap = (H->recv_cap + (int64_t)H->n_local * (kPairBM - 1) + kPairBM - 1) / kPairBM * kPairBM;
  H->has_shared = c.n_shared > 0;
  H->inter_shared = c.n_shared * c.inter;
  H->T_pad = ((int64_t)c.T + kPairBM - 1) / kPairBM * kPairBM;
  H->n_pad = (c.n_routed + 15) / 16 * 16;
  H->maxc = router_maxc(H->n_pad);
  H->maxk = combine_maxk(c.top_k);
  H->small_router = c.T <= kSmallMaxTok && c.d % kSmallBM == 0;
  H->router_rows = H->small_router ? 1 : router_tile_rows(c.T, H->n_sms);
  H->n_tiles = (c.T + H->router_rows - 1) / H->router_rows;
  if (H->small_router) H->router_cluster = router_small_cluster(c.T, H->n_sms);

  const size_t d = c.d, I = c.inter, Is = H->inter_shared, ks = c.n_shared, nl = H->n_local;
  const size_t nr = c.n_routed, T = c.T, K = c.top_k, nt = H->n_tiles, es = 2;
  DeviceArena& M = H->mem;
  cudaStream_t st;
  MOE_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  struct StreamGuard {
    cudaStream_t s;
    ~StreamGuard() { cudaStreamDestroy(s); }
  } guard{st};

  // ---- weights
  MOE_TRY(M.alloc_t(&H->bias, (size_t)H->n_pad * 4));
  MOE_CUDA(cudaMemsetAsync(H->bias, 0, (size_t)H->n_pad * 4, st));
  if (c.logit_bias) MOE_CUDA(cudaMemcpyAsync(H->bias, c.logit_bias, nr * 4, cudaMemcpyDeviceToDevice, st));
  MOE_TRY(M.alloc(&H->centroids, (size_t)H->n_pad * d * es));
  MOE_CUDA(cudaMemsetAsync(H->centroids, 0, (size_t)H->n_pad * d * es, st));
  MOE_CUDA(cudaMemcpyAsync(H->centroids, c.centroids, nr * d * es, cudaMemcpyDeviceToDevice, st));
  const char* wg = static_cast<const char*>(c.w_gate);
  const char* wu = static_cast<const char*>(c.w_up);
  const char* wd = static_cast<const char*>(c.w_down);
  const size_t blk = 64 * d * es;   // gate/up interleaved in blocks of 64 rows
  if (ks) {
    MOE_TRY(M.alloc(&H->w_gu_s, 2 * Is * d * es));
    MOE_CUDA(cudaMemcpy2DAsync(H->w_gu_s, 2 * blk, wg, blk, blk, Is / 64, cudaMemcpyDeviceToDevice, st));
    MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_gu_s) + blk, 2 * blk, wu, blk, blk, Is / 64,
                               cudaMemcpyDeviceToDevice, st));
    MOE_TRY(M.alloc(&H->w_d_s, d * Is * es));
    for (size_t j = 0; j < ks; ++j)
      MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_d_s) + j * I * es, Is * es, wd + j * d * I * es,
                                 I * es, I * es, d, cudaMemcpyDeviceToDevice, st));
  }
  MOE_TRY(M.alloc(&H->w_gu_r, 2 * nl * I * d * es));
  MOE_CUDA(cudaMemcpy2DAsync(H->w_gu_r, 2 * blk, wg + ks * I * d * es, blk, blk, nl * I / 64,
                             cudaMemcpyDeviceToDevice, st));
  MOE_CUDA(cudaMemcpy2DAsync(static_cast<char*>(H->w_gu_r) + blk, 2 * blk, wu + ks * I * d * es, blk, blk,
                             nl * I / 64, cudaMemcpyDeviceToDevice, st));
  MOE_TRY(M.alloc(&H->w_d_r, nl * d * I * es));
  MOE_CUDA(cudaMemcpyAsync(H->w_d_r, wd + ks * d * I * es, nl * d * I * es, cudaMemcpyDeviceToDevice, st));

  // ---- dispatch workspace
  MOE_TRY(M.alloc_t(&H->topk_rank, T * K * 4));
  MOE_TRY(M.alloc_t(&H->slot_row, T * K * 4));
  MOE_TRY(M.alloc_t(&H->tile_hist, nt * nr * 4));
  MOE_TRY(M.alloc_t(&H->tile_base, nt * nr * 4));
  MOE_TRY(M.alloc_t(&H->tile_psum, nt * nr * 4));
  MOE_TRY(M.alloc_t(&H->psum_total, nr * 4));
  MOE_TRY(M.alloc_t(&H->disp_grp, nr * 4));
  MOE_TRY(M.alloc_t(&H->disp_ts1, (nr + 1) * 4));
  MOE_TRY(M.alloc_t(&H->disp_ts2, (nr + 1) * 4));
  MOE_TRY(M.alloc_t(&H->err, 256));
  MOE_CUDA(cudaMemsetAsync(H->err, 0, 256, st));
  // ---- local experts
  const size_t rc = (size_t)H->rows_cap;
  MOE_TRY(M.alloc_t(&H->recv_off, (nr + 1) * 4));
  MOE_TRY(M.alloc_t(&H->block_dst, nr * 4));
  MOE_TRY(M.alloc_t(&H->row_map, (size_t)H->recv_cap * 4 + 4));
  MOE_TRY(M.alloc_t(&H->grp_row, nl * 4));
  MOE_TRY(M.alloc_t(&H->ts1, (nl + 1) * 4));
  MOE_TRY(M.alloc_t(&H->ts2, (nl + 1) * 4));
  MOE_TRY(M.alloc_t(&H->local_counts, nl * 4));
  MOE_TRY(M.alloc(&H->xp, rc * d * es));
  MOE_TRY(M.alloc(&H->hr, rc * I * es));
  MOE_TRY(M.alloc(&H->yr, rc * d * es));
  // ---- shared group: one group of T rows, tile tables fixed by T
  if (ks) {
    const size_t tp = (size_t)H->T_pad;
    MOE_TRY(M.alloc(&H->hs, tp * Is * es));
    MOE_TRY(M.alloc(&H->ys, tp * d * es));
    MOE_TRY(M.alloc_t(&H->sh_grp, 4));
    MOE_TRY(M.alloc_t(&H->sh_ts1, 8));
    MOE_TRY(M.alloc_t(&H->sh_ts2, 8));
    const int mt = (int)(H->T_pad / kPairBM);
    const int32_t grp0 = 0;
    const int32_t t1[2] = {0, mt * (int)((Is + kGemmBN / 2 - 1) / (kGemmBN / 2))};
    const int32_t t2[2] = {0, mt * (int)((d + kGemmBN - 1) / kGemmBN)};
    MOE_CUDA(cudaMemcpyAsync(H->sh_grp, &grp0, 4, cudaMemcpyHostToDevice, st));
    MOE_CUDA(cudaMemcpyAsync(H->sh_ts1, t1, 8, cudaMemcpyHostToDevice, st));
    MOE_CUDA(cudaMemcpyAsync(H->sh_ts2, t2, 8, cudaMemcpyHostToDevice, st));
  }
  MOE_CUDA(cudaStreamSynchronize(st));

  // ---- kernels' attributes, persistent GEMM grid, TMA descriptors
  if (H->small_router) {
    H->simt_router_smem = router_epi_bytes(H->n_pad);
    const void* rk = with_maxc(H->maxc, [](auto m) { return (const void*)router_small_kernel<m()>; });
    MOE_CUDA(cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H->simt_router_smem));
  } else {
    const RouterStages rs = router_stages(H->n_pad, H->router_rows);
    if (rs.stages < 2) return fail(MOE_ERR_UNSUPPORTED, "router stages do not fit in shared memory");
    H->router_kps = rs.kps;
    H->router_stages = rs.stages;
    H->router_smem = router_smem_bytes(H->n_pad, rs.kps, H->router_rows, rs.stages);
    H->router_tmem_cols = router_tmem_cols(H->n_pad);
    const void* rk = with_maxc(H->maxc, [](auto m) { return (const void*)router_tc_kernel<m()>; });
    MOE_CUDA(cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H->router_smem));
  }
  MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
  MOE_CUDA(cudaFuncSetAttribute((const void*)grouped_gemm_tc_kernel<kDown>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
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
    MOE_CUDA(cudaOccupancyMaxActiveClusters(&clusters, (const void*)grouped_gemm_tc_kernel<kGateUpSwiGLU>, &lc));
    if (clusters < 1) return fail(MOE_ERR_UNSUPPORTED, "no CTA pair of the GEMM kernel fits on this device");
    H->gemm_grid = 2 * clusters;
  }
  bool ok = encode_2d(&H->tmE, H->centroids, d, (uint64_t)H->n_pad, (uint32_t)H->n_pad) &&
            encode_2d(&H->tmXp, H->xp, d, rc, 128) && encode_2d(&H->tmHr, H->hr, I, rc, 128) &&
            encode_3d(&H->tmWguR, H->w_gu_r, d, 2 * I, nl, kGemmBN / 2) &&
            encode_3d(&H->tmWdR, H->w_d_r, I, d, nl, kGemmBN / 2);
  if (ks)
    ok = ok && encode_2d(&H->tmWguS, H->w_gu_s, d, 2 * Is, kGemmBN / 2) &&
         encode_2d(&H->tmHs, H->hs, Is, (uint64_t)H->T_pad, 128) &&
         encode_2d(&H->tmWdS, H->w_d_s, Is, d, kGemmBN / 2);
  else {
    H->tmWguS = H->tmWguR;
    H->tmHs = H->tmHr;
    H->tmWdS = H->tmWdR;
  }
  if (!ok) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight/workspace tensor");
  return MOE_OK;
}

bool on_device(const moe_ep_handle* H) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == H->device;
}

}  // namespace

extern "C" {

moe_status moe_ep_create(const moe_cfg* cfg, int32_t rank, int32_t world, int64_t recv_capacity,
                         moe_ep_handle** out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  MOE_TRY(ep_validate(cfg, rank, world, recv_capacity));
  moe_ep_handle* H = new (std::nothrow) moe_ep_handle();
  if (!H) return fail(MOE_ERR_OOM, "host allocation failed");
  const moe_status s = ep_create_impl(*cfg, rank, world, recv_capacity, H);
  if (s != MOE_OK) {
    cudaDeviceSynchronize();
    H->mem.free_all();
    delete H;
    return s;
  }
  *out = H;
  return MOE_OK;
}

moe_status moe_ep_dispatch(moe_ep_handle* H, const void* u, int32_t* topk_idx, float* topk_w,
                           int32_t* expert_counts, float* aux_loss, void* send_rows,
                           moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!u || !topk_idx || !topk_w || !expert_counts || !aux_loss || !send_rows)
    return fail(MOE_ERR_INVALID_ARG, "an input/output pointer is NULL");
  if (!aligned16(u) || !aligned16(send_rows))
    return fail(MOE_ERR_INVALID_ARG, "u and send_rows must be 16-byte aligned");
  if (!on_device(H)) return fail(MOE_ERR_INVALID_ARG, "the current device is not the handle's device");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const int T = c.T, d = c.d, K = c.top_k, nr = c.n_routed;
  // unpadded expert offsets (bm = 1): the rows of expert e start at the rows of experts < e
  ScanArgs sa{H->tile_hist, H->tile_psum, H->n_tiles, nr, T, /*has_shared=*/0, /*inter_shared=*/0,
              c.inter, d, /*bm=*/1, /*tile_rows=*/kPairBM, kGemmBN / 2, kGemmBN, c.alpha1,
              expert_counts, aux_loss, H->psum_total, H->tile_base, H->disp_grp, H->disp_ts1,
              H->disp_ts2, /*copy_done=*/nullptr};
  RouterOut ro{topk_idx, topk_w, H->topk_rank, H->tile_hist, H->tile_psum, H->err};
  if (H->small_router) {
    RouterSmallArgs ra{static_cast<const __nv_bfloat16*>(u),
                       static_cast<const __nv_bfloat16*>(H->centroids), H->bias, T, d, nr, K, 1, ro};
    with_maxc(H->maxc, [&](auto m) {
      launch_pdl_cluster(router_small_kernel<m()>, dim3(H->n_tiles * H->router_cluster), dim3(kRouterEpiThreads),
                         H->simt_router_smem, stream, (unsigned)H->router_cluster, ra);
      return 0;
    });
  } else {
    CUtensorMap tmUr;
    if (!encode_2d(&tmUr, u, d, T, (uint32_t)H->router_rows))
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for u");
    RouterTcArgs ra{T, d, nr, H->n_pad, K, H->router_kps, H->router_stages, H->router_rows, H->n_tiles,
                    H->router_tmem_cols, H->bias, ro};
    const int rgrid = H->n_tiles < H->n_sms ? H->n_tiles : H->n_sms;
    with_maxc(H->maxc, [&](auto m) {
      launch_pdl(router_tc_kernel<m()>, dim3(rgrid), dim3(kRouterThreads), H->router_smem, stream, tmUr,
                 H->tmE, ra);
      return 0;
    });
  }
  MOE_CUDA(cudaGetLastError());
  launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, stream, sa);
  MOE_CUDA(cudaGetLastError());
  PermuteArgs pa{static_cast<const uint8_t*>(u), topk_idx, H->topk_rank, H->tile_base, H->slot_row,
                 static_cast<uint8_t*>(send_rows), T, K, nr, T * K, H->router_rows, d * 2, H->err};
  launch_pdl(permute_kernel, dim3((T + kPermuteWarps - 1) / kPermuteWarps), dim3(kPermuteWarps * 32), 0,
             stream, pa);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status moe_ep_experts(moe_ep_handle* H, const void* recv_rows, const int32_t* recv_counts,
                          int64_t n_recv, void* out_rows, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!recv_counts || (n_recv > 0 && (!recv_rows || !out_rows)))
    return fail(MOE_ERR_INVALID_ARG, "an input/output pointer is NULL");
  if (n_recv < 0 || n_recv > H->recv_cap)
    return fail(MOE_ERR_INVALID_ARG, "n_recv=%lld outside [0, capacity %lld]", (long long)n_recv,
                (long long)H->recv_cap);
  if ((recv_rows && !aligned16(recv_rows)) || (out_rows && !aligned16(out_rows)))
    return fail(MOE_ERR_INVALID_ARG, "recv_rows and out_rows must be 16-byte aligned");
  if (!on_device(H)) return fail(MOE_ERR_INVALID_ARG, "the current device is not the handle's device");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const int d = c.d, I = c.inter;
  EpLayoutArgs la{recv_counts, H->world, H->n_local, H->recv_off,
                  ScanArgs{recv_counts, /*tile_psum=*/nullptr, H->world, H->n_local, /*T=*/1,
                           /*has_shared=*/0, /*inter_shared=*/0, I, d, kPairBM, kPairBM, kGemmBN / 2,
                           kGemmBN, 0.f, H->local_counts, /*aux_loss=*/nullptr, /*psum_total=*/nullptr,
                           H->block_dst, H->grp_row, H->ts1, H->ts2, nullptr}};
  launch_pdl(ep_layout_kernel, dim3(1), dim3(kScanThreads), 0, stream, la);
  MOE_CUDA(cudaGetLastError());
  const unsigned mgrid = (unsigned)((n_recv + kEpMoveWarps - 1) / kEpMoveWarps);
  if (n_recv > 0) {
    EpMoveArgs ga{static_cast<const uint8_t*>(recv_rows), static_cast<uint8_t*>(H->xp), H->recv_off,
                  H->block_dst, H->row_map, n_recv, H->world * H->n_local, d * 2, H->rows_cap, H->err, 1};
    launch_pdl(ep_move_kernel, dim3(mgrid), dim3(kEpMoveWarps * 32), 0, stream, ga);
    MOE_CUDA(cudaGetLastError());
  }
  GemmArgs g1{};
  g1.grp_row = H->grp_row; g1.ts = H->ts1; g1.G = H->n_local; g1.has_shared = 0;
  g1.kb_shared = d / kGemmBK; g1.kb_routed = d / kGemmBK;
  g1.nt_shared = g1.nt_routed = (I + kGemmBN / 2 - 1) / (kGemmBN / 2);
  g1.out_shared = g1.out_routed = static_cast<__nv_bfloat16*>(H->hr);
  g1.ld_shared = g1.ld_routed = I;
  g1.rows_shared = g1.rows_routed = H->rows_cap;
  g1.cols_shared = g1.cols_routed = I;
  g1.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kGateUpSwiGLU>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes,
             stream, H->tmXp, H->tmXp, H->tmWguR, H->tmWguR, g1);
  MOE_CUDA(cudaGetLastError());
  GemmArgs g2{};
  g2.grp_row = H->grp_row; g2.ts = H->ts2; g2.G = H->n_local; g2.has_shared = 0;
  g2.kb_shared = I / kGemmBK; g2.kb_routed = I / kGemmBK;
  g2.nt_shared = g2.nt_routed = (d + kGemmBN - 1) / kGemmBN;
  g2.out_shared = g2.out_routed = static_cast<__nv_bfloat16*>(H->yr);
  g2.ld_shared = g2.ld_routed = d;
  g2.rows_shared = g2.rows_routed = H->rows_cap;
  g2.cols_shared = g2.cols_routed = d;
  g2.err = H->err;
  launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
             H->tmHr, H->tmHr, H->tmWdR, H->tmWdR, g2);
  MOE_CUDA(cudaGetLastError());
  if (n_recv > 0) {
    EpMoveArgs sa{static_cast<const uint8_t*>(H->yr), static_cast<uint8_t*>(out_rows), H->recv_off,
                  H->block_dst, H->row_map, n_recv, H->world * H->n_local, d * 2, H->rows_cap, H->err, 0};
    launch_pdl(ep_move_kernel, dim3(mgrid), dim3(kEpMoveWarps * 32), 0, stream, sa);
    MOE_CUDA(cudaGetLastError());
  }
  return MOE_OK;
}

moe_status moe_ep_combine(moe_ep_handle* H, const void* u, const void* back_rows, const float* topk_w,
                          void* h, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (!u || !back_rows || !topk_w || !h) return fail(MOE_ERR_INVALID_ARG, "an input/output pointer is NULL");
  if (!aligned16(u) || !aligned16(back_rows) || !aligned16(h))
    return fail(MOE_ERR_INVALID_ARG, "u, back_rows and h must be 16-byte aligned");
  if (!on_device(H)) return fail(MOE_ERR_INVALID_ARG, "the current device is not the handle's device");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_cfg& c = H->cfg;
  const int T = c.T, d = c.d, K = c.top_k, Is = H->inter_shared;
  if (H->has_shared) {
    CUtensorMap tmU;
    if (!encode_2d(&tmU, u, d, T, 128)) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for u");
    GemmArgs g1{};
    g1.grp_row = H->sh_grp; g1.ts = H->sh_ts1; g1.G = 1; g1.has_shared = 1;
    g1.kb_shared = g1.kb_routed = d / kGemmBK;
    g1.nt_shared = g1.nt_routed = (Is + kGemmBN / 2 - 1) / (kGemmBN / 2);
    g1.out_shared = g1.out_routed = static_cast<__nv_bfloat16*>(H->hs);
    g1.ld_shared = g1.ld_routed = Is;
    g1.rows_shared = g1.rows_routed = H->T_pad;
    g1.cols_shared = g1.cols_routed = Is;
    g1.err = H->err;
    launch_pdl(grouped_gemm_tc_kernel<kGateUpSwiGLU>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes,
               stream, tmU, tmU, H->tmWguS, H->tmWguS, g1);
    MOE_CUDA(cudaGetLastError());
    GemmArgs g2{};
    g2.grp_row = H->sh_grp; g2.ts = H->sh_ts2; g2.G = 1; g2.has_shared = 1;
    g2.kb_shared = g2.kb_routed = Is / kGemmBK;
    g2.nt_shared = g2.nt_routed = (d + kGemmBN - 1) / kGemmBN;
    g2.out_shared = g2.out_routed = static_cast<__nv_bfloat16*>(H->ys);
    g2.ld_shared = g2.ld_routed = d;
    g2.rows_shared = g2.rows_routed = H->T_pad;
    g2.cols_shared = g2.cols_routed = d;
    g2.err = H->err;
    launch_pdl(grouped_gemm_tc_kernel<kDown>, dim3(H->gemm_grid), dim3(kGemmThreads), kGemmSmemBytes, stream,
               H->tmHs, H->tmHs, H->tmWdS, H->tmWdS, g2);
    MOE_CUDA(cudaGetLastError());
  }
  const int parts = combine_parts(T, d / 8, H->n_sms);
  CombineArgs<__nv_bfloat16> ca{static_cast<const __nv_bfloat16*>(u),
                                H->has_shared ? static_cast<const __nv_bfloat16*>(H->ys) : nullptr,
                                static_cast<const __nv_bfloat16*>(back_rows), H->slot_row, topk_w,
                                static_cast<__nv_bfloat16*>(h), T, d, K, parts};
  const int cgrid = (int)(((int64_t)T * parts + kCombineWarps - 1) / kCombineWarps);
  with_maxk(H->maxk, [&](auto m) {
    launch_pdl(combine_bf16_kernel<m()>, dim3(cgrid), dim3(kCombineWarps * 32), 0, stream, ca);
    return 0;
  });
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

moe_status moe_ep_expert_psum(moe_ep_handle* H, float* psum, moe_stream_t stream_) {
  if (!H || !psum) return fail(MOE_ERR_INVALID_ARG, "handle or psum is NULL");
  MOE_CUDA(cudaMemcpyAsync(psum, H->psum_total, (size_t)H->cfg.n_routed * 4, cudaMemcpyDeviceToDevice,
                           reinterpret_cast<cudaStream_t>(stream_)));
  return MOE_OK;
}

moe_status moe_ep_device_status(moe_ep_handle* H, moe_stream_t stream_) {
  if (!H) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  MOE_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream_)));
  int code = 0;
  MOE_CUDA(cudaMemcpy(&code, H->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code != 0) {
    MOE_CUDA(cudaMemset(H->err, 0, sizeof(int)));
    return fail(MOE_ERR_DEVICE_CHECK, "a kernel recorded device error 0x%x", code);
  }
  return MOE_OK;
}

int64_t moe_ep_recv_capacity(const moe_ep_handle* H) { return H ? H->recv_cap : 0; }

void moe_ep_destroy(moe_ep_handle* H) {
  if (!H) return;
  cudaDeviceSynchronize();
  H->mem.free_all();
  delete H;
}

}  // extern "C"
