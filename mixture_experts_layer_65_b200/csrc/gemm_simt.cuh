// gemm_simt.cuh -- fp32 grouped expert GEMMs on the CUDA cores (fp32 layers).
//
// Same grouping and tile tables as the tensor-core kernels (shared group first, then one
// group per routed expert, 128-row blocks); computes in fp32 FMA so an fp32 layer keeps
// fp32 accuracy end to end.
//   mode kGateUpSwiGLU:  Hmid = SiLU(X W_gate^T) * (X W_up^T)
//   mode kDown:          Y    = Hmid W_down^T
// A CTA of 256 threads computes a 128 x 64 output tile; each thread owns 8 x 4 outputs.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

constexpr int kSimtBM = 128, kSimtBN = 64, kSimtBK = 16, kSimtThreads = 256;

struct SimtGemmArgs {
  const int32_t* grp_row;
  const int32_t* ts;
  int G, has_shared;
  const float* a_shared;      // [a_rows_shared, K_shared]
  const float* a_routed;      // [a_rows_routed, K_routed]
  int64_t a_rows_shared, a_rows_routed;
  int K_shared, K_routed;
  const float* b0_shared;     // [N_shared, K_shared]
  const float* b1_shared;     // up weights (gate/up mode only)
  const float* b0_routed;     // [n_routed][N_routed, K_routed]
  const float* b1_routed;
  int64_t b_expert_stride;    // elements between routed experts
  int N_shared, N_routed;
  int nt_shared, nt_routed;
  float* out_shared;
  int64_t out_rows_shared;
  float* out_routed;
  int64_t out_rows_routed;
  int* err;
};

template <int MODE>
__global__ void __launch_bounds__(kSimtThreads) grouped_gemm_simt_kernel(SimtGemmArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float As[kSimtBK][kSimtBM + 4];
  __shared__ float Bs[2][kSimtBK][kSimtBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int total = a.ts[a.G];
  int g = 0;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    while (tile >= a.ts[g + 1]) ++g;
    const int local = tile - a.ts[g];
    const bool sh = a.has_shared && g == 0;
    const int nt = sh ? a.nt_shared : a.nt_routed;
    const int m = local / nt, n = local - m * nt;
    const int e = g - a.has_shared;
    const float* A = sh ? a.a_shared : a.a_routed;
    const int64_t arows = sh ? a.a_rows_shared : a.a_rows_routed;
    const int K = sh ? a.K_shared : a.K_routed;
    const int N = sh ? a.N_shared : a.N_routed;
    const float* B0 = sh ? a.b0_shared : a.b0_routed + (int64_t)e * a.b_expert_stride;
    const float* B1 = sh ? a.b1_shared : a.b1_routed + (int64_t)e * a.b_expert_stride;
    float* out = sh ? a.out_shared : a.out_routed;
    const int64_t orows = sh ? a.out_rows_shared : a.out_rows_routed;
    const int64_t row0 = (int64_t)a.grp_row[g] + (int64_t)m * kSimtBM;
    const int col0 = n * kSimtBN;

    float acc0[8][4], acc1[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) { acc0[i][j] = 0.f; acc1[i][j] = 0.f; }

    for (int k0 = 0; k0 < K; k0 += kSimtBK) {
#pragma unroll
      for (int l = 0; l < 2; ++l) {
        const int idx = tid + l * kSimtThreads;
        const int r = idx >> 2, kq = (idx & 3) * 4;
        const int64_t gr = row0 + r;
        const int k = k0 + kq;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (gr < arows && k < K) v = *reinterpret_cast<const float4*>(A + gr * K + k);
        As[kq][r] = v.x; As[kq + 1][r] = v.y; As[kq + 2][r] = v.z; As[kq + 3][r] = v.w;
      }
      {
        const int r = tid >> 2, kq = (tid & 3) * 4;
        const int gc = col0 + r;
        const int k = k0 + kq;
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (gc < N && k < K) {
          v0 = __ldg(reinterpret_cast<const float4*>(B0 + (int64_t)gc * K + k));
          if (MODE == kGateUpSwiGLU) v1 = __ldg(reinterpret_cast<const float4*>(B1 + (int64_t)gc * K + k));
        }
        Bs[0][kq][r] = v0.x; Bs[0][kq + 1][r] = v0.y; Bs[0][kq + 2][r] = v0.z; Bs[0][kq + 3][r] = v0.w;
        if (MODE == kGateUpSwiGLU) {
          Bs[1][kq][r] = v1.x; Bs[1][kq + 1][r] = v1.y; Bs[1][kq + 2][r] = v1.z; Bs[1][kq + 3][r] = v1.w;
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kSimtBK; ++kk) {
        float af[8], b0[4], b1[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) af[i] = As[kk][ty * 8 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b0[j] = Bs[0][kk][tx * 4 + j];
          b1[j] = (MODE == kGateUpSwiGLU) ? Bs[1][kk][tx * 4 + j] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc0[i][j] = fmaf(af[i], b0[j], acc0[i][j]);
            if (MODE == kGateUpSwiGLU) acc1[i][j] = fmaf(af[i], b1[j], acc1[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t orow = row0 + ty * 8 + i;
      if (orow >= orows) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int oc = col0 + tx * 4 + j;
        if (oc < N)
          out[orow * N + oc] =
              (MODE == kGateUpSwiGLU) ? silu_f32(acc0[i][j]) * acc1[i][j] : acc0[i][j];
      }
    }
  }
}

}  // namespace moe
