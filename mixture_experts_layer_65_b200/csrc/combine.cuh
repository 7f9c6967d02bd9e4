// combine.cuh -- gate-weighted combine with the residual, no atomics.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Routing in a classic MoE layer":
// h = sum_i g_i FFN_i(u) + u, with the K_s shared experts ("Where this sits", shared
// expert isolation) added with gate 1.  One warp owns one part of one token row (the
// whole row, unless there are too few tokens to keep the SMs' load slots busy) and sums,
// in fp32 and in a fixed order, u + (shared-group output) + g_0 Y_0 + ... + g_{K'-1}
// Y_{K'-1}, then rounds once to the output type.
#pragma once

#include "router.cuh"

namespace moe {

constexpr int kCombineWarps = 8;

// Compile-time bound on top_k for the per-vector load batch.
__host__ __device__ constexpr int combine_maxk(int top_k) {
  return top_k <= 4 ? 4 : top_k <= 6 ? 6 : top_k <= 8 ? 8 : top_k <= 12 ? 12 : 16;
}

template <typename T>
struct CombineArgs {
  const T* u;              // [T, d]
  const T* ys;             // [>= T, d] shared-group output, or nullptr when K_s = 0
  const T* yr;             // [rows_cap, d] routed outputs (expert-contiguous rows)
  const int32_t* slot_row; // [T, top_k]
  const float* topk_w;     // [T, top_k], or nullptr: every gate 1 (the backward's du)
  T* h;                    // [T, d]
  int T_, d, top_k;
  int parts;               // warps per token row, each a contiguous range of its vectors
  const T* xtra;           // [>= T, d] added last, or nullptr (the backward's router term)
};

// Warps per token row: 1 for large batches; for small ones enough to give the SMs about
// 16 warps each, with at least 32 vectors (one per lane) per part.
inline int combine_parts(int T, int nvec, int n_sms) {
  int p = (n_sms * 16) / (T > 0 ? T : 1);
  const int pmax = nvec / 32 > 1 ? nvec / 32 : 1;
  return p < 1 ? 1 : (p > pmax ? pmax : p);
}

// Vector range [v0, v1) of part `part` of a row of nvec vectors split into `parts`.
__device__ __forceinline__ void combine_range(int nvec, int parts, int part, int& v0, int& v1) {
  const int per = (nvec + parts - 1) / parts;
  v0 = part * per;
  v1 = v0 + per < nvec ? v0 + per : nvec;
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint4& v, float w) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
  }
}

// bf16 rows: 8 elements per 16-byte vector; each lane handles vectors lane, lane+32, ...
// All 2 + top_k loads of a vector are issued before the fixed-order accumulation.
template <int MAXK>
__global__ void __launch_bounds__(kCombineWarps * 32)
combine_bf16_kernel(CombineArgs<__nv_bfloat16> a) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kCombineWarps + warp;
  const int t = gw / a.parts;
  if (t >= a.T_) return;
  __shared__ int s_row[kCombineWarps][kMaxTopK];
  __shared__ float s_w[kCombineWarps][kMaxTopK];
  if (lane < a.top_k) {
    s_row[warp][lane] = a.slot_row[(size_t)t * a.top_k + lane];
    s_w[warp][lane] = a.topk_w ? a.topk_w[(size_t)t * a.top_k + lane] : 1.0f;
  }
  __syncwarp();
  const uint4* yk[MAXK];
  float wk[MAXK];
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    const bool on = k < a.top_k;
    yk[k] = reinterpret_cast<const uint4*>(a.yr + (size_t)(on ? s_row[warp][k] : 0) * a.d);
    wk[k] = on ? s_w[warp][k] : 0.f;
  }
  int v0, v1;
  combine_range(a.d >> 3, a.parts, gw - t * a.parts, v0, v1);
  const uint4* ur = reinterpret_cast<const uint4*>(a.u + (size_t)t * a.d);
  const uint4* sr = a.ys ? reinterpret_cast<const uint4*>(a.ys + (size_t)t * a.d) : nullptr;
  const uint4* xr = a.xtra ? reinterpret_cast<const uint4*>(a.xtra + (size_t)t * a.d) : nullptr;
  uint4* hr = reinterpret_cast<uint4*>(a.h + (size_t)t * a.d);
  for (int v = v0 + lane; v < v1; v += 32) {
    uint4 x[MAXK];
    const uint4 xu = __ldg(ur + v);
    const uint4 xs = sr ? __ldg(sr + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (k < a.top_k) x[k] = __ldg(yk[k] + v);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    add8(acc, xu, 1.0f);
    if (sr) add8(acc, xs, 1.0f);
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (k < a.top_k) add8(acc, x[k], wk[k]);
    if (xr) add8(acc, __ldg(xr + v), 1.0f);
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    hr[v] = o;
  }
}

// fp32 rows: 4 elements per 16-byte vector
static __global__ void __launch_bounds__(kCombineWarps * 32) combine_f32_kernel(CombineArgs<float> a) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kCombineWarps + warp;
  const int t = gw / a.parts;
  if (t >= a.T_) return;
  __shared__ int s_row[kCombineWarps][kMaxTopK];
  __shared__ float s_w[kCombineWarps][kMaxTopK];
  if (lane < a.top_k) {
    s_row[warp][lane] = a.slot_row[(size_t)t * a.top_k + lane];
    s_w[warp][lane] = a.topk_w[(size_t)t * a.top_k + lane];
  }
  __syncwarp();
  int v0, v1;
  combine_range(a.d >> 2, a.parts, gw - t * a.parts, v0, v1);
  const float4* ur = reinterpret_cast<const float4*>(a.u + (size_t)t * a.d);
  const float4* sr = a.ys ? reinterpret_cast<const float4*>(a.ys + (size_t)t * a.d) : nullptr;
  float4* hr = reinterpret_cast<float4*>(a.h + (size_t)t * a.d);
  for (int v = v0 + lane; v < v1; v += 32) {
    float4 acc = __ldg(ur + v);
    if (sr) {
      const float4 s = __ldg(sr + v);
      acc.x += s.x; acc.y += s.y; acc.z += s.z; acc.w += s.w;
    }
    for (int k = 0; k < a.top_k; ++k) {
      const int rk = s_row[warp][k];
      const float wk = s_w[warp][k];
      const float4 y = __ldg(reinterpret_cast<const float4*>(a.yr + (size_t)rk * a.d) + v);
      acc.x = fmaf(wk, y.x, acc.x); acc.y = fmaf(wk, y.y, acc.y);
      acc.z = fmaf(wk, y.z, acc.z); acc.w = fmaf(wk, y.w, acc.w);
    }
    hr[v] = acc;
  }
}

}  // namespace moe
