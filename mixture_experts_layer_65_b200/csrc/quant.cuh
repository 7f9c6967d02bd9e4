// quant.cuh -- per-row scaled e4m3 quantisation of bf16 rows, for the e4m3 gate/up
// variant of the layer (MOE_BF16_E4M3_GATEUP; not on the DeepSeekMoE pages).
//
// Row x of n bf16 values: a = max |x_i| (exact); a = 0 gives q = 0 and scale 0;
// otherwise inv = fp32(448 / a), q_i = e4m3(fp32(x_i * inv)) with round-to-nearest-even
// and saturation at +-448, scale = fp32(a / 448), so x_i ~ q_i * scale.  Divisions and
// products use the IEEE round-to-nearest forms explicitly.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace moe {

constexpr int kQuantWarps = 8;

struct QuantArgs {
  const __nv_bfloat16* src;   // [rows, cols], cols % 8 == 0, 16-byte aligned rows
  int64_t rows;
  int cols;
  uint8_t* dst;               // [rows, cols] e4m3 bytes
  float* scale;               // [rows]
};

// One warp per row: the row maximum by shuffles, then the row converted 8 values per lane
// and step.
static __global__ void __launch_bounds__(kQuantWarps * 32) quant_rows_e4m3_kernel(QuantArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = a.cols >> 3;
  for (int64_t r = (int64_t)blockIdx.x * kQuantWarps + warp; r < a.rows;
       r += (int64_t)gridDim.x * kQuantWarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a.src + r * a.cols);
    float amax = 0.f;
    for (int v = lane; v < nv; v += 32) {
      float f[8];
      bf16x8_to_f32(__ldg(src + v), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
    uint2* dst = reinterpret_cast<uint2*>(a.dst + r * a.cols);
    for (int v = lane; v < nv; v += 32) {
      float f[8];
      bf16x8_to_f32(__ldg(src + v), f);
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(f[4 * h], inv), __fmul_rn(f[4 * h + 1], inv)), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(f[4 * h + 2], inv), __fmul_rn(f[4 * h + 3], inv)), __NV_SATFINITE,
            __NV_E4M3);
        w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
      dst[v] = make_uint2(w[0], w[1]);
    }
    if (lane == 0) a.scale[r] = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
  }
}

}  // namespace moe
