// api_common.cuh -- host-side helpers shared by the C-ABI's translation units: status and
// error text, TMA descriptor encoding, device allocations owned by a handle, and the
// dispatch of the kernels' compile-time bounds.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <type_traits>
#include <vector>

#include "moe.h"

namespace moe {

void set_last_error(const char* msg);   // moe_api.cu: the text moe_last_error() returns

inline moe_status fail(moe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_last_error(buf);
  return st;
}

#define MOE_CUDA(expr)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess)                                                                    \
      return ::moe::fail(MOE_ERR_CUDA, "%s: %s (%s:%d)", #expr, cudaGetErrorString(e_),       \
                         __FILE__, __LINE__);                                                 \
  } while (0)

#define MOE_TRY(expr)              \
  do {                             \
    moe_status s_ = (expr);        \
    if (s_ != MOE_OK) return s_;   \
  } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major [outer, inner] matrix of `es`-byte elements (bf16: 2, e4m3: 1), box = box_outer
// rows x 128 bytes, 128-byte swizzle.
inline bool encode_2d_es(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                         uint32_t box_outer, int es) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)es};
  cuuint32_t box[2] = {128u / (uint32_t)es, box_outer};
  cuuint32_t ess[2] = {1, 1};
  return fn(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(ptr), dims, strides, box, ess, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [depth, outer, inner] of `es`-byte elements, box = box_outer rows x 128 bytes of one matrix.
inline bool encode_3d_es(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                         uint64_t depth, uint32_t box_outer, int es) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, outer, depth};
  cuuint64_t strides[2] = {inner * (uint64_t)es, inner * outer * (uint64_t)es};
  cuuint32_t box[3] = {128u / (uint32_t)es, box_outer, 1};
  cuuint32_t ess[3] = {1, 1, 1};
  return fn(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
            const_cast<void*>(ptr), dims, strides, box, ess, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool encode_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  return encode_2d_es(m, ptr, inner, outer, box_outer, 2);
}
inline bool encode_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t depth,
                      uint32_t box_outer) {
  return encode_3d_es(m, ptr, inner, outer, depth, box_outer, 2);
}
inline bool encode_2d_e4m3(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                           uint32_t box_outer) {
  return encode_2d_es(m, ptr, inner, outer, box_outer, 1);
}
inline bool encode_3d_e4m3(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                           uint64_t depth, uint32_t box_outer) {
  return encode_3d_es(m, ptr, inner, outer, depth, box_outer, 1);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device allocations a handle owns, freed together.
struct DeviceArena {
  std::vector<void*> allocs;
  size_t bytes = 0;
  moe_status alloc(void** p, size_t n) {
    *p = nullptr;
    if (n == 0) return MOE_OK;
    cudaError_t e = cudaMalloc(p, n);
    if (e != cudaSuccess) {
      cudaGetLastError();
      *p = nullptr;
      return fail(MOE_ERR_OOM, "cudaMalloc(%zu) failed: %s", n, cudaGetErrorString(e));
    }
    allocs.push_back(*p);
    bytes += n;
    return MOE_OK;
  }
  template <class T>
  moe_status alloc_t(T** p, size_t n) { return alloc(reinterpret_cast<void**>(p), n); }
  void free_all() {
    for (void* p : allocs) cudaFree(p);
    allocs.clear();
    bytes = 0;
  }
};

// Call f(std::integral_constant<int, MAXC>{}) for the router's bound on N_pad / 8.
template <class F>
auto with_maxc(int maxc, F&& f) {
  switch (maxc) {
    case 2: return f(std::integral_constant<int, 2>{});
    case 4: return f(std::integral_constant<int, 4>{});
    case 8: return f(std::integral_constant<int, 8>{});
    case 16: return f(std::integral_constant<int, 16>{});
    default: return f(std::integral_constant<int, 32>{});
  }
}

// Call f(std::integral_constant<int, MAXK>{}) for the combine's bound on top_k.
template <class F>
auto with_maxk(int maxk, F&& f) {
  switch (maxk) {
    case 4: return f(std::integral_constant<int, 4>{});
    case 6: return f(std::integral_constant<int, 6>{});
    case 8: return f(std::integral_constant<int, 8>{});
    case 12: return f(std::integral_constant<int, 12>{});
    default: return f(std::integral_constant<int, 16>{});
  }
}

}  // namespace moe
