// scan_permute.cuh -- expert-contiguous regrouping of the routed token rows.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Top-k routing, from affinities to gates":
// a production layer groups the tokens of each expert so that every expert runs one
// dense GEMM chain over its rows.  After the scan (scan.cuh)
// has placed every (router tile, expert) in the expert-contiguous row space, the permute
// copies each token row to its top_k destinations (order inside an expert = ascending token
// id): as a kernel of its own, or inside the copy warps of the gate/up GEMM.
#pragma once

#include "router.cuh"

namespace moe {

// One warp per token: compute the token's top_k destination rows, record them for the
// combine, and copy the row (16-byte vectors, read once, written top_k times).
struct PermuteArgs {
  const uint8_t* u;            // [T, row_bytes]
  const int32_t* topk_idx;     // [T, top_k]
  const int32_t* topk_rank;    // [T, top_k]
  const int32_t* tile_base;    // [n_tiles, n_routed]
  int32_t* slot_row;           // [T, top_k] destination row (output)
  uint8_t* xp;                 // [rows_cap, row_bytes]
  int T, top_k, n_routed, rows_cap;
  int tile_rows;               // tokens per router tile
  int row_bytes;               // multiple of 16
  int* err;
  const float* scale_src;      // [T] per-row scales copied along with the rows, or nullptr
  float* scale_dst;            // [rows_cap]
};

constexpr int kPermuteWarps = 8;
constexpr int kPermuteVec = 8;   // 16-byte vectors held per lane per pass

// One warp copies token t's row to its top_k destinations (and records them for the
// combine).  Used by permute_kernel and by the copy warps of the fused gate/up GEMM.
__device__ __forceinline__ void permute_token(const PermuteArgs& a, int t, int lane) {
  int my_dest = -1;
  if (lane < a.top_k) {
    const int e = a.topk_idx[(size_t)t * a.top_k + lane];
    if (e >= 0 && e < a.n_routed) {
      const int dst = a.tile_base[(size_t)(t / a.tile_rows) * a.n_routed + e] +
                      a.topk_rank[(size_t)t * a.top_k + lane];
      if (dst >= 0 && dst < a.rows_cap) my_dest = dst;
      else record_error(a.err, kErrPermuteRow);
    } else {
      record_error(a.err, kErrRouteIndex);
    }
    a.slot_row[(size_t)t * a.top_k + lane] = my_dest < 0 ? 0 : my_dest;
    if (my_dest >= 0 && a.scale_dst) a.scale_dst[my_dest] = a.scale_src[t];
  }
  const int nvec = a.row_bytes >> 4;
  const uint4* src = reinterpret_cast<const uint4*>(a.u + (size_t)t * a.row_bytes);
  for (int v0 = 0; v0 < nvec; v0 += 32 * kPermuteVec) {
    uint4 buf[kPermuteVec];
#pragma unroll
    for (int j = 0; j < kPermuteVec; ++j) {
      const int v = v0 + j * 32 + lane;
      if (v < nvec) buf[j] = __ldg(src + v);
    }
    for (int k = 0; k < a.top_k; ++k) {
      const int dst = __shfl_sync(0xffffffffu, my_dest, k);
      if (dst < 0) continue;
      uint4* out = reinterpret_cast<uint4*>(a.xp + (size_t)dst * a.row_bytes);
#pragma unroll
      for (int j = 0; j < kPermuteVec; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < nvec) out[v] = buf[j];
      }
    }
  }
}

static __global__ void __launch_bounds__(kPermuteWarps * 32) permute_kernel(PermuteArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kPermuteWarps + warp;
  if (t >= a.T) return;
  permute_token(a, t, lane);
}

}  // namespace moe
