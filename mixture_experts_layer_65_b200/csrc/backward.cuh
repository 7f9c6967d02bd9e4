// backward.cuh -- the SIMT kernels of the layer's backward pass (the GEMMs are the grouped
// tensor-core kernel of gemm_tc.cuh).
//
// The pages give the forward only ("Routing in a classic MoE layer": h = u + sum_shared
// FFN_j(u) + sum_i g_i FFN_i(u), g_i = s_i on the chosen experts; "Expert-level balance
// loss": L_ExpBal = alpha_1 sum_i f_i P_i).  Differentiating L = sum_t dh_t . h_t +
// d_aux * aux, with the top-k choice (and f_i = count_i / T) held fixed:
//   dY_{t,k}   = g_{t,k} dh_t                    the routed output rows' gradient
//   dg_{t,k}   = dh_t . Y_{t,k}                  the chosen gates' gradient
//   ds_{t,i}   = dg at the chosen experts + d_aux alpha_1 f_i / T
//   dl_{t,i}   = s_{t,i} (ds_{t,i} - sum_j s_{t,j} ds_{t,j})          (softmax backward)
//   du_t       = dh_t + dX_shared,t + sum_k dX_{t,k} + sum_i dl_{t,i} e_i
//   de_i       = sum_t dl_{t,i} u_t,   db_i = sum_t dl_{t,i}
// where dX is each expert's input gradient (the GEMMs: dHmid = dY W_down, the SwiGLU
// backward, [da db] [W_gate; W_up]).
#pragma once

#include "router.cuh"

namespace moe {

// -------------------------------------------------------------------------- transposes
// [batch][R][C] bf16 -> [batch][C][R], 32 x 32 tiles through shared memory (8 rows per
// thread step).  Used once, for the transposed weight copies of the backward GEMMs.
constexpr int kTrTile = 32;

static __global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* src,
                                                                    __nv_bfloat16* dst, int R,
                                                                    int C) {
  __shared__ __nv_bfloat16 tile[kTrTile][kTrTile + 2];
  const size_t plane = (size_t)R * C;
  const __nv_bfloat16* s = src + blockIdx.z * plane;
  __nv_bfloat16* d = dst + blockIdx.z * plane;
  const int c0 = blockIdx.x * kTrTile, r0 = blockIdx.y * kTrTile;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < kTrTile; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < R && c < C) tile[i][tx] = s[(size_t)r * C + c];
  }
  __syncthreads();
  for (int i = ty; i < kTrTile; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (r < R && c < C) d[(size_t)c * R + r] = tile[tx][i];
  }
}

// -------------------------------------------------------------------------- routed rows
struct BwdRowsArgs {
  const __nv_bfloat16* dh;     // [T, d] incoming gradient of h
  const float* topk_w;         // [T, K] gates
  const int32_t* slot_row;     // [T, K] the forward's row of (t, k)
  const __nv_bfloat16* yr;     // [rows, d] the forward's routed expert outputs
  __nv_bfloat16* dyr;          // [rows, d] out: g dh at row of (t, k)
  float* dg;                   // [T, K] out: dh . Y
  int T, d, K;
  int64_t rows;
  int* err;
};

constexpr int kBwdWarps = 8;

// One warp per token: the K scaled copies of dh_t and the K dot products dh_t . Y_{t,k}
// (each lane sums its 16-byte vectors lane, lane + 32, ... in order, then a butterfly).
static __global__ void __launch_bounds__(kBwdWarps * 32) bwd_rows_kernel(BwdRowsArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int nv = a.d >> 3;
  const uint4* dhr = reinterpret_cast<const uint4*>(a.dh + (size_t)t * a.d);
  for (int k = 0; k < a.K; ++k) {
    const int64_t row = __ldg(a.slot_row + (size_t)t * a.K + k);
    if (row < 0 || row >= a.rows) {
      if (lane == 0) record_error(a.err, kErrPermuteRow);
      continue;
    }
    const float g = __ldg(a.topk_w + (size_t)t * a.K + k);
    const uint4* yv = reinterpret_cast<const uint4*>(a.yr + row * a.d);
    uint4* out = reinterpret_cast<uint4*>(a.dyr + row * a.d);
    float dot = 0.f;
    for (int v = lane; v < nv; v += 32) {
      float x[8], y[8];
      bf16x8_to_f32(__ldg(dhr + v), x);
      bf16x8_to_f32(__ldg(yv + v), y);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(x[i], y[i], dot);
      out[v] = make_uint4(pack_bf16x2(g * x[0], g * x[1]), pack_bf16x2(g * x[2], g * x[3]),
                          pack_bf16x2(g * x[4], g * x[5]), pack_bf16x2(g * x[6], g * x[7]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) a.dg[(size_t)t * a.K + k] = dot;
  }
}

// -------------------------------------------------------------------------- router
struct BwdRouterArgs {
  const float* logits;         // [T, n_routed] the forward's logits (bias added)
  const int32_t* topk_idx;     // [T, K]
  const float* dg;             // [T, K]
  const int32_t* counts;       // [n_routed] the forward's expert counts
  int T, n_routed, K, n_pad;
  int kpad;                    // dlb's row length (n_pad rounded up to 64)
  float aux_scale;             // d_aux * alpha_1 / T^2 (times count_i: the balance term)
  float* dl;                   // [T, n_pad] out: dL/dlogit (fp32; columns past n_routed 0)
  __nv_bfloat16* dlb;          // [T_pad, kpad] out: the same in bf16 (A of the e-product GEMM)
};

// One warp per token, lane l holding columns l + 32 m: the affinities recomputed as in the
// forward (max by redux on the order-preserving keys, exp(l - max), butterfly sum), then
// ds, sum_j s_j ds_j (butterfly) and dl = s (ds - that sum).
template <int MAXC>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_router_kernel(BwdRouterArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int MC = (MAXC + 3) / 4;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const float* lr = a.logits + (size_t)t * a.n_routed;
  float x[MC], ds[MC];
  uint32_t kmax = 0u;
#pragma unroll
  for (int m = 0; m < MC; ++m) {
    const int c = lane + 32 * m;
    const bool in = c < a.n_routed;
    x[m] = in ? __ldg(lr + c) : 0.f;
    kmax = max(kmax, in ? logit_key(x[m]) : 0u);
    ds[m] = in ? a.aux_scale * (float)__ldg(a.counts + c) : 0.f;
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const float lmax = key_logit(kmax);
  float part = 0.f;
#pragma unroll
  for (int m = 0; m < MC; ++m) {
    const int c = lane + 32 * m;
    x[m] = c < a.n_routed ? __expf(x[m] - lmax) : 0.f;
    part += x[m];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const float inv = 1.0f / part;
  for (int k = 0; k < a.K; ++k) {   // chosen experts: + dg (a token picks an expert once)
    const int e = __ldg(a.topk_idx + (size_t)t * a.K + k);
    const float g = __ldg(a.dg + (size_t)t * a.K + k);
#pragma unroll
    for (int m = 0; m < MC; ++m)
      if (lane + 32 * m == e) ds[m] += g;
  }
  float sds = 0.f;
#pragma unroll
  for (int m = 0; m < MC; ++m) {
    x[m] *= inv;   // s
    sds = fmaf(x[m], ds[m], sds);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sds += __shfl_xor_sync(0xffffffffu, sds, o);
#pragma unroll
  for (int m = 0; m < MC; ++m) {
    const int c = lane + 32 * m;
    if (c < a.n_pad) {
      const float v = c < a.n_routed ? x[m] * (ds[m] - sds) : 0.f;
      a.dl[(size_t)t * a.n_pad + c] = v;
      a.dlb[(size_t)t * a.kpad + c] = __float2bfloat16_rn(v);
    }
  }
}

// -------------------------------------------------------------------------- centroids
// de_i = sum_t dl_{t,i} u_t and db_i = sum_t dl_{t,i}, in two fixed-order passes: CTA
// (column block, token chunk) sums its chunk's tokens in order into a partial; the reduce
// kernel adds the chunks' partials in order.
constexpr int kCenCols = 64;      // columns of d per CTA
constexpr int kCenChunk = 512;    // tokens per CTA
constexpr int kCenStep = 32;      // tokens staged in shared memory at a time

struct BwdCentroidArgs {
  const float* dl;             // [T, n_pad]
  const __nv_bfloat16* u;      // [T, d]
  int T, d, n_routed, n_pad, n_chunks;
  float* part;                 // [n_chunks, n_routed, d + 1]: column d holds the bias part
};

// 256 threads: thread (i, q) accumulates experts i0, i0 + 16, ... (at most MAXPER of them,
// MAXPER = ceil(n_routed / 16) rounded up to a power of two) over 4 of the CTA's 64 columns
// (q), plus, for q == 0, the bias sums; tokens in ascending order.
__host__ __device__ constexpr int centroid_maxper(int n_routed) {
  return n_routed <= 16 ? 1 : n_routed <= 32 ? 2 : n_routed <= 64 ? 4 : n_routed <= 128 ? 8 : 16;
}
template <int MAXPER>
__global__ void __launch_bounds__(256) bwd_centroid_partial_kernel(BwdCentroidArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float s_u[kCenStep][kCenCols];
  __shared__ float s_dl[kCenStep][kMaxRouted];
  const int col0 = blockIdx.x * kCenCols;
  const int chunk = blockIdx.y;
  const int t0 = chunk * kCenChunk, t1 = min(a.T, t0 + kCenChunk);
  const int q = threadIdx.x & 15;           // columns col0 + 4 q .. + 3
  const int i0 = threadIdx.x >> 4;          // experts i0, i0 + 16, ...
  constexpr int kMaxPer = MAXPER;
  float acc[kMaxPer][4];
  float bacc[kMaxPer];
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    bacc[j] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
  }
  for (int tb = t0; tb < t1; tb += kCenStep) {
    const int nt = min(kCenStep, t1 - tb);
    for (int idx = threadIdx.x; idx < kCenStep * kCenCols; idx += 256) {
      const int r = idx / kCenCols, c = idx - r * kCenCols;
      s_u[r][c] = (r < nt && col0 + c < a.d) ? __bfloat162float(a.u[(size_t)(tb + r) * a.d + col0 + c]) : 0.f;
    }
    for (int idx = threadIdx.x; idx < kCenStep * a.n_pad; idx += 256) {
      const int r = idx / a.n_pad, c = idx - r * a.n_pad;
      s_dl[r][c] = r < nt ? a.dl[(size_t)(tb + r) * a.n_pad + c] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < nt; ++r) {
      const float4 uv = *reinterpret_cast<const float4*>(&s_u[r][4 * q]);
#pragma unroll
      for (int j = 0; j < kMaxPer; ++j) {
        const int i = i0 + 16 * j;
        if (i < a.n_routed) {
          const float w = s_dl[r][i];
          acc[j][0] = fmaf(w, uv.x, acc[j][0]);
          acc[j][1] = fmaf(w, uv.y, acc[j][1]);
          acc[j][2] = fmaf(w, uv.z, acc[j][2]);
          acc[j][3] = fmaf(w, uv.w, acc[j][3]);
          bacc[j] += w;
        }
      }
    }
    __syncthreads();
  }
  const size_t ld = (size_t)a.d + 1;
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    const int i = i0 + 16 * j;
    if (i >= a.n_routed) continue;
    float* p = a.part + ((size_t)chunk * a.n_routed + i) * ld;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (col0 + 4 * q + c < a.d) p[col0 + 4 * q + c] = acc[j][c];
    if (blockIdx.x == 0 && q == 0) p[a.d] = bacc[j];
  }
}

// Sum the chunks' partials in chunk order: d_centroids [n_routed, d], d_bias [n_routed].
static __global__ void __launch_bounds__(256) bwd_centroid_reduce_kernel(const float* part, int n_chunks,
                                                                         int n_routed, int d,
                                                                         float* d_cen, float* d_bias) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t ld = (size_t)d + 1, n = (size_t)n_routed * ld;
  for (size_t idx = (size_t)blockIdx.x * 256 + threadIdx.x; idx < n; idx += (size_t)gridDim.x * 256) {
    float s = 0.f;
    for (int ch = 0; ch < n_chunks; ++ch) s += part[(size_t)ch * n + idx];
    const size_t i = idx / ld, c = idx - i * ld;
    if (c < (size_t)d) d_cen[i * d + c] = s;
    else if (d_bias) d_bias[i] = s;
  }
}

}  // namespace moe

namespace moe {

// -------------------------------------------------------------------------- weight grads
// The weight gradients are sums over each expert's rows (dW_down = dY^T Hmid,
// dW_{gate,up} = [da db]^T X): GEMMs whose K is the row dimension.  The grouped GEMM takes
// both operands K-major, so the row-major activations are first transposed into
// [width, rows] copies; rows that are padding between groups become zero columns (the
// forward leaves them unspecified, and they must add nothing).
struct MaskedTransposeArgs {
  const __nv_bfloat16* src;   // [rows, C] row-major, row stride ld_src
  __nv_bfloat16* dst;         // [C, ld_dst]: dst[c][r] = src[r][c] on valid rows, else 0
  int64_t rows;               // rows to transpose (columns of dst)
  int C;
  int64_t ld_src, ld_dst;
  const int32_t* grp_row;     // [G] first row of each group, or nullptr: rows < n_valid valid
  const int32_t* counts;      // [G - has_shared] rows of each routed group
  int G, has_shared, T;       // the shared group (group 0 when has_shared) holds T rows
  int64_t n_valid;
};

__device__ __forceinline__ bool masked_row_valid(const MaskedTransposeArgs& a, int64_t r) {
  if (!a.grp_row) return r < a.n_valid;
  int lo = 0, hi = a.G - 1;   // the last group starting at or before r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.grp_row + mid) <= r) lo = mid;
    else hi = mid - 1;
  }
  const int64_t n = (a.has_shared && lo == 0) ? a.T : __ldg(a.counts + lo - a.has_shared);
  return r - __ldg(a.grp_row + lo) < n;
}

// 64 x 64 tiles, 16-byte vectors both ways: 256 threads load the tile's 64 source rows
// (eight vectors each, coalesced) into shared memory, where each 128-byte row stores its
// vectors XOR-permuted by (row / 8) mod 8, then write 64 destination rows of eight vectors,
// each vector gathering one column of eight source rows; eight consecutive threads write one
// destination row's 128 bytes, and the gathers of a warp hit distinct banks.  A CTA takes
// kMtColTiles column tiles of one row tile: the rows' validity (a binary search over the
// groups per row) is looked up once, and each next tile's loads are in flight while the
// current tile is stored.  C and the strides must be multiples of 8 elements (the library's
// widths are multiples of 64).
constexpr int kMtTile = 64;
constexpr int kMtColTiles = 8;
static __global__ void __launch_bounds__(256) masked_transpose_kernel(MaskedTransposeArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ __align__(16) __nv_bfloat16 tile[kMtTile][kMtTile];
  __shared__ bool valid[kMtTile];
  const int64_t r0 = (int64_t)blockIdx.y * kMtTile;
  const int t = threadIdx.x;
  if (t < kMtTile) valid[t] = r0 + t < a.rows && masked_row_valid(a, r0 + t);
  __syncthreads();
  auto load = [&](int c0, uint4 (&v)[2]) {   // this thread's two source vectors of tile c0
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int row = t / 8 + 32 * i, vec = t % 8;
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (valid[row] && c0 + vec * 8 < a.C)
        v[i] = __ldg(reinterpret_cast<const uint4*>(a.src + (r0 + row) * a.ld_src + c0 + vec * 8));
    }
  };
  int c0 = (int)blockIdx.x * kMtColTiles * kMtTile;
  uint4 v[2];
  if (c0 < a.C) load(c0, v);
  for (int ct = 0; ct < kMtColTiles && c0 < a.C; ++ct, c0 += kMtTile) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int row = t / 8 + 32 * i, vec = t % 8;
      *reinterpret_cast<uint4*>(&tile[row][(vec ^ ((row >> 3) & 7)) * 8]) = v[i];
    }
    __syncthreads();
    if (ct + 1 < kMtColTiles && c0 + kMtTile < a.C) load(c0 + kMtTile, v);   // next tile in flight
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = t / 8 + 32 * i, rv = t % 8;   // destination row c0 + c, vector rv
      if (c0 + c >= a.C || r0 + rv * 8 >= a.rows) continue;
      const int ch = ((c >> 3) ^ rv) * 8 + (c & 7);   // column c of source rows 8 rv .. 8 rv + 7
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat16 lo = tile[rv * 8 + 2 * j][ch], hi = tile[rv * 8 + 2 * j + 1][ch];
        w[j] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
      }
      *reinterpret_cast<uint4*>(a.dst + (int64_t)(c0 + c) * a.ld_dst + r0 + rv * 8) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();   // the tile buffer is refilled next turn
  }
}

}  // namespace moe
