// scan_permute.cuh -- expert-contiguous regrouping of the routed token rows.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Top-k routing, from affinities to gates":
// a production layer groups the tokens of each expert so that every expert runs one
// dense GEMM chain over its rows.  The scan turns the router's per-tile histograms into
// per-expert totals (the expert_counts output), padded expert offsets, per-(tile, expert)
// destination bases and the grouped-GEMM tile tables; it also finishes the expert-level
// balance loss of the "Expert-level balance loss" section,
// aux = alpha_1 * sum_i (count_i / T) * (psum_i / T).  The permute kernel then copies each
// token row to its top_k destinations (order inside an expert = ascending token id).
#pragma once

#include "router.cuh"

namespace moe {

constexpr int kScanThreads = 1024;

struct ScanArgs {
  const int32_t* tile_hist;   // [n_tiles, n_routed]
  const float* tile_psum;     // [n_tiles, n_routed]
  int n_tiles, n_routed, T;
  int has_shared;             // group 0 = all shared experts as one group
  int inter_shared, inter, d; // widths of the shared group and of a routed expert
  int bm;                     // each group's rows are padded to a multiple of bm
  int tile_rows;              // rows per GEMM row tile; 0 = one tile per non-empty group
  int bn1, bn2;               // output columns per tile of the gate/up and down GEMMs
  float alpha1;
  // outputs
  int32_t* expert_counts;     // [n_routed]
  float* aux_loss;            // [1]
  float* psum_total;          // [n_routed]  sum_t s[t, i]
  int32_t* tile_base;         // [n_tiles, n_routed] first destination row of (tile, e)
  int32_t* grp_row;           // [G] first row of each group in its A matrix
  int32_t* ts1;               // [G + 1] tile prefix of the gate/up GEMM
  int32_t* ts2;               // [G + 1] tile prefix of the down GEMM
  int32_t* copy_done;         // counter of the fused GEMM's copy warps, zeroed here; or nullptr
};

static __global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(ScanArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int32_t s_cnt[kScanThreads];
  __shared__ float s_ps[kScanThreads];
  __shared__ int32_t s_base[kScanThreads];
  __shared__ int32_t s_off[kMaxRouted];
  const int nr = a.n_routed;
  int nseg = kScanThreads / nr;
  if (nseg > a.n_tiles) nseg = a.n_tiles;
  if (nseg < 1) nseg = 1;
  const int seg_len = (a.n_tiles + nseg - 1) / nseg;
  const int tid = threadIdx.x;
  const int e = tid % nr, seg = tid / nr;
  const bool active = seg < nseg;
  const int t0 = seg * seg_len;
  const int t1 = min(a.n_tiles, t0 + seg_len);
  if (tid == 0 && a.copy_done) *a.copy_done = 0;

  // 1. per-segment sums (tiles in ascending order)
  if (active) {
    int c = 0;
    float p = 0.f;
    for (int t = t0; t < t1; ++t) {
      c += a.tile_hist[(size_t)t * nr + e];
      p += a.tile_psum[(size_t)t * nr + e];
    }
    s_cnt[tid] = c;
    s_ps[tid] = p;
  }
  __syncthreads();
  // 2. per expert: segment bases, totals, padded sizes
  if (tid < nr) {
    int run = 0;
    float ps = 0.f;
    for (int s = 0; s < nseg; ++s) {
      s_base[s * nr + tid] = run;
      run += s_cnt[s * nr + tid];
      ps += s_ps[s * nr + tid];
    }
    a.expert_counts[tid] = run;
    a.psum_total[tid] = ps;
    s_off[tid] = run;   // count for now, offset after step 3
  }
  __syncthreads();
  // 3. expert offsets (padded to the GEMM row tile), tile tables, balance loss: inclusive
  //    scans over the experts (shuffles within a warp, then over warp totals) and a
  //    fixed-shape tree sum for the loss, so the result does not depend on scheduling
  {
    __shared__ int w_off[kScanThreads / 32], w_t1[kScanThreads / 32], w_t2[kScanThreads / 32];
    __shared__ double s_aux[kMaxRouted];
    const int lane = tid & 31, wid = tid >> 5;
    const int nt1 = (a.inter + a.bn1 - 1) / a.bn1;
    const int nt2 = (a.d + a.bn2 - 1) / a.bn2;
    const int sh_mt = !a.has_shared ? 0 : a.tile_rows > 0 ? (a.T + a.tile_rows - 1) / a.tile_rows : 1;
    const int sh_t1 = sh_mt * ((a.inter_shared + a.bn1 - 1) / a.bn1);
    const int sh_t2 = sh_mt * nt2;
    int cnt = 0, pad = 0, t1 = 0, t2 = 0;
    if (tid < nr) {
      cnt = s_off[tid];
      const int mt = a.tile_rows > 0 ? (cnt + a.tile_rows - 1) / a.tile_rows : (cnt > 0 ? 1 : 0);
      pad = (cnt + a.bm - 1) / a.bm * a.bm;
      t1 = mt * nt1;
      t2 = mt * nt2;
      const double invT = 1.0 / (double)a.T;
      s_aux[tid] = ((double)cnt * invT) * ((double)a.psum_total[tid] * invT);
    } else if (tid < kMaxRouted) {
      s_aux[tid] = 0.0;
    }
    int ip = pad, i1 = t1, i2 = t2;   // inclusive scans within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int xp = __shfl_up_sync(0xffffffffu, ip, o);
      const int x1 = __shfl_up_sync(0xffffffffu, i1, o);
      const int x2 = __shfl_up_sync(0xffffffffu, i2, o);
      if (lane >= o) { ip += xp; i1 += x1; i2 += x2; }
    }
    if (lane == 31) { w_off[wid] = ip; w_t1[wid] = i1; w_t2[wid] = i2; }
    __syncthreads();
    int bp = 0, b1 = 0, b2 = 0;
    for (int w2 = 0; w2 < wid; ++w2) { bp += w_off[w2]; b1 += w_t1[w2]; b2 += w_t2[w2]; }
    if (tid < nr) {
      const int g = a.has_shared + tid;
      const int off = bp + ip - pad;            // exclusive prefix of the padded sizes
      s_off[tid] = off;                         // read in step 4 after the barrier below
      a.grp_row[g] = off;
      a.ts1[g + 1] = sh_t1 + b1 + i1;
      a.ts2[g + 1] = sh_t2 + b2 + i2;
    }
    if (tid == 0) {
      a.ts1[0] = 0;
      a.ts2[0] = 0;
      if (a.has_shared) {
        a.grp_row[0] = 0;
        a.ts1[1] = sh_t1;
        a.ts2[1] = sh_t2;
      }
    }
    // loss: pairwise tree over 256 slots, always the same shape
    for (int stride = kMaxRouted / 2; stride > 0; stride >>= 1) {
      __syncthreads();
      if (tid < stride) s_aux[tid] += s_aux[tid + stride];
    }
    if (tid == 0) *a.aux_loss = (float)((double)a.alpha1 * s_aux[0]);
  }
  __syncthreads();
  // 4. destination base of every (tile, expert)
  if (active) {
    int run = s_off[e] + s_base[tid];
    for (int t = t0; t < t1; ++t) {
      a.tile_base[(size_t)t * nr + e] = run;
      run += a.tile_hist[(size_t)t * nr + e];
    }
  }
}

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
