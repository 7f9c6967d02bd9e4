// scan.cuh -- per-expert totals, padded group offsets, grouped-GEMM tile tables and the
// balance loss, from the router tiles' histograms and affinity sums.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Top-k routing, from affinities to gates":
// a production layer groups the tokens of each expert so that every expert runs one dense
// GEMM chain over its rows; the scan turns the router's per-tile histograms into the
// expert_counts output, each expert's first (padded) row, the first destination row of every
// (tile, expert) and the tile tables of both grouped GEMMs.  It also finishes the
// expert-level balance loss of the "Expert-level balance loss" section,
// aux = alpha_1 * sum_i (count_i / T) * (psum_i / T).  Every sum runs in a fixed order, so the
// results do not depend on scheduling.
//
// It runs as a kernel of its own, one CTA of 1024 threads, launched right after the router
// (programmatic dependent launch hides its launch); the expert-parallel layout kernel runs
// the same scan over received blocks.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kMaxTopK = 16;
constexpr int kMaxRouted = 256;
constexpr int kScanThreads = 1024;  // threads that run scan_tail (one CTA)

struct ScanArgs {
  const int32_t* tile_hist;   // [n_tiles, n_routed]
  const float* tile_psum;     // [n_tiles, n_routed], or nullptr (no affinity sums: the
                              // expert-parallel layout scan, which also has no loss output)
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
  int32_t* ts3;               // [G + 1] tile prefix of a GEMM with N = the group's
                              // intermediate width at bn2 columns per tile (the backward's
                              // dHmid GEMM), or nullptr
  // Routed-row indices (decode-sized layers, whose decode FFN kernel copies the token rows
  // itself): with slot_row != nullptr the scan ends by placing every (token, slot) —
  // slot_row[t, k] = its destination row, row_tok[row] = t — as the permute would.
  const int32_t* topk_idx;    // [T, top_k]
  const int32_t* topk_rank;   // [T, top_k]
  int32_t* slot_row;          // [T, top_k], or nullptr
  int32_t* row_tok;           // [rows_cap]
  int top_k, router_rows, rows_cap;
  int* err;
  int n_sync;                 // counters at copy_done to zero (0: one)
};

struct ScanSmem {
  int32_t cnt[kScanThreads];
  float ps[kScanThreads];
  int32_t base[kScanThreads];
  int32_t off[kMaxRouted];
  int32_t w_off[kScanThreads / 32], w_t1[kScanThreads / 32], w_t2[kScanThreads / 32];
  int32_t w_t3[kScanThreads / 32];
  double aux[kMaxRouted];
  float ps_tot[kMaxRouted];   // per-expert affinity totals (step 2), read again in step 3
};

constexpr int kScanBatch = 16;  // independent loads in flight per thread

// The kScanThreads threads of one CTA; `sync()` synchronises them.  The tiles' histograms
// and sums were written by the previous kernel; they are read through L2.
template <class Sync>
__device__ void scan_tail(const ScanArgs& a, int tid, uint8_t* smem, Sync sync) {
  ScanSmem& S = *reinterpret_cast<ScanSmem*>(smem);
  const int nr = a.n_routed;
  int nseg = kScanThreads / nr;
  if (nseg > a.n_tiles) nseg = a.n_tiles;
  if (nseg < 1) nseg = 1;
  const int seg_len = (a.n_tiles + nseg - 1) / nseg;
  const int e = tid % nr, seg = tid / nr;
  const bool active = seg < nseg;
  const int t0 = seg * seg_len;
  const int t1 = min(a.n_tiles, t0 + seg_len);
  if (a.copy_done)
    for (int i = tid; i < (a.n_sync > 1 ? a.n_sync : 1); i += kScanThreads) a.copy_done[i] = 0;

  // 1. per-segment sums, tiles in ascending order (loads batched, adds in order); a
  //    segment of at most kScanBatch tiles keeps its histogram entries for step 4
  int hkeep[kScanBatch];
  const bool keep = t1 - t0 <= kScanBatch;
  if (active) {
    int c = 0;
    float p = 0.f;
    for (int tb = t0; tb < t1; tb += kScanBatch) {
      int hv[kScanBatch];
      float pv[kScanBatch];
#pragma unroll
      for (int j = 0; j < kScanBatch; ++j) {
        const bool in = tb + j < t1;
        hv[j] = in ? __ldcg(a.tile_hist + (size_t)(tb + j) * nr + e) : 0;
        pv[j] = in && a.tile_psum ? __ldcg(a.tile_psum + (size_t)(tb + j) * nr + e) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kScanBatch; ++j) {
        if (tb + j < t1) {
          c += hv[j];
          p += pv[j];
        }
        hkeep[j] = hv[j];   // (the first and, when kept, only batch)
      }
    }
    S.cnt[tid] = c;
    S.ps[tid] = p;
  }
  sync();
  // 2. per expert: segment bases, totals
  if (tid < nr) {
    int run = 0;
    float ps = 0.f;
    for (int s = 0; s < nseg; ++s) {
      S.base[s * nr + tid] = run;
      run += S.cnt[s * nr + tid];
      ps += S.ps[s * nr + tid];
    }
    a.expert_counts[tid] = run;
    if (a.psum_total) a.psum_total[tid] = ps;
    S.ps_tot[tid] = ps;
    S.off[tid] = run;   // count for now, offset after step 3
  }
  sync();
  // 3. expert offsets (padded to the GEMM row tile), tile tables, balance loss: inclusive
  //    scans over the experts (shuffles within a warp, then over warp totals) and a
  //    fixed-shape tree sum for the loss
  {
    const int lane = tid & 31, wid = tid >> 5;
    const int nt1 = (a.inter + a.bn1 - 1) / a.bn1;
    const int nt2 = (a.d + a.bn2 - 1) / a.bn2;
    const int sh_mt = !a.has_shared ? 0 : a.tile_rows > 0 ? (a.T + a.tile_rows - 1) / a.tile_rows : 1;
    const int sh_t1 = sh_mt * ((a.inter_shared + a.bn1 - 1) / a.bn1);
    const int sh_t2 = sh_mt * nt2;
    const int nt3 = (a.inter + a.bn2 - 1) / a.bn2;
    const int sh_t3 = sh_mt * ((a.inter_shared + a.bn2 - 1) / a.bn2);
    int pad = 0, t1c = 0, t2c = 0, t3c = 0;
    if (tid < nr) {
      const int cnt = S.off[tid];
      const int mt = a.tile_rows > 0 ? (cnt + a.tile_rows - 1) / a.tile_rows : (cnt > 0 ? 1 : 0);
      pad = (cnt + a.bm - 1) / a.bm * a.bm;
      t1c = mt * nt1;
      t2c = mt * nt2;
      t3c = mt * nt3;
      const double invT = 1.0 / (double)a.T;
      S.aux[tid] = a.psum_total ? ((double)cnt * invT) * ((double)S.ps_tot[tid] * invT) : 0.0;
    } else if (tid < kMaxRouted) {
      S.aux[tid] = 0.0;
    }
    int ip = pad, i1 = t1c, i2 = t2c, i3 = t3c;   // inclusive scans within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int xp = __shfl_up_sync(0xffffffffu, ip, o);
      const int x1 = __shfl_up_sync(0xffffffffu, i1, o);
      const int x2 = __shfl_up_sync(0xffffffffu, i2, o);
      const int x3 = __shfl_up_sync(0xffffffffu, i3, o);
      if (lane >= o) { ip += xp; i1 += x1; i2 += x2; i3 += x3; }
    }
    if (lane == 31) { S.w_off[wid] = ip; S.w_t1[wid] = i1; S.w_t2[wid] = i2; S.w_t3[wid] = i3; }
    sync();
    int bp = 0, b1 = 0, b2 = 0, b3 = 0;
    for (int w2 = 0; w2 < wid; ++w2) {
      bp += S.w_off[w2]; b1 += S.w_t1[w2]; b2 += S.w_t2[w2]; b3 += S.w_t3[w2];
    }
    if (tid < nr) {
      const int g = a.has_shared + tid;
      const int off = bp + ip - pad;            // exclusive prefix of the padded sizes
      a.grp_row[g] = off;
      a.ts1[g + 1] = sh_t1 + b1 + i1;
      a.ts2[g + 1] = sh_t2 + b2 + i2;
      if (a.ts3) a.ts3[g + 1] = sh_t3 + b3 + i3;
    }
    if (tid == 0) {
      a.ts1[0] = 0;
      a.ts2[0] = 0;
      if (a.ts3) a.ts3[0] = 0;
      if (a.has_shared) {
        a.grp_row[0] = 0;
        a.ts1[1] = sh_t1;
        a.ts2[1] = sh_t2;
        if (a.ts3) a.ts3[1] = sh_t3;
      }
    }
    sync();   // every thread has read S.off (as a count) before it becomes the offset
    if (tid < nr) S.off[tid] = bp + ip - pad;
    // loss: pairwise tree over 256 slots, always the same shape
    for (int stride = kMaxRouted / 2; stride > 0; stride >>= 1) {
      sync();
      if (tid < stride) S.aux[tid] += S.aux[tid + stride];
    }
    if (tid == 0 && a.aux_loss) *a.aux_loss = (float)((double)a.alpha1 * S.aux[0]);
  }
  sync();
  // 4. destination base of every (tile, expert)
  if (active) {
    int run = S.off[e] + S.base[tid];
    for (int tb = t0; tb < t1; tb += kScanBatch) {
      int hv[kScanBatch];
#pragma unroll
      for (int j = 0; j < kScanBatch; ++j)
        hv[j] = keep ? hkeep[j] : tb + j < t1 ? __ldcg(a.tile_hist + (size_t)(tb + j) * nr + e) : 0;
#pragma unroll
      for (int j = 0; j < kScanBatch; ++j) {
        if (tb + j < t1) {
          a.tile_base[(size_t)(tb + j) * nr + e] = run;
          run += hv[j];
        }
      }
    }
  }
  // 5. (decode-sized layers) the destination row of every (token, slot) and the token of
  //    every destination row
  if (a.slot_row) {
    sync();   // the tile bases above, written by other threads
    const int n = a.T * a.top_k;
    for (int idx = tid; idx < n; idx += kScanThreads) {
      const int t = idx / a.top_k;
      const int ex = a.topk_idx[idx];
      int dst = -1;
      if (ex >= 0 && ex < nr) {
        dst = a.tile_base[(size_t)(t / a.router_rows) * nr + ex] + a.topk_rank[idx];
        if (dst < 0 || dst >= a.rows_cap) {
          record_error(a.err, kErrPermuteRow);
          dst = -1;
        }
      } else {
        record_error(a.err, kErrRouteIndex);
      }
      a.slot_row[idx] = dst < 0 ? 0 : dst;
      if (dst >= 0) a.row_tok[dst] = t;
    }
  }
}

// One CTA of kScanThreads threads, launched after the router.
static __global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(ScanArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ __align__(16) uint8_t smem[sizeof(ScanSmem)];
  scan_tail(a, threadIdx.x, smem, [] { __syncthreads(); });
}

}  // namespace moe
