// ep.cuh -- the row movement of the expert-parallel layer: received token rows into the
// local experts' padded groups, and the experts' outputs back into the received order.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Where this sits": the expert-level balance
// loss keeps the experts' loads even and a device-level one keeps the computation even
// "across devices" -- the experts of a layer are spread over several GPUs.  A rank receives,
// from every source rank s, the rows that s routed to each of this rank's experts e, as one
// block per (s, e) in (s, e) order, each block in the source's token order.  The grouped
// GEMMs want each expert's rows contiguous (and padded to the 256-row paired tile), so the
// layout scan gives block (s, e) its destination: the expert's group start plus the rows
// the earlier sources sent to the same expert; within an expert the rows are then ordered by
// (source rank, source token), which is the global token order when the ranks hold
// consecutive token ranges.
#pragma once

#include "scan.cuh"

namespace moe {

struct EpLayoutArgs {
  const int32_t* recv_counts;   // [world, n_local] rows block (s, e) brings
  int world, n_local;
  int32_t* recv_off;            // [world * n_local + 1] first received row of block (s, e)
  ScanArgs scan;                // tile_hist = recv_counts (tiles = source ranks)
};

// One CTA of kScanThreads threads (world * n_local <= 256 blocks): the blocks' offsets in the
// received buffer (an exclusive prefix in (s, e) order), then the group layout of the local
// experts (scan_tail: group starts, tile tables, each block's destination row).
static __global__ void __launch_bounds__(kScanThreads, 1) ep_layout_kernel(EpLayoutArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ __align__(16) uint8_t smem[sizeof(ScanSmem)];
  __shared__ int32_t warp_tot[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nb = a.world * a.n_local;
  const int c = tid < nb ? __ldg(a.recv_counts + tid) : 0;
  int inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += x;
  }
  if (lane == 31) warp_tot[wid] = inc;
  __syncthreads();
  int base = 0;
  for (int w2 = 0; w2 < wid; ++w2) base += warp_tot[w2];
  if (tid < nb) a.recv_off[tid] = base + inc - c;
  if (tid == nb - 1) a.recv_off[nb] = base + inc;
  __syncthreads();
  scan_tail(a.scan, tid, smem, [] { __syncthreads(); });
}

struct EpMoveArgs {
  const uint8_t* src;         // gather: received rows; scatter: expert outputs
  uint8_t* dst;               // gather: expert-contiguous rows; scatter: rows in received order
  const int32_t* recv_off;    // [nb + 1]
  const int32_t* block_dst;   // [nb] first destination row of block (s, e) (scan's tile_base)
  int32_t* row_map;           // [n_recv] gather writes it, scatter reads it
  int64_t n_recv;
  int nb;
  int row_bytes;              // multiple of 16
  int64_t dst_rows;           // rows of the expert-contiguous buffer (bounds check)
  int* err;
  int gather;                 // 1: received -> grouped, 0: grouped -> received order
};

constexpr int kEpMoveWarps = 8;

// One warp per received row j: its block b (the last block starting at or before j; empty
// blocks share their successor's start), its grouped row block_dst[b] + (j - recv_off[b]),
// and a 16-byte-vector copy of the row in the requested direction.
static __global__ void __launch_bounds__(kEpMoveWarps * 32) ep_move_kernel(EpMoveArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t j = (int64_t)blockIdx.x * kEpMoveWarps + (threadIdx.x >> 5);
  if (j >= a.n_recv) return;
  int64_t g;
  if (a.gather) {
    int lo = 0, hi = a.nb - 1;   // largest b with recv_off[b] <= j
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.recv_off + mid) <= j) lo = mid;
      else hi = mid - 1;
    }
    g = (int64_t)__ldg(a.block_dst + lo) + (j - __ldg(a.recv_off + lo));
    if (g < 0 || g >= a.dst_rows) {
      if (lane == 0) record_error(a.err, kErrPermuteRow);
      return;
    }
    if (lane == 0) a.row_map[j] = (int32_t)g;
  } else {
    g = __ldg(a.row_map + j);
    if (g < 0 || g >= a.dst_rows) {
      if (lane == 0) record_error(a.err, kErrPermuteRow);
      return;
    }
  }
  const int nvec = a.row_bytes >> 4;
  const uint4* s = reinterpret_cast<const uint4*>(a.src + (size_t)(a.gather ? j : g) * a.row_bytes);
  uint4* d = reinterpret_cast<uint4*>(a.dst + (size_t)(a.gather ? g : j) * a.row_bytes);
  for (int v = lane; v < nvec; v += 32) d[v] = __ldg(s + v);
}

}  // namespace moe
