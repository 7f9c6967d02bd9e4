// gemm_tc.cuh -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, 2-SM).
//
// The expert FFN is SwiGLU, FFN(x) = W_down (SiLU(W_gate x) * (W_up x)) (the GLU-variant
// FFN cited by the observer.broadside.tech card; the DeepSeekMoE pages only say "FFN").
// Following the DeepSeekMoE (deepforge.srivtx.xyz) article, "Top-k routing, from
// affinities to gates", the tokens of each expert are grouped and each expert runs one
// dense GEMM chain over its rows; the K_s shared experts ("Where this sits", shared
// expert isolation) form one extra always-on group whose intermediate width is K_s * I
// (fine-grained segmentation makes the sum of K_s experts the same computation as one
// expert K_s times as wide).
//
//   mode kGateUpSwiGLU:  Hmid[r, :] = SiLU(X W_gate^T) * (X W_up^T)      (K = d)
//   mode kDown:          Y[r, :]    = Hmid W_down^T                        (K = I_g; with
//                        e4m3 operands, scaled by the A row's and W_down row's scales)
//                        (also any plain D = A B^T with a bf16 output: the backward's
//                        dHmid = dY W_down and dX = [da db] [W_gate; W_up] products)
//   mode kGateUpBwd:     the gate/up products recomputed, a = X W_gate^T, b = X W_up^T, and
//                        with the incoming dHmid the SwiGLU backward in the epilogue:
//                        da = dHmid * b * SiLU'(a), db = dHmid * SiLU(a), stored interleaved
//                        like the gate/up weight rows (K = d)
//   mode kWgrad:         weight gradients dW[g] = A_g B_g^T with K = the group's (padded)
//                        rows: A and B are transposed activations [width, rows] read at the
//                        group's row offset; fp32 outputs, one matrix per group, gate/up rows
//                        de-interleaved on the way out
//
// Design: persistent clusters of two CTAs (one per SM); each cluster computes 256 x 256
// output tiles with the paired-SM MMA (tcgen05.mma.cta_group::2, M = 256, N = 256,
// K = 16): CTA r of the pair stages rows [128 r, 128 r + 128) of the A tile and rows
// [128 r, 128 r + 128) of the B tile, so each SM holds half of B and the MMA reads both
// SMs' shared memory.  448 threads per CTA (640 for the e4m3 gate/up GEMM):
//   warp 0      one thread issues the TMA loads of this CTA's halves (128 rows x 128
//               bytes each per k-block, 128-byte swizzle) into a ring of 3 stages of two
//               k-blocks; completion is counted on the leader CTA's "full" barrier (the
//               leader expects both CTAs' bytes);
//   warp 1      allocates 512 TMEM columns in both CTAs (two 256-column fp32
//               accumulators); in the leader one thread issues the MMAs and commits with a
//               multicast arrive to both CTAs' "empty" / "accumulator full" barriers;
//   warps 2..9  epilogue in both CTAs (warps 2..17 for e4m3): tcgen05.ld of the CTA's
//               128 accumulator rows (one TMEM lane per output row; two warps per lane
//               quadrant, each taking half of the columns, or four for e4m3), SiLU(gate)*up
//               in fp32 or a plain convert, bf16 stores; one arrive per warp on the
//               leader's "accumulator empty" barrier;
//   4 warps     after the epilogue warps: the fused row copy of the gate/up GEMM (idle
//               when there is none).
// Gate/up weight rows are interleaved in blocks of 64 (64 gate rows, then the 64 matching
// up rows), so a 256-row B tile yields 128 Hmid columns.  Tiles are enumerated group by
// group (row block major, column block minor) and handed out round-robin over clusters.
// No load uses multicast.
#pragma once

#include "scan_permute.cuh"

namespace moe {

constexpr int kPairBM = 256;                 // output rows per cluster tile (128 per CTA)
constexpr int kGemmBN = 256;                 // output columns (B rows) per tile
constexpr int kGemmBK = 64;                  // k-block (one 128-byte swizzle row of bf16)
// A stage carries two k-blocks: the MMA issuer's wait on a stage (and the producer's)
// costs a few hundred cycles of issue latency, which two k-blocks of MMAs hide better
// than one.  Three such stages keep the same bytes in flight as six single ones.
constexpr int kGemmKPS = 2;
constexpr int kGemmStages = 3;
constexpr int kGemmEpiWarps = 8;             // two warps per TMEM lane quadrant
constexpr int kGemmCopyWarps = 4;            // row copies of the fused permute (gate/up GEMM)
constexpr int kGemmThreads = 64 + 32 * (kGemmEpiWarps + kGemmCopyWarps);
// The e4m3 gate/up GEMM finishes a tile's MMAs in half the time, so its SwiGLU epilogue
// (which also applies the row scales) gets twice the warps: four per TMEM lane quadrant,
// working in steps of 16 outputs to stay within the smaller register budget.
__host__ __device__ constexpr int gemm_epi_warps(bool f8) { return f8 ? 16 : kGemmEpiWarps; }
__host__ __device__ constexpr int gemm_threads(bool f8) {
  return 64 + 32 * (gemm_epi_warps(f8) + kGemmCopyWarps);
}
constexpr uint32_t kGemmABytes = 128 * kGemmBK * 2;           // this CTA's half of A, per k-block
constexpr uint32_t kGemmBBytes = (kGemmBN / 2) * kGemmBK * 2; // this CTA's half of B, per k-block
constexpr uint32_t kGemmBOff = kGemmKPS * kGemmABytes;        // B blocks after the A blocks
constexpr uint32_t kGemmStageBytes = kGemmKPS * (kGemmABytes + kGemmBBytes);
constexpr uint32_t kGemmTmemCols = 512;
constexpr size_t kGemmSmemBytes = 1024 + (size_t)kGemmStages * kGemmStageBytes + 256;

enum GemmMode : int { kGateUpSwiGLU = 0, kDown = 1, kGateUpBwd = 2, kWgrad = 3 };

// bf16 outputs are written 32 bytes per thread (st.global.v8): out_* must be 32-byte aligned
// and ld_* a multiple of 16 elements (the library's buffers: cudaMalloc'd, d and the
// intermediate widths multiples of 64).
struct GemmArgs {
  const int32_t* grp_row;   // [G] first row of the group in A (and in the output)
  const int32_t* ts;        // [G + 1] tile prefix (256-row tiles)
  int G, has_shared;
  int kb_shared, kb_routed; // K / 64 of the shared group and of a routed group
  int nt_shared, nt_routed; // column tiles per group
  __nv_bfloat16* out_shared;
  int64_t ld_shared, rows_shared;
  int cols_shared;
  __nv_bfloat16* out_routed;
  int64_t ld_routed, rows_routed;
  int cols_routed;
  int* err;
  // Fused permute (gate/up GEMM with a shared group): the copy warps of every CTA copy the
  // token rows to their expert-contiguous A rows (`perm`) while the shared group's tiles,
  // which read the token matrix itself, run first; each copy warp then adds 1 to
  // *copy_done, and a CTA's producer waits for all gridDim.x * kGemmCopyWarps of them
  // before loading its first routed tile.  copy_done == nullptr: no fused copy.  The
  // wait relies on the whole grid being resident at once (it is sized from the occupancy
  // of this kernel).
  PermuteArgs perm;
  int* copy_done;
  // e4m3 operands (kernel template F8): per-row scales of A (token rows of the shared
  // group, permuted rows of the routed groups) and of B (gate/up weight rows in their
  // interleaved order; routed: sb_routed + e * sb_routed_stride)
  const float* sa_shared;
  const float* sa_routed;
  const float* sb_shared;
  const float* sb_routed;
  int64_t sb_routed_stride;
  // kGateUpBwd: the incoming gradient of the SwiGLU activation, [rows, width] bf16 (shared
  // group: width K_s * I; routed: I); the outputs (out_*) hold [rows, 2 * width]
  const __nv_bfloat16* dh_shared;
  const __nv_bfloat16* dh_routed;
  int64_t ld_dh_shared, ld_dh_routed;
  // kWgrad: K of a routed group = its rows rounded up to wg_bm (counts from the scan), of the
  // shared group kb_shared; output rows_* = M, cols_* = N; fp32 outputs [M, N] per group
  // (routed: + e * wg_stride), or with wg_split the interleaved gate/up rows of M = 2 I
  // split into out0 (gate) and out1 (up), [I, N] each
  const int32_t* wg_counts;
  int wg_bm, wg_split;
  int wg_colsplit;   // > 0: the shared group's output columns are side-by-side
                     // [M, wg_colsplit] matrices (its K_s experts), each after the previous
  float *wg_out0_shared, *wg_out1_shared, *wg_out0_routed, *wg_out1_routed;
  int64_t wg_stride;
  int wg_v8;         // the fp32 outputs are 32-byte aligned: 32-byte stores
};

struct TileCoord {
  int g, m, n, e;
  bool shared;
};

__device__ __forceinline__ void gemm_decode(int tile, int& g, const GemmArgs& a, TileCoord& c) {
  while (tile >= __ldg(&a.ts[g + 1])) ++g;
  const int local = tile - __ldg(&a.ts[g]);
  c.shared = a.has_shared && g == 0;
  const int nt = c.shared ? a.nt_shared : a.nt_routed;
  c.m = local / nt;
  c.n = local - c.m * nt;
  c.e = g - a.has_shared;
  c.g = g;
}

// K-blocks of a tile: fixed per group kind, or (kWgrad, routed groups) the group's rows
// rounded up to wg_bm, / 64 (0 for an expert without rows: the tile is written as zeros).
template <int MODE>
__device__ __forceinline__ int gemm_kblocks(const GemmArgs& a, const TileCoord& c) {
  if (c.shared) return a.kb_shared;
  if constexpr (MODE == kWgrad) {
    const int n = __ldg(a.wg_counts + c.e);
    return (n + a.wg_bm - 1) / a.wg_bm * (a.wg_bm / kGemmBK);
  }
  return a.kb_routed;
}

// F8: A and B are e4m3 (k-blocks of 128 elements = the same 128-byte rows), MMAs of kind
// f8f6f4, and the gate/up epilogue multiplies each accumulator by its two row scales.
template <int MODE, bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_threads(F8), 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA_s,
                       const __grid_constant__ CUtensorMap tmA_r,
                       const __grid_constant__ CUtensorMap tmB_s,
                       const __grid_constant__ CUtensorMap tmB_r, GemmArgs a) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ctl = base + (size_t)kGemmStages * kGemmStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);   // used in the leader
  uint64_t* empty = full + kGemmStages;                 // both CTAs
  uint64_t* acc_full = empty + kGemmStages;             // both CTAs
  uint64_t* acc_empty = acc_full + 2;                   // used in the leader
  uint64_t* drain = acc_empty + 2;                      // both CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();            // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&acc_full[s]), 1);
      mbar_init(smem_u32(&acc_empty[s]), 2 * gemm_epi_warps(F8));   // epilogue warps of both CTAs
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA_s);
    tma_prefetch_desc(&tmA_r);
    tma_prefetch_desc(&tmB_s);
    tma_prefetch_desc(&tmB_r);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kGemmTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();   // the tile tables and operands come from the previous kernels
  const int total = __ldg(&a.ts[a.G]);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0, g = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool rows_ready = a.copy_done == nullptr;
      for (int tile = cid; tile < total && ok; tile += ncl) {
        TileCoord c;
        gemm_decode(tile, g, a, c);
        if (!c.shared && !rows_ready) {
          ok = counter_wait(a.copy_done, (int)gridDim.x * kGemmCopyWarps, abort_flag, a.err,
                            kErrWaitCopy);
          if (!ok) break;
          fence_proxy_async_global();   // the copied rows, seen by the TMA loads below
          rows_ready = true;
        }
        const CUtensorMap* ta = c.shared ? &tmA_s : &tmA_r;
        // weight gradients: rows of A are the output rows, the group's rows are K (at the
        // group's column offset in the transposed routed activations)
        const int kbase = (MODE == kWgrad && !c.shared) ? __ldg(&a.grp_row[c.g]) : 0;
        const int arow = (MODE == kWgrad ? 0 : __ldg(&a.grp_row[c.g])) + c.m * kPairBM + (int)rank * 128;
        const int brow = c.n * kGemmBN + (int)rank * (kGemmBN / 2);
        const int kbn = gemm_kblocks<MODE>(a, c);
        for (int kb0 = 0; kb0 < kbn; kb0 += kGemmKPS) {
          ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.err, kErrWaitProducer);
          if (!ok) break;
          const uint32_t sa = smem_u32(base + (size_t)stage * kGemmStageBytes);
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          const int nk = kbn - kb0 < kGemmKPS ? kbn - kb0 : kGemmKPS;
          if (leader)
            mbar_arrive_expect_tx(smem_u32(&full[stage]), 2u * (uint32_t)nk * (kGemmABytes + kGemmBBytes));
          for (int j = 0; j < nk; ++j) {
            const int kx = kbase + (kb0 + j) * (F8 ? 2 * kGemmBK : kGemmBK);   // elements
            tma_load_2d_pair(sa + j * kGemmABytes, ta, fb, kx, arow);
            if (c.shared || MODE == kWgrad)
              tma_load_2d_pair(sa + kGemmBOff + j * kGemmBBytes, c.shared ? &tmB_s : &tmB_r, fb, kx, brow);
            else tma_load_3d_pair(sa + kGemmBOff + j * kGemmBBytes, &tmB_r, fb, kx, brow, c.e);
          }
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
      }
      // every copy this CTA started has landed once its stage came back empty: wait for
      // the MMAs to release all stages (bounded), so no copy is in flight at exit
      if (ok) {
        for (int s = 0; s < kGemmStages; ++s) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.err, kErrWaitDrain)) break;
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      const uint32_t idesc = F8 ? idesc_e4m3_f32(kPairBM, kGemmBN) : idesc_bf16_f32(kPairBM, kGemmBN);
      int stage = 0, g = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cid; tile < total && ok; tile += ncl, ++it) {
        TileCoord c;
        gemm_decode(tile, g, a, c);
        const int kbn = gemm_kblocks<MODE>(a, c);
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        ok = mbar_wait(smem_u32(&acc_empty[acc]), acc_par ^ 1u, abort_flag, a.err, kErrWaitMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(acc * kGemmBN);
        for (int kb0 = 0; kb0 < kbn; kb0 += kGemmKPS) {
          ok = mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.err, kErrWaitMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(base + (size_t)stage * kGemmStageBytes);
          const int nk = kbn - kb0 < kGemmKPS ? kbn - kb0 : kGemmKPS;
          for (int j = 0; j < nk; ++j) {
            const uint64_t adesc = sdesc_k_sw128(sa + j * kGemmABytes);
            const uint64_t bdesc = sdesc_k_sw128(sa + kGemmBOff + j * kGemmBBytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {   // 32-byte K steps: 16 bf16 or 32 e4m3 values
              if (F8) tc_mma_f8_pair(dt, adesc + 2u * k, bdesc + 2u * k, idesc, (kb0 | j | k) != 0);
              else tc_mma_f16_pair(dt, adesc + 2u * k, bdesc + 2u * k, idesc, (kb0 | j | k) != 0);
            }
          }
          tc_commit_pair_mc(smem_u32(&empty[stage]), 0x3);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit_pair_mc(smem_u32(&acc_full[acc]), 0x3);
      }
      tc_commit_pair_mc(smem_u32(drain), 0x3);
    }
    __syncwarp();
  } else if (warp >= 2 + gemm_epi_warps(F8)) {
    // ------------------------------------------------------------------ row copies
    if (a.copy_done != nullptr) {
      const int nw = (int)gridDim.x * kGemmCopyWarps;
      for (int t = (int)blockIdx.x * kGemmCopyWarps + (warp - 2 - gemm_epi_warps(F8)); t < a.perm.T;
           t += nw)
        permute_token(a.perm, t, lane);
      fence_proxy_async_global();
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(a.copy_done, 1);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    constexpr int WPQ = gemm_epi_warps(F8) / 4;   // epilogue warps per quadrant
    const int part = (warp - 2) >> 2;       // which 1/WPQ of the tile's columns
    const int half = part;                  // (WPQ == 2) which half of the tile's columns
    const int rr = q * 32 + lane;
    int g = 0, it = 0;
    for (int tile = cid; tile < total; tile += ncl, ++it) {
      TileCoord c;
      gemm_decode(tile, g, a, c);
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      // lane 0 polls the accumulator barrier, the other lanes wait in __syncwarp
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait(smem_u32(&acc_full[acc]), acc_par, abort_flag, a.err, kErrWaitEpilogue);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;   // warp-uniform decision
      tc_fence_after();
      const uint32_t trow =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kGemmBN);
      // output row: in the group's rows of A, or (kWgrad) in the gradient matrix itself
      const int64_t orow = (MODE == kWgrad ? 0 : (int64_t)__ldg(&a.grp_row[c.g])) +
                           (int64_t)c.m * kPairBM + (int64_t)rank * 128 + rr;
      __nv_bfloat16* out = c.shared ? a.out_shared : a.out_routed;
      const int64_t ld = c.shared ? a.ld_shared : a.ld_routed;
      const int64_t rows = c.shared ? a.rows_shared : a.rows_routed;
      const int cols = c.shared ? a.cols_shared : a.cols_routed;
      const bool row_ok = orow < rows;
      // (a weight gradient's last row tile may reach past its M rows: those rows are skipped)
      if (!row_ok && MODE != kWgrad) record_error(a.err, kErrOutRow);
      if constexpr (MODE == kWgrad) {
        // fp32 rows of the group's weight gradient; a group without rows gives zeros
        const bool kzero = gemm_kblocks<MODE>(a, c) == 0;
        const int64_t mrow = orow;
        const bool mok = row_ok;
        float* dst = nullptr;
        if (mok) {
          float* o0 = c.shared ? a.wg_out0_shared : a.wg_out0_routed + (int64_t)c.e * a.wg_stride;
          float* o1 = c.shared ? a.wg_out1_shared : a.wg_out1_routed + (int64_t)c.e * a.wg_stride;
          if (a.wg_split) {   // interleaved gate/up rows: blocks of 64, gate first
            const int64_t blk = mrow >> 6;
            dst = ((blk & 1) ? o1 : o0) + ((blk >> 1) * 64 + (mrow & 63)) * (int64_t)cols;
          } else if (c.shared && a.wg_colsplit > 0) {
            dst = o0 + mrow * (int64_t)a.wg_colsplit;   // column c: matrix c / colsplit
          } else {
            dst = o0 + mrow * (int64_t)cols;
          }
        }
#pragma unroll 1
        for (int cc = half * (kGemmBN / 2); cc < (half + 1) * (kGemmBN / 2); cc += 32) {
          const int col = c.n * kGemmBN + cc;
          if (col >= cols) break;
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(trow + static_cast<uint32_t>(cc), v);
          tmem_ld_wait(v);
          if (mok) {
            // (with wg_colsplit, a 32-column chunk never straddles two matrices: the widths
            // are multiples of 64)
            float* dcol = (c.shared && a.wg_colsplit > 0)
                              ? dst + (int64_t)(col / a.wg_colsplit) * rows * a.wg_colsplit + col % a.wg_colsplit
                              : dst + col;
            if (kzero) {
#pragma unroll
              for (int x = 0; x < 32; ++x) v[x] = 0u;
            }
            if (a.wg_v8) {
#pragma unroll
              for (int x = 0; x < 4; ++x)
                st_global_v8(dcol + 8 * x, make_uint4(v[8 * x], v[8 * x + 1], v[8 * x + 2], v[8 * x + 3]),
                             make_uint4(v[8 * x + 4], v[8 * x + 5], v[8 * x + 6], v[8 * x + 7]));
            } else {
              uint4* d4 = reinterpret_cast<uint4*>(dcol);
#pragma unroll
              for (int x = 0; x < 8; ++x) d4[x] = make_uint4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
            }
          }
        }
      } else if constexpr (MODE == kGateUpBwd) {
        // SwiGLU backward on 16 outputs at a time: with a = gate, b = up, s = sigmoid(a),
        // SiLU(a) = a s and SiLU'(a) = s (1 + a (1 - s)); the incoming dHmid of the same
        // outputs is read from global memory; da and db go to the interleaved columns of the
        // accumulator they came from (64 gate columns, then the 64 matching up columns)
        const int hb = half;
        const int col0 = c.n * (kGemmBN / 2) + hb * 64;   // activation column
        const __nv_bfloat16* dhp = (c.shared ? a.dh_shared : a.dh_routed) +
                                   orow * (c.shared ? a.ld_dh_shared : a.ld_dh_routed) + col0;
        const int64_t ocol = (int64_t)c.n * kGemmBN + hb * 128;   // interleaved output column
#pragma unroll 1
        for (int j = 0; j < 64 && col0 < cols; j += 16) {
          uint32_t gv[16], uv[16];
          __syncwarp();
          tmem_ld16(trow + static_cast<uint32_t>(hb * 128 + j), gv);
          tmem_ld16(trow + static_cast<uint32_t>(hb * 128 + 64 + j), uv);
          tmem_ld_wait16(gv);
          tmem_ld_wait16(uv);
          uint4 dv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
          if (row_ok) {
            dv[0] = *reinterpret_cast<const uint4*>(dhp + j);
            dv[1] = *reinterpret_cast<const uint4*>(dhp + j + 8);
          }
          float dh[16];
          bf16x8_to_f32(dv[0], *reinterpret_cast<float(*)[8]>(&dh[0]));
          bf16x8_to_f32(dv[1], *reinterpret_cast<float(*)[8]>(&dh[8]));
          uint32_t pa[8], pb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float da2[2], db2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const float av = __uint_as_float(gv[2 * i + k]);
              const float bv = __uint_as_float(uv[2 * i + k]);
              const float sg = __fdividef(1.0f, 1.0f + __expf(fminf(-av, 80.0f)));
              da2[k] = dh[2 * i + k] * bv * (sg * (1.0f + av * (1.0f - sg)));
              db2[k] = dh[2 * i + k] * (av * sg);
            }
            pa[i] = pack_bf16x2(da2[0], da2[1]);
            pb[i] = pack_bf16x2(db2[0], db2[1]);
          }
          if (row_ok) {
            __nv_bfloat16* orow_p = out + orow * ld + ocol + j;
            st_global_v8(orow_p, make_uint4(pa[0], pa[1], pa[2], pa[3]), make_uint4(pa[4], pa[5], pa[6], pa[7]));
            st_global_v8(orow_p + 64, make_uint4(pb[0], pb[1], pb[2], pb[3]),
                         make_uint4(pb[4], pb[5], pb[6], pb[7]));
          }
        }
      } else if (MODE == kGateUpSwiGLU) {
        float sa = 1.f;                 // e4m3: the A row's scale, and the B rows' scales
        const float* sbv = nullptr;
        if (F8) {
          sa = row_ok ? __ldg((c.shared ? a.sa_shared : a.sa_routed) + orow) : 0.f;
          sbv = (c.shared ? a.sb_shared : a.sb_routed + (int64_t)c.e * a.sb_routed_stride) +
                (int64_t)c.n * kGemmBN;
        }
        if constexpr (!F8) {
          const int hb = half;
          const int col0 = c.n * (kGemmBN / 2) + hb * 64;
#pragma unroll 1
          for (int j = 0; j < 64 && col0 < cols; j += 32) {
            uint32_t gv[32], uv[32];
            __syncwarp();
            tmem_ld32(trow + static_cast<uint32_t>(hb * 128 + j), gv);
            tmem_ld32(trow + static_cast<uint32_t>(hb * 128 + 64 + j), uv);
            tmem_ld_wait(gv);
            tmem_ld_wait(uv);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_fast(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
              const float h1 =
                  silu_fast(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            if (row_ok) {
              __nv_bfloat16* dst = out + orow * ld + col0 + j;
              st_global_v8(dst, make_uint4(pk[0], pk[1], pk[2], pk[3]), make_uint4(pk[4], pk[5], pk[6], pk[7]));
              st_global_v8(dst + 16, make_uint4(pk[8], pk[9], pk[10], pk[11]),
                           make_uint4(pk[12], pk[13], pk[14], pk[15]));
            }
          }
        } else {
          // four warps per quadrant: 32 of the tile's 128 outputs each, 16 per step
          const int hb = part >> 1;
          const int jb = (part & 1) * 32;
          const int col0 = c.n * (kGemmBN / 2) + hb * 64;
          const float* sg = sbv + hb * 128;      // weight-row scales of the gate columns
#pragma unroll 1
          for (int j = jb; j < jb + 32 && col0 < cols; j += 16) {
            uint32_t gv[16], uv[16];
            __syncwarp();
            tmem_ld16(trow + static_cast<uint32_t>(hb * 128 + j), gv);
            tmem_ld16(trow + static_cast<uint32_t>(hb * 128 + 64 + j), uv);
            tmem_ld_wait16(gv);
            tmem_ld_wait16(uv);
            const float4* sg4 = reinterpret_cast<const float4*>(sg + j);
            const float4* su4 = reinterpret_cast<const float4*>(sg + 64 + j);
            uint32_t pk[8];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 a4 = __ldg(sg4 + v), b4 = __ldg(su4 + v);
              const float ga[4] = {a4.x, a4.y, a4.z, a4.w}, ub[4] = {b4.x, b4.y, b4.z, b4.w};
              float hv[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float gg = __uint_as_float(gv[4 * v + i]) * sa * ga[i];
                const float uu = __uint_as_float(uv[4 * v + i]) * sa * ub[i];
                hv[i] = silu_fast(gg) * uu;
              }
              pk[2 * v] = pack_bf16x2(hv[0], hv[1]);
              pk[2 * v + 1] = pack_bf16x2(hv[2], hv[3]);
            }
            if (row_ok)
              st_global_v8(out + orow * ld + col0 + j, make_uint4(pk[0], pk[1], pk[2], pk[3]),
                           make_uint4(pk[4], pk[5], pk[6], pk[7]));
          }
        }
      } else {
        // plain D = A B^T, bf16 out: each of the quadrant's WPQ warps takes kGemmBN / WPQ
        // columns; with e4m3 operands every accumulator is first multiplied by its A row's
        // and B row's scales (16 columns at a time, within the smaller register budget)
        constexpr int CW = kGemmBN / WPQ;
        if constexpr (F8) {
          const float sa = row_ok ? __ldg((c.shared ? a.sa_shared : a.sa_routed) + orow) : 0.f;
          const float* sbv = c.shared ? a.sb_shared : a.sb_routed + (int64_t)c.e * a.sb_routed_stride;
#pragma unroll 1
          for (int cc = part * CW; cc < (part + 1) * CW; cc += 16) {
            const int col = c.n * kGemmBN + cc;
            if (col >= cols) break;
            uint32_t v[16];
            __syncwarp();
            tmem_ld16(trow + static_cast<uint32_t>(cc), v);
            tmem_ld_wait16(v);
            const float4* sb4 = reinterpret_cast<const float4*>(sbv + col);
            uint32_t pk[8];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 b4 = __ldg(sb4 + q4);
              pk[2 * q4] = pack_bf16x2(__uint_as_float(v[4 * q4]) * sa * b4.x,
                                       __uint_as_float(v[4 * q4 + 1]) * sa * b4.y);
              pk[2 * q4 + 1] = pack_bf16x2(__uint_as_float(v[4 * q4 + 2]) * sa * b4.z,
                                           __uint_as_float(v[4 * q4 + 3]) * sa * b4.w);
            }
            if (row_ok)
              st_global_v8(out + orow * ld + col, make_uint4(pk[0], pk[1], pk[2], pk[3]),
                           make_uint4(pk[4], pk[5], pk[6], pk[7]));
          }
        } else {
#pragma unroll 1
          for (int cc = part * CW; cc < (part + 1) * CW; cc += 32) {
            const int col = c.n * kGemmBN + cc;
            if (col >= cols) break;
            uint32_t v[32];
            __syncwarp();
            tmem_ld32(trow + static_cast<uint32_t>(cc), v);
            tmem_ld_wait(v);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (row_ok) {
              __nv_bfloat16* dst = out + orow * ld + col;
              st_global_v8(dst, make_uint4(pk[0], pk[1], pk[2], pk[3]), make_uint4(pk[4], pk[5], pk[6], pk[7]));
              st_global_v8(dst + 16, make_uint4(pk[8], pk[9], pk[10], pk[11]),
                           make_uint4(pk[12], pk[13], pk[14], pk[15]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
    }
  }

  // teardown: all MMAs of the pair have completed before TMEM is released in either CTA
  if (warp == 1 && lane == 0)
    mbar_wait(smem_u32(drain), 0, abort_flag, a.err, kErrWaitDrain);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kGemmTmemCols);
  }
}

}  // namespace moe
