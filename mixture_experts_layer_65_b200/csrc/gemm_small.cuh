// gemm_small.cuh -- the expert FFN for small token counts (decode): both grouped GEMMs,
// weights on M, in one persistent kernel (decode_ffn_kernel).
//
// Same FFN as gemm_tc.cuh (SwiGLU experts, K_s shared experts as one always-on group), for
// layers whose groups hold few tokens (every group's token count <= n_tok <= 128).  The
// products are computed transposed, D^T = W X^T, so the MMA's M dimension (128) runs over
// weight rows and its N dimension over the group's tokens: each weight tile is streamed
// from HBM once and the tensor cores do almost no padding work, which makes the kernel a
// weight-streaming one, as a decode step is.  Groups without tokens get no tiles.
//
// A tile is two 128-row weight blocks that share the token operand: per k-block two MMAs
// (M = 128, N = n_tok) write the two halves of one accumulator, columns [0, n_tok) and
// [n_tok, 2 n_tok).
//   mode kGateUpSwiGLU: the gate rows and the up rows of 128 intermediate features (the
//                       interleaved weight layout keeps 64-row gate and up blocks, so each
//                       half is two 64-row loads); TMEM lane L then holds gate and up of
//                       feature L side by side and the SwiGLU needs no exchange.
//   mode kDown:         W_down rows of 256 output features, 128 per half.
// Rows past a group's width (its last tile) are outside the weight tensor map's box range
// and arrive as zeros; their outputs are not stored.
//
// One CTA per SM (persistent), 192 threads: warp 0 issues TMA loads (weights 2 x 128 x 64
// and tokens n_tok x 64, 128-byte swizzle) into a multi-stage ring; warp 1 allocates TMEM
// (two 2 n_tok-column fp32 accumulators) and one thread issues tcgen05.mma; warps 2..5
// drain the accumulator (one TMEM lane = one output feature per thread) and store each
// token's features straight from registers (a warp writes 32 consecutive features, 64
// bytes, per token).  No shared memory besides the ring, so the ring holds as many stages
// as fit: the kernel's speed follows the weight bytes in flight per SM.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

constexpr int kSmallBM = 128;               // weight rows per MMA (M)
constexpr uint32_t kSmallWBytes = kSmallBM * 128u;   // one 128-row weight block per k-block
constexpr int kSmallThreads = 192;
constexpr int kSmallMaxTok = 128;
constexpr int kSmallMaxStages = 8;

// One of the decode FFN kernel's two GEMMs.
struct SmallPhase {
  const int32_t* ts;              // [G + 1] tile prefix (a group has tiles only if it has tokens)
  int kb_shared, kb_routed;       // K / 64
  int cols_shared, cols_routed;   // output features of a group (its tiles cover them in
                                  // steps of 128 (gate/up) or 256 (down))
  __nv_bfloat16* out_shared;
  int64_t ld_shared;
  __nv_bfloat16* out_routed;
  int64_t ld_routed;
};

struct SmallGemmArgs {
  const int32_t* grp_row;   // [G] first token row of each group in the token operands / outputs
  const int32_t* counts;    // [n_routed] tokens of each routed group (shared group: T)
  int G, has_shared, T;
  int n_tok;                // N of the MMA: multiple of 16, >= every group's token count
  int stages;
  SmallPhase ph[2];         // 0: gate/up + SwiGLU -> Hmid, 1: down -> Y
  int* err;
  // Row copy: the epilogue warps, before their first tile, copy token row row_tok[r] of u
  // to row r of xp for every routed row r < n_rows (16-byte vectors, copy_vecs per row),
  // then each adds 1 to sync[0]; a CTA's producer waits for all gridDim.x * 4 of them
  // before loading its first routed token tile (the shared group reads u itself).
  const int32_t* row_tok;
  const __nv_bfloat16* u;
  __nv_bfloat16* xp;
  int n_rows, copy_vecs;
  // Counters, zeroed by the scan: sync[0] the row copies; sync[1 + g] the epilogue warps
  // that have stored group g's activations (four per gate/up tile), which a producer waits
  // for before loading one of g's down tiles.  Both waits rely on the whole grid being
  // resident at once (one CTA per SM, at most one CTA per SM launched).
  int* sync;
};

// smem: stages x (weights 2 x 16 KB + tokens n_tok x 128 B) | barriers
__host__ __device__ constexpr uint32_t small_stage_bytes(int n_tok) {
  return 2u * kSmallWBytes + (((uint32_t)n_tok * 128u + 1023u) & ~1023u);
}
// dynamic shared memory: alignment slack, stage ring, control block
__host__ __device__ constexpr size_t small_smem_bytes(int n_tok, int stages) {
  return 1024 + (size_t)stages * small_stage_bytes(n_tok) + 256;
}
// The ring takes as many stages as the opt-in shared memory holds (at most kSmallMaxStages,
// at least 2): the kernel streams weights, and the more weight bytes it keeps in flight per
// SM the faster it streams them (16B decode: 96 -> 128 KB in flight, 215.1 -> 211.6 us per
// forward).
__host__ __device__ constexpr int small_stages(int n_tok) {
  const long st = ((long)kRouterSmemBudget - (long)small_smem_bytes(n_tok, 0)) / (long)small_stage_bytes(n_tok);
  return st > kSmallMaxStages ? kSmallMaxStages : (st < 2 ? 2 : (int)st);
}
// TMEM columns: two accumulators of 2 n_tok columns, a power of two >= 32
__host__ __device__ constexpr uint32_t small_tmem_cols(int n_tok) {
  return 4u * (uint32_t)n_tok <= 32u ? 32u : 4u * (uint32_t)n_tok <= 64u ? 64u
         : 4u * (uint32_t)n_tok <= 128u ? 128u : 4u * (uint32_t)n_tok <= 256u ? 256u : 512u;
}

// The decode FFN: both GEMMs in one persistent kernel.  The gate/up tiles (phase 0) and then
// the down tiles (phase 1) are handed out round-robin over one list, so the down tiles fill
// the gaps the gate/up tiles leave and the weights stream without a break between the two
// GEMMs.  A down tile of group g waits (bounded) until every gate/up tile of g has stored
// its activations.
static __global__ void __launch_bounds__(kSmallThreads, 1)
decode_ffn_kernel(const __grid_constant__ CUtensorMap tmW0_s, const __grid_constant__ CUtensorMap tmW0_r,
                  const __grid_constant__ CUtensorMap tmX0_s, const __grid_constant__ CUtensorMap tmX0_r,
                  const __grid_constant__ CUtensorMap tmW1_s, const __grid_constant__ CUtensorMap tmW1_r,
                  const __grid_constant__ CUtensorMap tmX1_s, const __grid_constant__ CUtensorMap tmX1_r,
                  SmallGemmArgs a) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = a.stages;
  const int nt = a.n_tok;
  const uint32_t stage_bytes = small_stage_bytes(nt);
  const uint32_t x_bytes = (uint32_t)nt * 128u;
  uint8_t* ctl = base + (size_t)S * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kSmallMaxStages;
  uint64_t* acc_full = empty + kSmallMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tmem_cols = small_tmem_cols(nt);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&acc_full[s]), 1);
      mbar_init(smem_u32(&acc_empty[s]), 4);   // one arrive per epilogue warp
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW0_s);
    tma_prefetch_desc(&tmW0_r);
    tma_prefetch_desc(&tmX0_s);
    tma_prefetch_desc(&tmX0_r);
    tma_prefetch_desc(&tmW1_s);
    tma_prefetch_desc(&tmW1_r);
    tma_prefetch_desc(&tmX1_s);
    tma_prefetch_desc(&tmX1_r);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();   // the tile tables and operands come from the previous kernels
  const int total0 = __ldg(&a.ph[0].ts[a.G]);
  const int total = total0 + __ldg(&a.ph[1].ts[a.G]);

  // position -> (phase, group g, weight tile m of the group, routed expert e, shared?);
  // each role walks its positions in increasing order with a group cursor that restarts
  // when the phase changes
  struct Cursor { int phase = 0, g = 0; };
  auto decode = [&](int pos, Cursor& cu, int& m, int& e, bool& sh) {
    const int ph = pos < total0 ? 0 : 1;
    if (ph != cu.phase) { cu.phase = ph; cu.g = 0; }
    const int tile = ph ? pos - total0 : pos;
    const int32_t* ts = a.ph[ph].ts;
    while (cu.g < a.G - 1 && tile >= __ldg(&ts[cu.g + 1])) ++cu.g;
    m = tile - __ldg(&ts[cu.g]);
    sh = a.has_shared && cu.g == 0;
    e = cu.g - a.has_shared;
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      Cursor cu;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      bool rows_ready = false;
      for (int pos = blockIdx.x; pos < total && ok; pos += gridDim.x) {
        int m, e;
        bool sh;
        decode(pos, cu, m, e, sh);
        const int ph = cu.phase, g = cu.g;
        if (ph == 0 && !sh && !rows_ready) {   // the routed token rows, copied by the epilogue warps
          ok = counter_wait(a.sync, (int)gridDim.x * 4, abort_flag, a.err, kErrWaitCopy);
          if (!ok) break;
          fence_proxy_async_global();   // the copied rows, seen by the TMA loads below
          rows_ready = true;
        }
        if (ph == 1) {   // the group's activations, stored by the epilogues of its gate/up tiles
          const int need = 4 * (__ldg(&a.ph[0].ts[g + 1]) - __ldg(&a.ph[0].ts[g]));
          ok = counter_wait(a.sync + 1 + g, need, abort_flag, a.err, kErrWaitHidden);
          if (!ok) break;
          fence_proxy_async_global();
        }
        const CUtensorMap* tw = ph == 0 ? (sh ? &tmW0_s : &tmW0_r) : (sh ? &tmW1_s : &tmW1_r);
        const CUtensorMap* tx = ph == 0 ? (sh ? &tmX0_s : &tmX0_r) : (sh ? &tmX1_s : &tmX1_r);
        const int xrow = sh ? 0 : __ldg(&a.grp_row[g]);
        const int kbn = sh ? a.ph[ph].kb_shared : a.ph[ph].kb_routed;
        for (int kb = 0; kb < kbn; ++kb) {
          ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.err, kErrWaitProducer);
          if (!ok) break;
          const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, 2u * kSmallWBytes + x_bytes);
          // weight halves: gate/up -- half 0 the gate rows, half 1 the up rows of features
          // [128 m, 128 m + 128), each from the 64-row blocks 2m and 2m + 1 of the
          // interleaved layout (rows 256 m + 128 h + 64 half); down -- rows 256 m + 128 half
          for (int half = 0; half < 2; ++half) {
            for (int h = 0; h < (ph == 0 ? 2 : 1); ++h) {
              const uint32_t dst = sa + (uint32_t)half * kSmallWBytes + (uint32_t)h * (kSmallWBytes / 2);
              const int row = ph == 0 ? 256 * m + 128 * h + 64 * half : 256 * m + 128 * half;
              if (sh) tma_load_2d(dst, tw, fb, kb * 64, row);
              else tma_load_3d(dst, tw, fb, kb * 64, row, e);
            }
          }
          tma_load_2d(sa + 2u * kSmallWBytes, tx, fb, kb * 64, xrow);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s))
          mbar_wait(smem_u32(&full[s]), (last_par >> s) & 1u, abort_flag, a.err, kErrWaitDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kSmallBM, nt);
      int stage = 0, it = 0;
      Cursor cu;
      uint32_t phase = 0;
      bool ok = true;
      for (int pos = blockIdx.x; pos < total && ok; pos += gridDim.x, ++it) {
        int m, e;
        bool sh;
        decode(pos, cu, m, e, sh);
        const int kbn = sh ? a.ph[cu.phase].kb_shared : a.ph[cu.phase].kb_routed;
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        ok = mbar_wait(smem_u32(&acc_empty[acc]), acc_par ^ 1u, abort_flag, a.err, kErrWaitMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * 2 * nt);
        for (int kb = 0; kb < kbn; ++kb) {
          ok = mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.err, kErrWaitMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
          const uint64_t a0 = sdesc_k_sw128(sa), a1 = sdesc_k_sw128(sa + kSmallWBytes);
          const uint64_t bdesc = sdesc_k_sw128(sa + 2u * kSmallWBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            tc_mma_f16(dt, a0 + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
            tc_mma_f16(dt + (uint32_t)nt, a1 + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
          }
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit(smem_u32(&acc_full[acc]));
      }
      tc_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, abort_flag, a.err, kErrWaitDrain);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;              // TMEM lane quadrant
    const int L = q * 32 + lane;         // TMEM lane = weight row of each half
    const int et = threadIdx.x - 64;     // 0..127
    {
      // the routed token rows, one warp per row (eight 16-byte vectors per lane in flight)
      constexpr int kV = 8;
      const int nw = (int)gridDim.x * 4;
      for (int r = (int)blockIdx.x * 4 + (et >> 5); r < a.n_rows; r += nw) {
        const int t = __ldg(a.row_tok + r);
        if (t < 0 || t >= a.T) {
          record_error(a.err, kErrPermuteRow);
          continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a.u + (size_t)t * a.copy_vecs * 8);
        uint4* dst = reinterpret_cast<uint4*>(a.xp + (size_t)r * a.copy_vecs * 8);
        for (int v0 = 0; v0 < a.copy_vecs; v0 += 32 * kV) {
          uint4 buf[kV];
#pragma unroll
          for (int j = 0; j < kV; ++j) {
            const int v = v0 + j * 32 + lane;
            if (v < a.copy_vecs) buf[j] = __ldg(src + v);
          }
#pragma unroll
          for (int j = 0; j < kV; ++j) {
            const int v = v0 + j * 32 + lane;
            if (v < a.copy_vecs) dst[v] = buf[j];
          }
        }
      }
      fence_proxy_async_global();
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(a.sync, 1);
    }
    int it = 0;
    Cursor cu;
    for (int pos = blockIdx.x; pos < total; pos += gridDim.x, ++it) {
      int m, e;
      bool sh;
      decode(pos, cu, m, e, sh);
      const int ph = cu.phase;
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&acc_full[acc]), acc_par, abort_flag, a.err, kErrWaitEpilogue);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;   // warp-uniform decision
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)(acc * 2 * nt);
      const SmallPhase& P = a.ph[ph];
      const int rows = sh ? a.T : __ldg(&a.counts[e]);
      const int64_t row0 = sh ? 0 : __ldg(&a.grp_row[cu.g]);
      __nv_bfloat16* out = sh ? P.out_shared : P.out_routed;
      const int64_t ld = sh ? P.ld_shared : P.ld_routed;
      const int cols = sh ? P.cols_shared : P.cols_routed;
      // this thread's output features: gate/up -- feature 128 m + L (gate in the first half
      // of the accumulator, up in the second); down -- 256 m + L and 256 m + 128 + L
      const int f0 = (ph == 0 ? 128 : 256) * m + L;
      const int f1 = f0 + 128;
      for (int c = 0; c < rows; c += 16) {
        uint32_t v0[16], v1[16];
        __syncwarp();
        tmem_ld16(trow + (uint32_t)c, v0);
        tmem_ld16(trow + (uint32_t)(nt + c), v1);
        tmem_ld_wait16(v0);
        tmem_ld_wait16(v1);
        __nv_bfloat16* o = out + (row0 + c) * ld;
        const int nj = rows - c < 16 ? rows - c : 16;
        if (ph == 0) {
          if (f0 < cols) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < nj)
                o[(int64_t)j * ld + f0] = __float2bfloat16_rn(silu_fast(__uint_as_float(v0[j])) *
                                                              __uint_as_float(v1[j]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < nj) {
              if (f0 < cols) o[(int64_t)j * ld + f0] = __float2bfloat16_rn(__uint_as_float(v0[j]));
              if (f1 < cols) o[(int64_t)j * ld + f1] = __float2bfloat16_rn(__uint_as_float(v1[j]));
            }
          }
        }
      }
      tc_fence_before();
      if (ph == 0) {   // the group's activations, for the TMA loads of its down tiles
        fence_proxy_async_global();
        __threadfence();
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&acc_empty[acc]));
        if (ph == 0) atomicAdd(a.sync + 1 + cu.g, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace moe
