// gemm_tc.cuh -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05).
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
//   mode kDown:          Y[r, :]    = Hmid W_down^T                        (K = I_g)
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      one thread issues TMA tile loads (A 128x64, B 256x64 bf16, 128-byte
//               swizzle) into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and one
//               thread issues tcgen05.mma (M=128, N=256, K=16) per 16-wide K step;
//   warps 2..5  epilogue: tcgen05.ld the accumulator rows (one TMEM lane = one output
//               row per thread), apply SiLU(gate)*up in fp32 or convert, store bf16.
// The accumulators are double-buffered so the epilogue of tile i overlaps the MMAs of
// tile i+1.  For the gate/up GEMM the weight rows are interleaved in blocks of 64
// (64 gate rows, then the 64 matching up rows) so one 256-row B tile yields 128 Hmid
// columns.  Tiles are enumerated group by group (row block major, column block minor)
// and handed out round-robin over the CTAs.
#pragma once

#include "scan_permute.cuh"

namespace moe {

constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint32_t kGemmABytes = kGemmBM * kGemmBK * 2;
constexpr uint32_t kGemmBBytes = kGemmBN * kGemmBK * 2;
constexpr uint32_t kGemmStageBytes = kGemmABytes + kGemmBBytes;
constexpr uint32_t kGemmTmemCols = 512;
constexpr size_t kGemmSmemBytes = 1024 + (size_t)kGemmStages * kGemmStageBytes + 256;

enum GemmMode : int { kGateUpSwiGLU = 0, kDown = 1 };

struct GemmArgs {
  const int32_t* grp_row;   // [G] first row of the group in A (and in the output)
  const int32_t* ts;        // [G + 1] tile prefix
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

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA_s,
                       const __grid_constant__ CUtensorMap tmA_r,
                       const __grid_constant__ CUtensorMap tmB_s,
                       const __grid_constant__ CUtensorMap tmB_r, GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ctl = base + (size_t)kGemmStages * kGemmStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kGemmStages;
  uint64_t* acc_full = empty + kGemmStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = __ldg(&a.ts[a.G]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&acc_full[s]), 1);
      mbar_init(smem_u32(&acc_empty[s]), 128);
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
    tmem_alloc(smem_u32(tmem_slot), kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0, g = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileCoord c;
        gemm_decode(tile, g, a, c);
        const CUtensorMap* ta = c.shared ? &tmA_s : &tmA_r;
        const int arow = __ldg(&a.grp_row[c.g]) + c.m * kGemmBM;
        const int brow = c.n * kGemmBN;
        const int kbn = c.shared ? a.kb_shared : a.kb_routed;
        for (int kb = 0; kb < kbn; ++kb) {
          ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.err, kErrWaitProducer);
          if (!ok) break;
          const uint32_t sa = smem_u32(base + (size_t)stage * kGemmStageBytes);
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, kGemmStageBytes);
          tma_load_2d(sa, ta, fb, kb * kGemmBK, arow);
          if (c.shared) tma_load_2d(sa + kGemmABytes, &tmB_s, fb, kb * kGemmBK, brow);
          else tma_load_3d(sa + kGemmABytes, &tmB_r, fb, kb * kGemmBK, brow, c.e);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < kGemmStages; ++s)
        if (issued & (1u << s))
          mbar_wait(smem_u32(&full[s]), (last_par >> s) & 1u, abort_flag, a.err, kErrWaitDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN);
      int stage = 0, g = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        TileCoord c;
        gemm_decode(tile, g, a, c);
        const int kbn = c.shared ? a.kb_shared : a.kb_routed;
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        ok = mbar_wait(smem_u32(&acc_empty[acc]), acc_par ^ 1u, abort_flag, a.err, kErrWaitMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(acc * kGemmBN);
        for (int kb = 0; kb < kbn; ++kb) {
          ok = mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.err, kErrWaitMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(base + (size_t)stage * kGemmStageBytes);
          const uint64_t adesc = sdesc_k_sw128(sa);
          const uint64_t bdesc = sdesc_k_sw128(sa + kGemmABytes);
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)
            tc_mma_f16(dt, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit(smem_u32(&acc_full[acc]));
      }
      tc_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, abort_flag, a.err, kErrWaitDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int rr = q * 32 + lane;
    int g = 0, it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      TileCoord c;
      gemm_decode(tile, g, a, c);
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      const bool ok =
          mbar_wait(smem_u32(&acc_full[acc]), acc_par, abort_flag, a.err, kErrWaitEpilogue);
      if (!__all_sync(0xffffffffu, ok)) break;   // warp-uniform decision
      tc_fence_after();
      const uint32_t trow =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kGemmBN);
      const int64_t orow = (int64_t)__ldg(&a.grp_row[c.g]) + (int64_t)c.m * kGemmBM + rr;
      __nv_bfloat16* out = c.shared ? a.out_shared : a.out_routed;
      const int64_t ld = c.shared ? a.ld_shared : a.ld_routed;
      const int64_t rows = c.shared ? a.rows_shared : a.rows_routed;
      const int cols = c.shared ? a.cols_shared : a.cols_routed;
      const bool row_ok = orow < rows;
      if (!row_ok) record_error(a.err, kErrOutRow);
      if (MODE == kGateUpSwiGLU) {
#pragma unroll 1
        for (int hb = 0; hb < 2; ++hb) {
          const int col0 = c.n * (kGemmBN / 2) + hb * 64;
          if (col0 >= cols) break;
#pragma unroll 1
          for (int j = 0; j < 64; j += 32) {
            uint32_t gv[32], uv[32];
            __syncwarp();
            tmem_ld32(trow + static_cast<uint32_t>(hb * 128 + j), gv);
            tmem_ld32(trow + static_cast<uint32_t>(hb * 128 + 64 + j), uv);
            tmem_ld_wait(gv);
            tmem_ld_wait(uv);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
              const float h1 =
                  silu_f32(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            if (row_ok) {
              uint4* dst = reinterpret_cast<uint4*>(out + orow * ld + col0 + j);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < kGemmBN; cc += 32) {
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
            uint4* dst = reinterpret_cast<uint4*>(out + orow * ld + col);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kGemmTmemCols);
  }
}

}  // namespace moe
