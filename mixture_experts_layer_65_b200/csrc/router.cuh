// router.cuh -- fused router: centroid GEMM, softmax over the routed experts, top-k with
// lower-index tie-break, gates, per-tile expert histograms / within-tile ranks and
// per-tile affinity sums.
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Routing in a classic MoE layer":
// s_i = softmax_i(u^T e_i), g_i = s_i for the top-K affinities, else 0; "Top-k routing,
// from affinities to gates": softmax over all routed experts before the cut, gates not
// renormalised, stable ranking (equal logits -> lower index first); "Expert-level balance
// loss": counts and mean affinities per routed expert.
//
// One CTA handles a tile of R <= 128 tokens (R is chosen so the tiles cover all SMs).
// The bf16 kernel computes the 128 x N_pad logit tile with tcgen05.mma into tensor memory
// (A = the tile's token rows streamed by TMA, B = the padded centroid matrix; rows past R
// are never read back).  Sixteen epilogue warps then share the rows: four threads per
// token row (one per 16-column slice modulo 4), which reduce their partial maxima, sums
// and top-k lists through shared memory.  The fp32 kernel computes the same logits with
// FMA and shares the epilogue.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace moe {

constexpr int kMaxTopK = 16;
constexpr int kMaxRouted = 256;
constexpr int kRouterBM = 128;          // MMA rows (and the largest token tile)
constexpr int kRouterEpiThreads = 512;  // 4 threads per row
constexpr int kRouterThreads = 64 + kRouterEpiThreads;   // warp 0 TMA, warp 1 MMA
constexpr int kRouterMaxStages = 8;

struct RouterOut {
  int32_t* topk_idx;    // [T, top_k]
  float* topk_w;        // [T, top_k]
  int32_t* topk_rank;   // [T, top_k] rank of the token among the tile's tokens of that expert
  int32_t* tile_hist;   // [n_tiles, n_routed]
  float* tile_psum;     // [n_tiles, n_routed]  sum over the tile's tokens of s[t, i]
  int* err;
};

struct RouterEpiSmem {
  uint32_t mask[kMaxRouted][4];   // bit r of mask[e][r/32]: token r of the tile chose e
  float bias[kMaxRouted];
  float ppart[4][kMaxRouted];     // per-expert sums over 32-row quarters of the tile
  float inv_sum[kRouterBM];       // 1 / softmax denominator per row (0 for rows past T)
  float rowmax[kRouterBM];
  float maxpart[4][kRouterBM];    // [sub][row]: lanes of a warp hit consecutive banks
  float sumpart[4][kRouterBM];
};

// Epilogue scratch: RouterEpiSmem, then one region that first holds the per-thread top-k
// lists [4][MAXK][128] (u64, row fastest) and then the exp(l - max) rows [128][ld] (fp32).
__host__ __device__ constexpr int router_row_ld(int n_routed) { return ((n_routed + 31) & ~31) + 1; }
__host__ __device__ constexpr size_t router_region_bytes(int n_routed, int maxk) {
  return (size_t)kRouterBM * router_row_ld(n_routed) * 4 > (size_t)kRouterBM * 4 * maxk * 8
             ? (size_t)kRouterBM * router_row_ld(n_routed) * 4
             : (size_t)kRouterBM * 4 * maxk * 8;
}
__host__ __device__ constexpr size_t router_epi_bytes(int n_routed, int maxk) {
  return sizeof(RouterEpiSmem) + router_region_bytes(n_routed, maxk);
}
// Length of the per-thread top-k list (compile-time, so it stays in registers): the
// insertion chain costs one 64-bit compare-exchange per slot, so it is sized tightly.
__host__ __device__ constexpr int router_maxk(int top_k) {
  return top_k <= 4 ? 4 : top_k <= 6 ? 6 : top_k <= 8 ? 8 : top_k <= 12 ? 12 : 16;
}

// Total order on (logit, expert): larger logit first; on equal logits the lower index.
// NaN ranks as -inf and -0 as +0, so every slot gets a real index and equal values tie.
__device__ __forceinline__ uint64_t route_key(float l, int i) {
  uint32_t b = (l != l) ? 0xFF800000u : __float_as_uint(l);
  if (b == 0x80000000u) b = 0u;
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<uint64_t>(ord) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - (uint32_t)i);
}

__device__ __forceinline__ int key_index(uint64_t key) {
  return (int)(0xFFFFFFFFu - (uint32_t)key);
}

// Epilogue of one token tile.  Thread (r, sub), r < 128, sub < 4, owns the 16-column
// slices j == sub (mod 4) of row r.  `load16(col, v)` yields the 16 raw fp32 logits of
// columns col..col+15 of row r (called uniformly by all 512 threads); `sync()`
// synchronises the 512 epilogue threads.
template <int MAXK, class Load16, class Sync>
__device__ __forceinline__ void router_epilogue(int r, int sub, int tile, int tile_rows, int T,
                                                int n_routed, int n_pad, int top_k,
                                                const float* __restrict__ bias, uint8_t* epi,
                                                const RouterOut& o, Load16 load16, Sync sync) {
  RouterEpiSmem& S = *reinterpret_cast<RouterEpiSmem*>(epi);
  uint8_t* region = epi + sizeof(RouterEpiSmem);
  uint64_t* tops = reinterpret_cast<uint64_t*>(region);
  float* rows = reinterpret_cast<float*>(region);
  const int ld = router_row_ld(n_routed);
  const int tid = sub * kRouterBM + r;
  const int t = tile * tile_rows + r;
  const bool valid = r < tile_rows && t < T;
  const int nch = n_pad >> 4;

  for (int e = tid; e < kMaxRouted; e += kRouterEpiThreads) {
    S.mask[e][0] = 0u; S.mask[e][1] = 0u; S.mask[e][2] = 0u; S.mask[e][3] = 0u;
    S.bias[e] = e < n_routed ? bias[e] : 0.f;
  }
  sync();

  // pass 1: partial max and partial top-MAXK (64-bit keys, sorted by a compare-exchange
  // chain in registers) over this thread's slices
  uint64_t top[MAXK];
#pragma unroll
  for (int p = 0; p < MAXK; ++p) top[p] = 0ull;
  float lmax = -INFINITY;
  uint32_t v[16];
  for (int j = sub; j < nch; j += 4) {
    load16(j * 16, v);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int i = j * 16 + k;
      if (i < n_routed) {
        const float l = __uint_as_float(v[k]) + S.bias[i];
        lmax = fmaxf(lmax, l);
        uint64_t key = route_key(l, i);
        if (key > top[MAXK - 1]) {
#pragma unroll
          for (int p = 0; p < MAXK; ++p) {
            const uint64_t hi = top[p] > key ? top[p] : key;
            key = top[p] > key ? key : top[p];
            top[p] = hi;
          }
        }
      }
    }
  }
#pragma unroll
  for (int p = 0; p < MAXK; ++p) tops[(size_t)(sub * MAXK + p) * kRouterBM + r] = top[p];
  S.maxpart[sub][r] = lmax;
  sync();

  // row owner (sub 0): merge the four sorted lists, row max in a fixed order
  if (sub == 0) {
    const uint64_t* L = tops + r;    // element (s, p) at L[(s * MAXK + p) * 128]
    int h0 = 0, h1 = 0, h2 = 0, h3 = 0;
#pragma unroll
    for (int p = 0; p < MAXK; ++p) {
      const uint64_t a0 = h0 < MAXK ? L[(size_t)h0 * kRouterBM] : 0ull;
      const uint64_t a1 = h1 < MAXK ? L[(size_t)(MAXK + h1) * kRouterBM] : 0ull;
      const uint64_t a2 = h2 < MAXK ? L[(size_t)(2 * MAXK + h2) * kRouterBM] : 0ull;
      const uint64_t a3 = h3 < MAXK ? L[(size_t)(3 * MAXK + h3) * kRouterBM] : 0ull;
      const uint64_t m01 = a0 > a1 ? a0 : a1, m23 = a2 > a3 ? a2 : a3;
      const uint64_t m = m01 > m23 ? m01 : m23;
      top[p] = m;
      if (m == a0) ++h0; else if (m == a1) ++h1; else if (m == a2) ++h2; else ++h3;
    }
    S.rowmax[r] = fmaxf(fmaxf(S.maxpart[0][r], S.maxpart[1][r]),
                        fmaxf(S.maxpart[2][r], S.maxpart[3][r]));
  }
  sync();   // the list region is reused for the exp rows below

  // pass 2: exp(l - max) into the row buffer, partial denominators in slice order
  {
    const float rmax = S.rowmax[r];
    float part = 0.f;
    float* my = rows + (size_t)r * ld;
    for (int j = sub; j < nch; j += 4) {
      load16(j * 16, v);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int i = j * 16 + k;
        if (i < n_routed) {
          // rows past the tile hold values computed from stale shared memory: store 0
          const float e = valid ? __expf(__uint_as_float(v[k]) + S.bias[i] - rmax) : 0.f;
          part += e;
          my[i] = e;
        }
      }
    }
    S.sumpart[sub][r] = part;
  }
  sync();
  float inv_sum = 0.f;
  if (sub == 0) {
    const float sum = ((S.sumpart[0][r] + S.sumpart[1][r]) + S.sumpart[2][r]) + S.sumpart[3][r];
    inv_sum = 1.0f / sum;
    S.inv_sum[r] = valid ? inv_sum : 0.f;
    if (valid) {
#pragma unroll
      for (int p = 0; p < MAXK; ++p) {
        if (p < top_k) {
          const int e = key_index(top[p]);
          if (e >= 0 && e < n_routed) atomicOr(&S.mask[e][r >> 5], 1u << (r & 31));
        }
      }
    }
  }
  sync();

  // the tile's per-expert affinity sums: four 32-row quarters, then a fixed-order total
  {
    const int quarter = tid >> 7;
    for (int c = tid & (kRouterBM - 1); c < n_routed; c += kRouterBM) {
      float a = 0.f;
#pragma unroll 8
      for (int rr = quarter * 32; rr < quarter * 32 + 32; ++rr)
        a += rows[(size_t)rr * ld + c] * S.inv_sum[rr];
      S.ppart[quarter][c] = a;
    }
  }
  sync();
  for (int c = tid; c < n_routed; c += kRouterEpiThreads) {
    o.tile_psum[(size_t)tile * n_routed + c] =
        ((S.ppart[0][c] + S.ppart[1][c]) + S.ppart[2][c]) + S.ppart[3][c];
    o.tile_hist[(size_t)tile * n_routed + c] =
        __popc(S.mask[c][0]) + __popc(S.mask[c][1]) + __popc(S.mask[c][2]) + __popc(S.mask[c][3]);
  }

  // outputs and within-tile ranks (tokens of the tile that chose e before this one)
  if (sub == 0 && valid) {
    const int q = r >> 5;
    const uint32_t below = (1u << (r & 31)) - 1u;
    const float* my = rows + (size_t)r * ld;
#pragma unroll
    for (int p = 0; p < MAXK; ++p) {
      if (p < top_k) {
        int e = key_index(top[p]);
        int rank = 0;
        float g = 0.f;
        if (e >= 0 && e < n_routed) {
          for (int qq = 0; qq < q; ++qq) rank += __popc(S.mask[e][qq]);
          rank += __popc(S.mask[e][q] & below);
          g = my[e] * inv_sum;
        } else {
          record_error(o.err, kErrRouteIndex);
          e = 0;
        }
        const size_t at = (size_t)t * top_k + p;
        o.topk_idx[at] = e;
        o.topk_w[at] = g;
        o.topk_rank[at] = rank;
      }
    }
  }
}

// 32 lanes x 16 consecutive fp32 columns of TMEM.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// ------------------------------------------------------------------------ bf16, tcgen05
struct RouterTcArgs {
  int T, d, n_routed, n_pad, top_k, stages;
  int tile_rows;       // R: tokens per CTA (<= 128, multiple of 8); the U map's box height
  uint32_t tmem_cols;
  const float* bias;   // [>= n_routed] (zeros where no bias)
  RouterOut out;
};

// stage = A (room for 128 rows of 128 B; R are written) + B (n_pad rows of 128 B)
__host__ __device__ constexpr uint32_t router_stage_bytes(int n_pad) {
  return kRouterBM * 128u + (((uint32_t)n_pad * 128u + 1023u) & ~1023u);
}

template <int MAXK>
__global__ void __launch_bounds__(kRouterThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                 RouterTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t a_off = kRouterBM * 128u;                         // B's offset in a stage
  const uint32_t a_bytes = (uint32_t)a.tile_rows * 128u;           // bytes TMA writes for A
  const uint32_t b_bytes = static_cast<uint32_t>(a.n_pad) * 128u;
  const uint32_t stage_bytes = router_stage_bytes(a.n_pad);
  const int S = a.stages;
  uint8_t* ctl = base + (size_t)S * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kRouterMaxStages;
  uint64_t* acc_full = empty + kRouterMaxStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int kblocks = a.d / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(smem_u32(&full[s]), 1); mbar_init(smem_u32(&empty[s]), 1); }
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmE);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.out.err, kErrWaitProducer)) break;
        const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
        mbar_arrive_expect_tx(smem_u32(&full[stage]), a_bytes + b_bytes);
        tma_load_2d(sa, &tmU, smem_u32(&full[stage]), kb * 64, tile * a.tile_rows);
        tma_load_2d(sa + a_off, &tmE, smem_u32(&full[stage]), kb * 64, 0);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      // every copy this thread started must have landed before the CTA exits
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s))
          mbar_wait(smem_u32(&full[s]), (last_par >> s) & 1u, abort_flag, a.out.err, kErrWaitDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, a.n_pad);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < kblocks && ok; ++kb) {
        ok = mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.out.err, kErrWaitMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
        const uint64_t adesc = sdesc_k_sw128(sa), bdesc = sdesc_k_sw128(sa + a_off);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_f16(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
        tc_commit(smem_u32(&empty[stage]));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (ok) tc_commit(smem_u32(acc_full));
      tc_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, abort_flag, a.out.err, kErrWaitDrain);
    }
    __syncwarp();
  } else {
    const int w = warp - 2;              // 0..15
    const int q = warp & 3;              // TMEM lane quadrant this warp may access
    const int sub = w >> 2;              // which slices of the row
    const int r = q * 32 + lane;
    // one thread polls the accumulator barrier; the others sleep in the named barrier,
    // and all sixteen warps take the same branch (they synchronise inside it)
    bool ok = true;
    if (w == 0 && lane == 0)
      ok = mbar_wait(smem_u32(acc_full), 0, abort_flag, a.out.err, kErrWaitEpilogue);
    if (!named_bar_any(1, kRouterEpiThreads, !ok)) {
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      auto load16 = [&](int c, uint32_t (&v)[16]) {
        __syncwarp();
        tmem_ld16(trow + static_cast<uint32_t>(c), v);
        tmem_ld_wait16(v);
      };
      auto sync = [] { named_bar_sync(1, kRouterEpiThreads); };
      router_epilogue<MAXK>(r, sub, tile, a.tile_rows, a.T, a.n_routed, a.n_pad, a.top_k, a.bias,
                            base, a.out, load16, sync);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

// ------------------------------------------------------------------------ fp32, FMA
struct RouterSimtArgs {
  const float* u;     // [T, d]
  const float* cen;   // [n_routed, d]
  const float* bias;  // [>= n_routed]
  int T, d, n_routed, top_k;
  RouterOut out;
};

// 512 threads, tiles of 128 tokens.  dynamic smem: router_epi_bytes(n_routed, MAXK) plus a
// [128][ld] logit buffer.  n_routed <= 128.
template <int MAXK>
__global__ void __launch_bounds__(kRouterEpiThreads) router_simt_kernel(RouterSimtArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int ld = router_row_ld(a.n_routed);
  float* logits = reinterpret_cast<float*>(smem_raw + router_epi_bytes(a.n_routed, MAXK));
  const int tid = threadIdx.x;
  const int r = tid & (kRouterBM - 1), sub = tid >> 7;
  const int tile = blockIdx.x;
  const int t = tile * kRouterBM + r;
  const int n_pad = (a.n_routed + 15) & ~15;
  // thread (r, sub) computes the logits of the slices it owns in the epilogue
  for (int j = sub; j < (n_pad >> 4); j += 4) {
    for (int i = j * 16; i < j * 16 + 16 && i < a.n_routed; ++i) {
      float acc = 0.f;
      if (t < a.T) {
        const float4* ur = reinterpret_cast<const float4*>(a.u + (size_t)t * a.d);
        const float4* er = reinterpret_cast<const float4*>(a.cen + (size_t)i * a.d);
        for (int k = 0; k < a.d / 4; ++k) {
          const float4 x = ur[k], y = __ldg(&er[k]);
          acc = fmaf(x.x, y.x, acc); acc = fmaf(x.y, y.y, acc);
          acc = fmaf(x.z, y.z, acc); acc = fmaf(x.w, y.w, acc);
        }
      }
      logits[(size_t)r * ld + i] = acc;
    }
  }
  auto load16 = [&](int c, uint32_t (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 16; ++k)
      v[k] = (c + k < a.n_routed) ? __float_as_uint(logits[(size_t)r * ld + c + k]) : 0u;
  };
  auto sync = [] { __syncthreads(); };
  router_epilogue<MAXK>(r, sub, tile, kRouterBM, a.T, a.n_routed, n_pad, a.top_k, a.bias,
                        smem_raw, a.out, load16, sync);
}

}  // namespace moe
