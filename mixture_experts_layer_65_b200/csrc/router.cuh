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
// One CTA handles a tile of 128 tokens.  The bf16 kernel computes the 128 x N_pad logit
// tile with tcgen05.mma into tensor memory (A = token rows streamed by TMA, B = the
// padded centroid matrix); four epilogue warps then own one token row each.  The fp32
// kernel computes the same logits with FMA and shares the epilogue.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace moe {

constexpr int kMaxTopK = 16;
constexpr int kMaxRouted = 256;
constexpr int kRouterBM = 128;
constexpr int kRouterThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
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
  float inv_sum[kRouterBM];       // 1 / softmax denominator per row (0 for rows past T)
};

// Epilogue scratch: RouterEpiSmem followed by a [128][ld] fp32 row buffer.
__host__ __device__ constexpr int router_row_ld(int n_routed) { return ((n_routed + 31) & ~31) + 1; }
__host__ __device__ constexpr size_t router_epi_bytes(int n_routed) {
  return sizeof(RouterEpiSmem) + (size_t)kRouterBM * router_row_ld(n_routed) * 4;
}

// Total order on (logit, expert): larger logit first; on equal logits the lower index.
// NaN ranks as -inf and -0 as +0, so every slot gets a real index and equal values tie.
__device__ __forceinline__ uint64_t route_key(float l, int i) {
  uint32_t b = (l != l) ? 0xFF800000u : __float_as_uint(l);
  if (b == 0x80000000u) b = 0u;
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<uint64_t>(ord) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - (uint32_t)i);
}

// One epilogue thread = one token row r (0..127) of tile `tile`.  `load(c, v)` yields the
// 32 raw fp32 logits (bit patterns) of columns c..c+31 of this row and is called uniformly
// by all 128 threads; `sync()` synchronises the 128 epilogue threads.  `rows` is a
// [128][ld] fp32 buffer (it may hold the logits on entry; load() reads a chunk before
// this function overwrites it).
template <int MAXK, class Load, class Sync>
__device__ __forceinline__ void router_epilogue(int r, int tile, int T, int n_routed, int n_cols,
                                                int top_k, const float* __restrict__ bias,
                                                RouterEpiSmem& S, float* rows, const RouterOut& o,
                                                Load load, Sync sync) {
  const int t = tile * kRouterBM + r;
  const bool valid = t < T;
  const int ld = router_row_ld(n_routed);
  float* my = rows + (size_t)r * ld;
  for (int e = r; e < kMaxRouted; e += kRouterBM) {
    S.mask[e][0] = 0u; S.mask[e][1] = 0u; S.mask[e][2] = 0u; S.mask[e][3] = 0u;
    S.bias[e] = e < n_routed ? bias[e] : 0.f;
  }
  sync();

  // pass 1: row max and the MAXK largest (logit, index) keys, kept sorted descending by a
  // compare-exchange chain in registers
  uint64_t top[MAXK];
#pragma unroll
  for (int p = 0; p < MAXK; ++p) top[p] = 0ull;
  float lmax = -INFINITY;
  uint32_t v[32];
  for (int c = 0; c < n_cols; c += 32) {
    load(c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = c + j;
      if (i < n_routed) {
        const float l = __uint_as_float(v[j]) + S.bias[i];
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

  // pass 2: exp(l - max) per expert into the row buffer, denominator in ascending order
  float sum = 0.f;
  for (int c = 0; c < n_cols; c += 32) {
    load(c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = c + j;
      if (i < n_routed) {
        const float e = __expf(__uint_as_float(v[j]) + S.bias[i] - lmax);
        sum += e;
        my[i] = e;
      }
    }
  }
  const float inv_sum = 1.0f / sum;
  S.inv_sum[r] = valid ? inv_sum : 0.f;

  // gates g = s at the selected experts, and the expert bitmasks of this tile
  if (valid) {
#pragma unroll
    for (int p = 0; p < MAXK; ++p) {
      if (p < top_k) {
        const int e = (int)(0xFFFFFFFFu - (uint32_t)top[p]);
        if (e >= 0 && e < n_routed) atomicOr(&S.mask[e][r >> 5], 1u << (r & 31));
      }
    }
  }
  sync();

  // the tile's per-expert affinity sums: one column per thread, rows in order
  for (int c = r; c < n_routed; c += kRouterBM) {
    float a = 0.f;
#pragma unroll 8
    for (int rr = 0; rr < kRouterBM; ++rr) a += rows[(size_t)rr * ld + c] * S.inv_sum[rr];
    o.tile_psum[(size_t)tile * n_routed + c] = a;
    o.tile_hist[(size_t)tile * n_routed + c] =
        __popc(S.mask[c][0]) + __popc(S.mask[c][1]) + __popc(S.mask[c][2]) + __popc(S.mask[c][3]);
  }

  // outputs and within-tile ranks (tokens of the tile that chose e before this one)
  if (valid) {
    const int q = r >> 5;
    const uint32_t below = (1u << (r & 31)) - 1u;
#pragma unroll
    for (int p = 0; p < MAXK; ++p) {
      if (p < top_k) {
        int e = (int)(0xFFFFFFFFu - (uint32_t)top[p]);
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

// ------------------------------------------------------------------------ bf16, tcgen05
struct RouterTcArgs {
  int T, d, n_routed, n_pad, top_k, stages;
  uint32_t tmem_cols;
  const float* bias;   // [n_pad] (zeros where no bias)
  RouterOut out;
};

template <int MAXK>
__global__ void __launch_bounds__(kRouterThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                 RouterTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t a_bytes = kRouterBM * 64 * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(a.n_pad) * 128u;
  const uint32_t stage_bytes = a_bytes + ((b_bytes + 1023u) & ~1023u);
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
        tma_load_2d(sa, &tmU, smem_u32(&full[stage]), kb * 64, tile * kRouterBM);
        tma_load_2d(sa + a_bytes, &tmE, smem_u32(&full[stage]), kb * 64, 0);
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
        const uint64_t adesc = sdesc_k_sw128(sa), bdesc = sdesc_k_sw128(sa + a_bytes);
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
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool ok = mbar_wait(smem_u32(acc_full), 0, abort_flag, a.out.err, kErrWaitEpilogue);
    // all four epilogue warps take the same branch (they synchronise inside it)
    if (!named_bar_any(1, 128, !ok)) {
      tc_fence_after();
      RouterEpiSmem& E = *reinterpret_cast<RouterEpiSmem*>(base);
      float* rows = reinterpret_cast<float*>(base + sizeof(RouterEpiSmem));
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      auto load = [&](int c, uint32_t (&v)[32]) {
        __syncwarp();
        tmem_ld32(trow + static_cast<uint32_t>(c), v);
        tmem_ld_wait(v);
      };
      auto sync = [] { named_bar_sync(1, 128); };
      router_epilogue<MAXK>(r, tile, a.T, a.n_routed, a.n_pad, a.top_k, a.bias, E, rows, a.out,
                            load, sync);
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

// dynamic smem: router_epi_bytes(n_routed) (the row buffer first holds the logits)
template <int MAXK>
__global__ void __launch_bounds__(kRouterBM) router_simt_kernel(RouterSimtArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RouterEpiSmem& E = *reinterpret_cast<RouterEpiSmem*>(smem_raw);
  float* rows = reinterpret_cast<float*>(smem_raw + sizeof(RouterEpiSmem));
  const int ld = router_row_ld(a.n_routed);
  const int r = threadIdx.x;
  const int tile = blockIdx.x;
  const int t = tile * kRouterBM + r;
  for (int i = 0; i < a.n_routed; ++i) {
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
    rows[(size_t)r * ld + i] = acc;
  }
  const int n_cols = (a.n_routed + 31) & ~31;
  auto load = [&](int c, uint32_t (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = (c + j < a.n_routed) ? __float_as_uint(rows[(size_t)r * ld + c + j]) : 0u;
  };
  auto sync = [] { __syncthreads(); };
  router_epilogue<MAXK>(r, tile, a.T, a.n_routed, n_cols, a.top_k, a.bias, E, rows, a.out, load, sync);
}

}  // namespace moe
