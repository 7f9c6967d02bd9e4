// router.cuh -- fused router: centroid GEMM, softmax over the routed experts, top-k with
// lower-index tie-break, gates, per-tile expert histograms / within-tile ranks and
// per-tile affinity sums (the scan kernel of scan.cuh turns them into the layer's totals).
//
// DeepSeekMoE (deepforge.srivtx.xyz article), "Routing in a classic MoE layer":
// s_i = softmax_i(u^T e_i), g_i = s_i for the top-K affinities, else 0; "Top-k routing,
// from affinities to gates": softmax over all routed experts before the cut, gates not
// renormalised, stable ranking (equal logits -> lower index first); "Expert-level balance
// loss": counts and mean affinities per routed expert.
//
// Tiles of R <= 128 tokens, as many as there are SMs, so that each SM streams the centroid
// matrix once per tile and issues the fewest MMAs.  The bf16 kernel computes the 128 x N_pad
// logit tile with tcgen05.mma into one of two tensor-memory accumulators (A = the tile's
// token rows streamed by TMA, B = the padded centroid matrix; accumulator rows past R are
// never read back); a CTA with several tiles (large T) overlaps the next tile's loads with
// the epilogue.  Sixteen epilogue warps copy the logits (+ bias) to shared memory in passes
// of 64 rows and work on each pass with eight threads per token row: row max and softmax
// denominator by shuffles, the top-k by a bitonic sort of each thread's 64-bit (logit,
// index) keys and three bitonic merges across the row's threads (or, for top_k > 8 or wide
// rows, top_k rounds of a group-wide maximum).  The fp32 kernel and the decode-sized bf16
// kernel compute the same logits with FMA into the same shared-memory layout and share the
// rest.
#pragma once

#include <climits>

#include "scan.cuh"

namespace moe {

constexpr int kRouterBM = 128;          // MMA rows = largest token tile
constexpr int kRouterPass = 64;         // token rows per epilogue pass
constexpr int kRouterGroup = 8;         // threads per token row in the epilogue
constexpr int kRouterEpiThreads = 512;  // kRouterPass * kRouterGroup
constexpr int kRouterThreads = 64 + kRouterEpiThreads;   // warp 0 TMA, warp 1 MMA
constexpr int kRouterMaxStages = 8;
#ifndef MOE_ROUTER_MAX_KPS
#define MOE_ROUTER_MAX_KPS 4
#endif
constexpr int kRouterMaxKps = MOE_ROUTER_MAX_KPS;   // 64-wide k-blocks per pipeline stage, at most
constexpr size_t kRouterSmemBudget = 232448;   // opt-in dynamic shared memory per block
constexpr size_t kRouterCtlBytes = 512;        // mbarriers, TMEM slot, abort flag

struct RouterOut {
  int32_t* topk_idx;    // [T, top_k]
  float* topk_w;        // [T, top_k]
  int32_t* topk_rank;   // [T, top_k] rank of the token among the tile's tokens of that expert
  int32_t* tile_hist;   // [n_tiles, n_routed]
  float* tile_psum;     // [n_tiles, n_routed]  sum over the tile's tokens of s[t, i]
  int* err;
  float* logits;        // [T, n_routed] the logits (bias added) for the backward, or nullptr
};

// 16-byte aligned size: the logit rows that follow it take float4 stores.
struct alignas(16) RouterEpiSmem {
  float bias[kMaxRouted];
  uint32_t mask[kMaxRouted][4];            // bit r of mask[e][r/32]: token r of the tile chose e
  int32_t sel[kRouterBM][kMaxTopK];        // chosen experts of each row, in rank order
  float gsel[kRouterBM][kMaxTopK];         // their gates s[t, e]
  float inv_sum[kRouterPass];              // 1 / softmax denominator (0 for rows past T)
  float ppart[8][kMaxRouted];              // per-expert sums over row parts of the tile
};
static_assert(sizeof(RouterEpiSmem) % 16 == 0, "the logit rows after the scratch need 16-byte alignment");

// Epilogue scratch: RouterEpiSmem, then the logit rows of one pass lg[64][ld] (fp32, bias
// added), overwritten in place by exp(l - max).  ld = N_pad + 4 keeps the float4 row
// stores of a warp and the eight-thread row reads free of bank conflicts.
__host__ __device__ constexpr int router_ld(int n_pad) { return n_pad + 4; }
__host__ __device__ constexpr size_t router_epi_bytes(int n_pad) {
  return sizeof(RouterEpiSmem) + (size_t)kRouterPass * router_ld(n_pad) * 4;
}
// Compile-time bound on N_pad / 8 (the kernels are instantiated per bound); each lane of a
// routing warp holds up to MAXC / 4 = ceil(N_pad / 32) columns of a row.
__host__ __device__ constexpr int router_maxc(int n_pad) {
  return n_pad <= 16 ? 2 : n_pad <= 32 ? 4 : n_pad <= 64 ? 8 : n_pad <= 128 ? 16 : 32;
}
// Tokens per bf16 router tile for T tokens on n_sms SMs: the fewest tiles of <= 128
// tokens (a multiple of 8) with one tile per SM per round.
inline int router_tile_rows(int T, int n_sms) {
  const int per_sm = (T + n_sms - 1) / n_sms;
  const int k = (per_sm + kRouterBM - 1) / kRouterBM;
  return (((per_sm + k - 1) / k) + 7) / 8 * 8;
}
// TMEM columns of the tc router: two tiles' accumulators (N_pad each) in flight, a power of
// two >= 32.
__host__ __device__ constexpr uint32_t router_tmem_cols(int n_pad) {
  return 2u * (uint32_t)n_pad <= 32u ? 32u : 2u * (uint32_t)n_pad <= 64u ? 64u
         : 2u * (uint32_t)n_pad <= 128u ? 128u : 2u * (uint32_t)n_pad <= 256u ? 256u : 512u;
}
// Parts the rows of a pass are split into for the per-expert sums.
__host__ __device__ constexpr int router_psum_parts(int n_pad) {
  return kRouterEpiThreads / n_pad > 8 ? 8 : kRouterEpiThreads / n_pad;
}

// Order-preserving 32-bit key of a logit: a larger logit gets a larger key; NaN ranks as
// -inf and -0 as +0, so every expert gets a real rank and equal values tie.  Key 0 is below
// every logit (unused columns, experts already chosen).
__device__ __forceinline__ uint32_t logit_key(float l) {
  uint32_t b = (l != l) ? 0xFF800000u : __float_as_uint(l);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// The logit of a key (inverse of logit_key for keys >= 1).
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
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

// Descending bitonic sort of N keys held in registers.
template <int N>
__device__ __forceinline__ void bitonic_sort_desc(uint64_t (&k)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ stride;
        if (l > i) {
          const bool desc = (i & size) == 0;
          const uint64_t x = k[i], y = k[l];
          const bool sw = desc ? (x < y) : (x > y);
          k[i] = sw ? y : x;
          k[l] = sw ? x : y;
        }
      }
    }
  }
}

// One epilogue pass: the pass's logit rows (bias added) are in lg[r][i] for r < rows,
// i < N_pad, and the masks are zero (first pass) or hold the earlier passes' choices.
// Thread tid (of 512) works on row r = tid / 8 of the pass (tile row 64 * pass + r) with
// the eight threads of its row owning consecutive column blocks of C = N_pad / 8.  Writes
// sel/gsel/mask for its rows and adds the pass's per-expert affinity sums into ppart.
// `sync()` synchronises the 512 threads; returns with the scratch still in use.
template <int MAXC, class Sync>
__device__ __forceinline__ void router_pass(int tid, int pass, int tile, int R, int T,
                                            int n_routed, int n_pad, int top_k, uint8_t* epi,
                                            const RouterOut& o, Sync sync) {
  RouterEpiSmem& S = *reinterpret_cast<RouterEpiSmem*>(epi);
  float* lg = reinterpret_cast<float*>(epi + sizeof(RouterEpiSmem));
  const int ld = router_ld(n_pad);
  const int r = tid >> 3, j = tid & 7;
  const int tr = pass * kRouterPass + r;                  // row in the tile
  const int rows = min(kRouterPass, R - pass * kRouterPass);
  const int C = n_pad >> 3;              // even: N_pad is a multiple of 16
  const int c0 = j * C;
  const int t = tile * R + tr;
  const bool valid = r < rows && t < T;
  float* row = lg + (size_t)r * ld;

  // warps whose four rows all lie past the pass skip the per-row work (they still take
  // part in every barrier)
  if ((tid >> 5) * 4 < rows) {
  // keys and the row max; rows past the tile or past T are treated as zeros
  uint64_t key[MAXC];
  float lmax = -INFINITY;
#pragma unroll
  for (int k = 0; k < MAXC; k += 2) {
    float2 x = make_float2(0.f, 0.f);
    if (k < C && valid) x = *reinterpret_cast<const float2*>(row + c0 + k);
    const bool in0 = k < C && c0 + k < n_routed, in1 = k < C && c0 + k + 1 < n_routed;
    key[k] = in0 ? route_key(x.x, c0 + k) : 0ull;
    key[k + 1] = in1 ? route_key(x.y, c0 + k + 1) : 0ull;
    if (valid && o.logits) {   // the logits (bias added), kept for the backward
      if (in0) o.logits[(size_t)t * n_routed + c0 + k] = x.x;
      if (in1) o.logits[(size_t)t * n_routed + c0 + k + 1] = x.y;
    }
    if (in0) lmax = fmaxf(lmax, x.x);
    if (in1) lmax = fmaxf(lmax, x.y);
  }
#pragma unroll
  for (int m = 1; m < kRouterGroup; m <<= 1)
    lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, m));

  // exp(l - max) in place, denominator: column order within a thread, then a fixed tree
  float part = 0.f;
#pragma unroll
  for (int k = 0; k < MAXC; k += 2) {
    if (k < C) {
      const float2 x = *reinterpret_cast<const float2*>(row + c0 + k);
      const float e0 = (valid && c0 + k < n_routed) ? __expf(x.x - lmax) : 0.f;
      const float e1 = (valid && c0 + k + 1 < n_routed) ? __expf(x.y - lmax) : 0.f;
      part += e0;
      part += e1;
      *reinterpret_cast<float2*>(row + c0 + k) = make_float2(e0, e1);
    }
  }
#pragma unroll
  for (int m = 1; m < kRouterGroup; m <<= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
  const float inv_sum = 1.0f / part;
  if (j == 0) S.inv_sum[r] = valid ? inv_sum : 0.f;
  __syncwarp();   // the row's exp values (written by the eight threads of a warp) are read below

  auto record_e = [&](int p, int e) {
    if (e < 0 || e >= n_routed) {
      record_error(o.err, kErrRouteIndex);
      e = 0;
    }
    if (valid) {
      S.sel[tr][p] = e;
      S.gsel[tr][p] = row[e] * inv_sum;
      atomicOr(&S.mask[e][tr >> 5], 1u << (tr & 31));
    }
  };
  auto record = [&](int p, uint64_t g) { record_e(p, key_index(g)); };

  // Fast path (top_k <= 7, the bitonic network below on 32-bit keys): the logit's order
  // key with its low ib bits replaced by the inverted expert index, ib = bits of N_pad - 1.
  // It ranks as the exact (logit, index) order except among logits whose keys agree above
  // those bits; so when ranks 0 .. top_k hold no such pair the chosen experts and their
  // ranks are exactly those of the 64-bit order, and otherwise the warp redoes its rows
  // with 64-bit keys.
  bool done = false;
  if (MAXC <= 8 && top_k <= 7) {
    const int ib = 32 - __clz(n_pad - 1);
    const uint32_t mk = (1u << ib) - 1u;
    uint32_t kk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint64_t k64 = i < MAXC ? key[i < MAXC ? i : 0] : 0ull;
      kk[i] = k64 ? (((uint32_t)(k64 >> 32) & ~mk) | (mk - (uint32_t)key_index(k64))) : 0u;
    }
#pragma unroll
    for (int size = 2; size <= 8; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int l = i ^ stride;
          if (l > i) {
            const uint32_t x = kk[i], y = kk[l];
            const bool desc = (i & size) == 0;
            kk[i] = desc ? max(x, y) : min(x, y);
            kk[l] = desc ? min(x, y) : max(x, y);
          }
        }
      }
    }
#pragma unroll
    for (int m = 1; m < kRouterGroup; m <<= 1) {
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = __shfl_xor_sync(0xffffffffu, kk[i], m);
#pragma unroll
      for (int i = 0; i < 8; ++i) kk[i] = max(kk[i], pk[7 - i]);
#pragma unroll
      for (int stride = 4; stride > 0; stride >>= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int l = i ^ stride;
          if (l > i) {
            const uint32_t x = kk[i], y = kk[l];
            kk[i] = max(x, y);
            kk[l] = min(x, y);
          }
        }
      }
    }
    bool tie = false;   // the same for the row's eight threads (they hold the same list)
#pragma unroll
    for (int r = 0; r < 7; ++r)
      tie |= r < top_k && kk[r + 1] != 0u && ((kk[r] ^ kk[r + 1]) & ~mk) == 0u;
    if (!__any_sync(0xffffffffu, tie)) {
      uint32_t mine = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) mine = i == j ? kk[i] : mine;
      if (j < top_k) record_e(j, mine ? (int)(mk - (mine & mk)) : -1);
      done = true;
    }
  }
  if (done) {
  } else if (MAXC <= 8 && top_k <= 8) {
    // sort the thread's keys (padded to 8 with zeros), then three bitonic merges with the
    // partner threads: every thread of the row ends up with the row's 8 largest keys
    uint64_t kk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) kk[i] = i < MAXC ? key[i < MAXC ? i : 0] : 0ull;
    bitonic_sort_desc<8>(kk);
#pragma unroll
    for (int m = 1; m < kRouterGroup; m <<= 1) {
      uint64_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = __shfl_xor_sync(0xffffffffu, kk[i], m);
#pragma unroll
      for (int i = 0; i < 8; ++i) kk[i] = kk[i] > pk[7 - i] ? kk[i] : pk[7 - i];   // bitonic
#pragma unroll
      for (int stride = 4; stride > 0; stride >>= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int l = i ^ stride;
          if (l > i) {
            const uint64_t x = kk[i], y = kk[l];
            kk[i] = x > y ? x : y;
            kk[l] = x > y ? y : x;
          }
        }
      }
    }
    // thread j of the row records rank j
    uint64_t mine = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) mine = i == j ? kk[i] : mine;
    if (j < top_k) record(j, mine);
  } else {
    // top_k rounds: the group's largest remaining key; its owner records it and drops it
#pragma unroll 1
    for (int p = 0; p < top_k; ++p) {
      uint64_t best = key[0];
#pragma unroll
      for (int k = 1; k < MAXC; ++k) best = key[k] > best ? key[k] : best;
      uint64_t g = best;
#pragma unroll
      for (int m = 1; m < kRouterGroup; m <<= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, g, m);
        g = y > g ? y : g;
      }
      if (best == g) {   // keys are distinct (distinct indices): exactly one owner
        record(p, g);
#pragma unroll
        for (int k = 0; k < MAXC; ++k) key[k] = key[k] == g ? 0ull : key[k];
      }
    }
  }
  }   // warps with rows
  sync();

  // the pass's per-expert affinity sums: row parts, added to the earlier passes' parts
  const int P = router_psum_parts(n_pad);
  const int RP = (rows + P - 1) / P;
  for (int idx = tid; idx < P * n_pad; idx += kRouterEpiThreads) {
    const int pp = idx / n_pad, c = idx - pp * n_pad;
    const int r0 = pp * RP, r1 = min(rows, r0 + RP);
    float a = 0.f;
    for (int rr = r0; rr < r1; ++rr) a += lg[(size_t)rr * ld + c] * S.inv_sum[rr];
    S.ppart[pp][c] = pass == 0 ? a : S.ppart[pp][c] + a;
  }
}

// After every pass of the tile (and a sync): the tile's histogram and affinity sums, and
// the routing outputs with within-tile ranks (tokens of the tile that chose e before this
// one), written in [T, top_k] order.
__device__ __forceinline__ void router_tile_outputs(int tid, int tile, int R, int T, int n_routed,
                                                    int n_pad, int top_k, uint8_t* epi,
                                                    const RouterOut& o) {
  RouterEpiSmem& S = *reinterpret_cast<RouterEpiSmem*>(epi);
  const int P = router_psum_parts(n_pad);
  for (int c = tid; c < n_routed; c += kRouterEpiThreads) {
    float a = 0.f;
    for (int pp = 0; pp < P; ++pp) a += S.ppart[pp][c];
    o.tile_psum[(size_t)tile * n_routed + c] = a;
    o.tile_hist[(size_t)tile * n_routed + c] = __popc(S.mask[c][0]) + __popc(S.mask[c][1]) +
                                               __popc(S.mask[c][2]) + __popc(S.mask[c][3]);
  }
  const int rows = min(R, T - tile * R);
  for (int idx = tid; idx < rows * top_k; idx += kRouterEpiThreads) {
    const int tr = idx / top_k, p = idx - tr * top_k;
    const int e = S.sel[tr][p];
    const int q = tr >> 5;
    int rank = __popc(S.mask[e][q] & ((1u << (tr & 31)) - 1u));
    for (int qq = 0; qq < q; ++qq) rank += __popc(S.mask[e][qq]);
    const size_t at = (size_t)tile * R * top_k + idx;
    o.topk_idx[at] = e;
    o.topk_w[at] = S.gsel[tr][p];
    o.topk_rank[at] = rank;
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
  int T, d, n_routed, n_pad, top_k;
  int kps, stages;     // k-blocks per stage (1 .. 4), stages in the ring
  int tile_rows;       // R: tokens per tile (<= 128, multiple of 8); the U map's box height
  int n_tiles;         // tiles, handed out round-robin over the CTAs
  uint32_t tmem_cols;  // router_tmem_cols(n_pad): two tiles' accumulators in flight
  const float* bias;   // [>= n_routed] (zeros where no bias)
  RouterOut out;
};

// A stage holds kps (1 .. 4) 64-wide k-blocks: A_0 .. A_{kps-1} (the tile's R token rows of
// 128 B, rounded up to 1 KB) then B_0 .. B_{kps-1} (n_pad centroid rows of 128 B each, also
// rounded up).  A barrier round trip (the producer's wait on `empty`, the MMA issuer's
// wait on `full`) costs a few hundred cycles, about as long as the four N <= 64 MMAs of
// one k-block, so a stage carries as many k-blocks as keep the most of them in flight.  The
// M = 128 MMA reads 128 A rows; rows R..127 fall on the next block of the same stage (or the
// tail padding), which the same TMA batch has filled: they only produce accumulator rows
// that are never read.
__host__ __device__ constexpr uint32_t router_a_bytes(int R) { return ((uint32_t)R * 128u + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t router_b_bytes(int n_pad) { return ((uint32_t)n_pad * 128u + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t router_stage_bytes(int n_pad, int kps, int R) {
  return (uint32_t)kps * (router_a_bytes(R) + router_b_bytes(n_pad)) >
                 (uint32_t)(kps - 1) * router_a_bytes(R) + kRouterBM * 128u
             ? (uint32_t)kps * (router_a_bytes(R) + router_b_bytes(n_pad))
             : (uint32_t)(kps - 1) * router_a_bytes(R) + kRouterBM * 128u;
}
// dynamic shared memory: alignment slack, stage ring, epilogue scratch, control block
__host__ __device__ constexpr size_t router_smem_bytes(int n_pad, int kps, int R, int stages) {
  return 1024 + (size_t)stages * router_stage_bytes(n_pad, kps, R) + router_epi_bytes(n_pad) +
         kRouterCtlBytes;
}
// Stage shape: the {k-blocks per stage, stages} (at least two stages) that fits
// kRouterSmemBudget with the most k-blocks in flight, the larger stage on a tie (fewer
// barrier round trips); stages < 2 when nothing fits.
struct RouterStages { int kps, stages; };
inline RouterStages router_stages(int n_pad, int R) {
  RouterStages best{1, 0};
  for (int kps = 1; kps <= kRouterMaxKps; ++kps) {
    long st = ((long)kRouterSmemBudget - (long)router_smem_bytes(n_pad, kps, R, 0)) /
              (long)router_stage_bytes(n_pad, kps, R);
    if (st > kRouterMaxStages) st = kRouterMaxStages;
    if (st < 2) continue;
    if (best.stages < 2 || st * kps >= (long)best.stages * best.kps) best = RouterStages{kps, (int)st};
  }
  return best;
}

// Persistent: CTA b handles tiles b, b + gridDim.x, ...  With several tiles per CTA the
// producer and the MMA issuer run ahead into the next tile while the epilogue warps work.
template <int MAXC>
__global__ void __launch_bounds__(kRouterThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                 RouterTcArgs a) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t a_bytes = (uint32_t)a.tile_rows * 128u;           // bytes TMA writes per A block
  const uint32_t b_bytes = static_cast<uint32_t>(a.n_pad) * 128u;   // per B block
  const uint32_t a_slot = router_a_bytes(a.tile_rows);
  const uint32_t b_slot = router_b_bytes(a.n_pad);
  const uint32_t b_off = (uint32_t)a.kps * a_slot;                 // B_0's offset in a stage
  const uint32_t stage_bytes = router_stage_bytes(a.n_pad, a.kps, a.tile_rows);
  const int S = a.stages;
  uint8_t* epi = base + (size_t)S * stage_bytes;
  uint8_t* ctl = epi + router_epi_bytes(a.n_pad);
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kRouterMaxStages;
  uint64_t* acc_full = empty + kRouterMaxStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = a.d / 64;
  const int ksteps = (kblocks + a.kps - 1) / a.kps;   // stages per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(smem_u32(&full[s]), 1); mbar_init(smem_u32(&empty[s]), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(smem_u32(&acc_full[s]), 1); mbar_init(smem_u32(&acc_empty[s]), 1); }
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
  pdl_wait();   // u (and the bias) may come from the previous kernel

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        for (int ks = 0; ks < ksteps; ++ks) {
          ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, a.out.err, kErrWaitProducer);
          if (!ok) break;
          const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
          const int kb0 = ks * a.kps;
          const int nk = kblocks - kb0 < a.kps ? kblocks - kb0 : a.kps;
          mbar_arrive_expect_tx(smem_u32(&full[stage]), (uint32_t)nk * (a_bytes + b_bytes));
          for (int j = 0; j < nk; ++j) {
            tma_load_2d(sa + j * a_slot, &tmU, smem_u32(&full[stage]), (kb0 + j) * 64,
                        tile * a.tile_rows);
            tma_load_2d(sa + b_off + j * b_slot, &tmE, smem_u32(&full[stage]), (kb0 + j) * 64, 0);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      // every copy this thread started must have landed before the CTA exits
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s))
          mbar_wait(smem_u32(&full[s]), (last_par >> s) & 1u, abort_flag, a.out.err, kErrWaitDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kRouterBM, a.n_pad);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        ok = mbar_wait(smem_u32(&acc_empty[acc]), ((it >> 1) & 1) ^ 1u, abort_flag, a.out.err,
                       kErrWaitMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * a.n_pad);
        for (int ks = 0; ks < ksteps; ++ks) {
          ok = mbar_wait(smem_u32(&full[stage]), phase, abort_flag, a.out.err, kErrWaitMma);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(base + (size_t)stage * stage_bytes);
          const int kb0 = ks * a.kps;
          const int nk = kblocks - kb0 < a.kps ? kblocks - kb0 : a.kps;
          for (int j = 0; j < nk; ++j) {
            const uint64_t adesc = sdesc_k_sw128(sa + j * a_slot);
            const uint64_t bdesc = sdesc_k_sw128(sa + b_off + j * b_slot);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_f16(dt, adesc + 2u * k, bdesc + 2u * k, idesc, (ks | j | k) != 0);
          }
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit(smem_u32(&acc_full[acc]));
      }
      tc_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, abort_flag, a.out.err, kErrWaitDrain);
    }
    __syncwarp();
  } else {
    const int tid = threadIdx.x - 64;     // 0..511
    const int w = warp - 2;               // 0..15
    const int q = warp & 3;               // TMEM lane quadrant this warp may access
    const int sub = w >> 2;               // which 16-column slices it copies
    RouterEpiSmem& SM = *reinterpret_cast<RouterEpiSmem*>(epi);
    float* lg = reinterpret_cast<float*>(epi + sizeof(RouterEpiSmem));
    const int ld = router_ld(a.n_pad);
    const int nch = a.n_pad >> 4;
    const int npass = (a.tile_rows + kRouterPass - 1) / kRouterPass;
    auto sync = [] { named_bar_sync(1, kRouterEpiThreads); };
    for (int e = tid; e < kMaxRouted; e += kRouterEpiThreads)
      SM.bias[e] = e < a.n_routed ? a.bias[e] : 0.f;
    int it = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      // one thread polls the accumulator barrier; the others sleep in the named barrier,
      // and all sixteen warps take the same branch (they synchronise inside it)
      bool ok = true;
      if (tid == 0)
        ok = mbar_wait(smem_u32(&acc_full[acc]), (it >> 1) & 1, abort_flag, a.out.err,
                       kErrWaitEpilogue);
      if (named_bar_any(1, kRouterEpiThreads, !ok)) break;
      tc_fence_after();
      for (int e = tid; e < 4 * kMaxRouted; e += kRouterEpiThreads) (&SM.mask[0][0])[e] = 0u;
      for (int pass = 0; pass < npass; ++pass) {
        // accumulator rows 64 pass .. 64 pass + 63 -> shared memory (bias added): the
        // quadrants 2 pass and 2 pass + 1, four warps each, one 16-column slice per turn
        if ((q >> 1) == pass) {
          const int tr = q * 32 + lane;
          const uint32_t trow =
              tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)(acc * a.n_pad);
          for (int jj = sub; jj < nch; jj += 4) {
            uint32_t v[16];
            __syncwarp();
            tmem_ld16(trow + static_cast<uint32_t>(jj * 16), v);
            tmem_ld_wait16(v);
            if (tr < a.tile_rows) {
              float4* dst = reinterpret_cast<float4*>(lg + (size_t)(tr - pass * kRouterPass) * ld + jj * 16);
              const float* bb = SM.bias + jj * 16;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_float4(__uint_as_float(v[4 * k]) + bb[4 * k],
                                     __uint_as_float(v[4 * k + 1]) + bb[4 * k + 1],
                                     __uint_as_float(v[4 * k + 2]) + bb[4 * k + 2],
                                     __uint_as_float(v[4 * k + 3]) + bb[4 * k + 3]);
            }
          }
        }
        if (pass == npass - 1) tc_fence_before();
        sync();
        if (pass == npass - 1 && tid == 0) mbar_arrive(smem_u32(&acc_empty[acc]));   // accumulator free
        router_pass<MAXC>(tid, pass, tile, a.tile_rows, a.T, a.n_routed, a.n_pad, a.top_k, epi,
                          a.out, sync);
        sync();
      }
      router_tile_outputs(tid, tile, a.tile_rows, a.T, a.n_routed, a.n_pad, a.top_k, epi, a.out);
      sync();   // scratch free for the next tile
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

// 512 threads, one tile of 64 tokens (one epilogue pass) per CTA.  dynamic smem:
// router_epi_bytes(n_pad).
template <int MAXC>
__global__ void __launch_bounds__(kRouterEpiThreads) router_simt_kernel(RouterSimtArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RouterEpiSmem& SM = *reinterpret_cast<RouterEpiSmem*>(smem_raw);
  float* lg = reinterpret_cast<float*>(smem_raw + sizeof(RouterEpiSmem));
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int n_pad = (a.n_routed + 15) & ~15;
  const int ld = router_ld(n_pad);
  for (int e = tid; e < 4 * kMaxRouted; e += kRouterEpiThreads) (&SM.mask[0][0])[e] = 0u;
  for (int idx = tid; idx < kRouterPass * a.n_routed; idx += kRouterEpiThreads) {
    const int r = idx / a.n_routed, i = idx - r * a.n_routed;
    const int t = tile * kRouterPass + r;
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
    lg[(size_t)r * ld + i] = acc + a.bias[i];
  }
  __syncthreads();
  auto sync = [] { __syncthreads(); };
  router_pass<MAXC>(tid, 0, tile, kRouterPass, a.T, a.n_routed, n_pad, a.top_k, smem_raw, a.out,
                    sync);
  __syncthreads();
  router_tile_outputs(tid, tile, kRouterPass, a.T, a.n_routed, n_pad, a.top_k, smem_raw, a.out);
}

// ------------------------------------------------------------------------ bf16, few tokens
constexpr int kSmallPairs = 2;   // (token, expert) dot products a warp computes together
constexpr int kSmallVecSteps = 4;   // 16-byte vector steps of each whose loads are in flight together

struct RouterSmallArgs {
  const __nv_bfloat16* u;     // [T, d]
  const __nv_bfloat16* cen;   // [n_routed, d]
  const float* bias;          // [>= n_routed]
  int T, d, n_routed, top_k;
  int tile_rows;              // tokens per cluster (1..64)
  RouterOut out;
};

// For decode-sized batches (a handful of tokens), where the tensor-core router would
// stream the whole centroid matrix through its TMA ring for a tile of a few rows: each
// cluster of C CTAs (router_small_cluster: as many as the SMs allow for a single wave, at
// most kRouterSmallCluster) takes tile_rows tokens, and CTA q of it the logits of experts
// [q E, (q + 1) E), E = ceil(N_r / C), so that each SM streams only its share of the
// centroid matrix.  Each warp computes kSmallPairs (token, expert)
// dot products at a time with the lanes splitting d (16-byte vectors, kSmallVecSteps steps
// of loads in flight) and a fixed shuffle tree; the logits (bias added) go straight into the leader CTA's logit rows through
// distributed shared memory, and after a cluster barrier the leader runs the shared
// epilogue.  512 threads per CTA; dynamic smem router_epi_bytes(n_pad).
constexpr int kRouterSmallCluster = 4;
// CTAs per token cluster for T tokens on n_sms SMs (one CTA of 512 threads per SM).
inline int router_small_cluster(int T, int n_sms) {
  const int c = T > 0 ? n_sms / T : 1;
  return c < 1 ? 1 : (c > kRouterSmallCluster ? kRouterSmallCluster : c);
}
template <int MAXC>
__global__ void __launch_bounds__(kRouterEpiThreads) router_small_kernel(RouterSmallArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RouterEpiSmem& SM = *reinterpret_cast<RouterEpiSmem*>(smem_raw);
  float* lg = reinterpret_cast<float*>(smem_raw + sizeof(RouterEpiSmem));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t q = cluster_ctarank();
  const int C = (int)cluster_nctarank();
  const int tile = (int)blockIdx.x / C, R = a.tile_rows;
  const int n_pad = (a.n_routed + 15) & ~15;
  const int ld = router_ld(n_pad);
  const int nv = a.d >> 3;
  const int E = (a.n_routed + C - 1) / C;
  const int e0 = (int)q * E;
  const int ne = a.n_routed - e0 < E ? (a.n_routed - e0 > 0 ? a.n_routed - e0 : 0) : E;
  if (q == 0)
    for (int e = tid; e < 4 * kMaxRouted; e += kRouterEpiThreads) (&SM.mask[0][0])[e] = 0u;
  const uint32_t lg_leader = mapa_shared(smem_u32(lg), 0);
  cluster_sync_all();   // every CTA of the cluster is running before the first remote store
  // round by round, warp w takes pairs w, w + 16, ... (kSmallPairs of them) so that their
  // loads are in flight together; every dot product keeps its own order of operations
  constexpr int kWarps = kRouterEpiThreads / 32;
  const int npairs = R * ne;
  for (int p0 = 0; p0 < npairs; p0 += kWarps * kSmallPairs) {
    const uint4* ur[kSmallPairs];
    const uint4* er[kSmallPairs];
    bool on[kSmallPairs];
    float acc[kSmallPairs];
#pragma unroll
    for (int j = 0; j < kSmallPairs; ++j) {
      const int pj = p0 + j * kWarps + warp;
      const int p = pj < npairs ? pj : npairs - 1;
      const int r = p / ne, i = e0 + (p - r * ne);
      const int t = tile * R + r;
      on[j] = pj < npairs && t < a.T;
      ur[j] = reinterpret_cast<const uint4*>(a.u + (size_t)(t < a.T ? t : 0) * a.d);
      er[j] = reinterpret_cast<const uint4*>(a.cen + (size_t)i * a.d);
      acc[j] = 0.f;
    }
    for (int v0 = lane; v0 < nv; v0 += 32 * kSmallVecSteps) {
      uint4 xu[kSmallVecSteps][kSmallPairs], xe[kSmallVecSteps][kSmallPairs];
#pragma unroll
      for (int b = 0; b < kSmallVecSteps; ++b) {
#pragma unroll
        for (int j = 0; j < kSmallPairs; ++j) {
          if (on[j] && v0 + 32 * b < nv) {
            xu[b][j] = __ldg(ur[j] + v0 + 32 * b);
            xe[b][j] = __ldg(er[j] + v0 + 32 * b);
          }
        }
      }
      // each pair's products in ascending vector order, as one FMA chain
#pragma unroll
      for (int b = 0; b < kSmallVecSteps; ++b) {
#pragma unroll
        for (int j = 0; j < kSmallPairs; ++j) {
          if (on[j] && v0 + 32 * b < nv) {
            float x[8], y[8];
            bf16x8_to_f32(xu[b][j], x);
            bf16x8_to_f32(xe[b][j], y);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[j] = fmaf(x[k], y[k], acc[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kSmallPairs; ++j) {
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], m);
      const int p = p0 + j * kWarps + warp;
      if (lane == 0 && p < npairs) {
        const int r = p / ne, i = e0 + (p - r * ne);
        st_shared_cluster_f32(lg_leader + 4u * (uint32_t)(r * ld + i), acc[j] + a.bias[i]);
      }
    }
  }
  cluster_sync_all();   // the cluster's logits are in the leader's rows
  if (q != 0) return;
  auto sync = [] { __syncthreads(); };
  router_pass<MAXC>(tid, 0, tile, R, a.T, a.n_routed, n_pad, a.top_k, smem_raw, a.out, sync);
  __syncthreads();
  router_tile_outputs(tid, tile, R, a.T, a.n_routed, n_pad, a.top_k, smem_raw, a.out);
}

}  // namespace moe
