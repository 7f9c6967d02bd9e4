// Host-side tiling rules of the kernels, checked exhaustively without a GPU (the program
// makes no CUDA call).  Exit status 0 = every rule holds; the first violation is printed.
#include <algorithm>
#include <cstdio>
#include <vector>

#include "combine.cuh"
#include "gemm_small.cuh"
#include "gemm_tc.cuh"
#include "router.cuh"

using namespace moe;

static int fails = 0;
#define CHECK(cond, ...)                                  \
  do {                                                    \
    if (!(cond)) {                                        \
      if (fails++ < 10) {                                 \
        std::printf("FAIL %s: ", #cond);                  \
        std::printf(__VA_ARGS__);                         \
        std::printf("\n");                                \
      }                                                   \
    }                                                     \
  } while (0)

int main() {
  // router tiles: a multiple of 8 rows, at most the MMA's 128, and the tiles cover T with
  // at most ceil(T / (SMs * 128)) tiles per SM
  for (int n_sms : {132, 148, 160}) {
    for (int T = 1; T <= 70000; T += (T < 4096 ? 1 : 97)) {
      const int R = router_tile_rows(T, n_sms);
      CHECK(R >= 8 && R <= kRouterBM && R % 8 == 0, "T=%d sms=%d R=%d", T, n_sms, R);
      const long tiles = (T + R - 1) / R;
      const long rounds = (T + (long)n_sms * kRouterBM - 1) / ((long)n_sms * kRouterBM);
      CHECK(tiles <= (long)n_sms * rounds, "T=%d sms=%d R=%d tiles=%ld", T, n_sms, R, tiles);
    }
  }
  // router stages: every padded expert count and tile height gets a ring of >= 2 stages
  // inside the shared-memory budget; the M = 128 MMA reading 128 rows from a stage's last
  // A block stays inside that stage; two accumulators fit the 512 TMEM columns
  for (int n_pad = 16; n_pad <= kMaxRouted; n_pad += 16) {
    for (int R = 8; R <= kRouterBM; R += 8) {
      const RouterStages rs = router_stages(n_pad, R);
      CHECK(rs.stages >= 2 && rs.stages <= kRouterMaxStages, "n_pad=%d R=%d stages=%d", n_pad, R, rs.stages);
      CHECK(rs.kps >= 1 && rs.kps <= kRouterMaxKps, "n_pad=%d R=%d kps=%d", n_pad, R, rs.kps);
      CHECK(router_smem_bytes(n_pad, rs.kps, R, rs.stages) <= kRouterSmemBudget,
            "n_pad=%d R=%d bytes=%zu", n_pad, R, router_smem_bytes(n_pad, rs.kps, R, rs.stages));
      const uint32_t stage = router_stage_bytes(n_pad, rs.kps, R);
      CHECK((uint32_t)(rs.kps - 1) * router_a_bytes(R) + kRouterBM * 128u <= stage,
            "n_pad=%d R=%d MMA A read past the stage", n_pad, R);
      CHECK((uint32_t)rs.kps * (router_a_bytes(R) + router_b_bytes(n_pad)) <= stage,
            "n_pad=%d R=%d blocks past the stage", n_pad, R);
      CHECK(router_a_bytes(R) % 1024 == 0 && router_b_bytes(n_pad) % 1024 == 0 && stage % 1024 == 0,
            "n_pad=%d R=%d 1 KB alignment of the swizzled blocks", n_pad, R);
      // the epilogue's logit rows (float4 stores) and the control block (mbarriers) after
      // the 1 KB-aligned ring stay 16-byte aligned
      CHECK(sizeof(RouterEpiSmem) % 16 == 0 && (router_ld(n_pad) * 4) % 16 == 0 &&
                router_epi_bytes(n_pad) % 16 == 0,
            "n_pad=%d epilogue scratch alignment", n_pad);
      // two tiles' accumulators fit the 512 TMEM columns (a power of two >= 32)
      const uint32_t cols = router_tmem_cols(n_pad);
      CHECK(cols <= 512 && cols >= 2u * n_pad && (cols & (cols - 1)) == 0,
            "n_pad=%d TMEM columns %u", n_pad, cols);
      CHECK(router_maxc(n_pad) * kRouterGroup >= n_pad, "n_pad=%d maxc=%d", n_pad, router_maxc(n_pad));
    }
  }
  // the scan in the router's last CTA: (segment, expert) pairs fit its 512 threads and the
  // segments cover every tile
  for (int nr = 1; nr <= kMaxRouted; ++nr) {
    for (int n_tiles = 1; n_tiles <= 700; ++n_tiles) {
      int nseg = kScanThreads / nr;
      if (nseg > n_tiles) nseg = n_tiles;
      if (nseg < 1) nseg = 1;
      const int seg_len = (n_tiles + nseg - 1) / nseg;
      CHECK(nseg * nr <= kScanThreads && (long)nseg * seg_len >= n_tiles,
            "nr=%d n_tiles=%d nseg=%d seg_len=%d", nr, n_tiles, nseg, seg_len);
    }
  }
  // combine: warps per row between 1 and one lane-wide vector batch per part
  for (int T = 1; T <= 70000; T += (T < 4096 ? 1 : 97)) {
    for (int nvec : {4, 8, 16, 32, 33, 64, 100, 160, 256, 512}) {
      const int p = combine_parts(T, nvec, 148);
      CHECK(p >= 1 && (p == 1 || p <= nvec / 32), "T=%d nvec=%d parts=%d", T, nvec, p);
      CHECK((long)T * p < (1L << 31), "T=%d parts=%d overflows the grid", T, p);
    }
  }
  // decode FFN kernel: for every token width a ring of 2 .. kSmallMaxStages stages that fits
  // the opt-in shared memory with the control block, and two accumulators of 2 n_tok
  // columns that fit its TMEM allocation
  for (int nt = 16; nt <= kSmallMaxTok; nt += 16) {
    const int st = small_stages(nt);
    CHECK(st >= 2 && st <= kSmallMaxStages, "n_tok=%d stages=%d", nt, st);
    CHECK(small_smem_bytes(nt, st) <= kRouterSmemBudget, "n_tok=%d bytes=%zu", nt, small_smem_bytes(nt, st));
    CHECK(small_stage_bytes(nt) % 1024 == 0, "n_tok=%d stage %u", nt, small_stage_bytes(nt));
    const uint32_t tc = small_tmem_cols(nt);
    CHECK(tc >= 4u * nt && tc <= 512 && (tc & (tc - 1)) == 0, "n_tok=%d TMEM columns %u", nt, tc);
  }
  // the paired GEMM's ring and control block fit the opt-in shared memory
  CHECK(kGemmSmemBytes <= kRouterSmemBudget, "GEMM smem %zu", kGemmSmemBytes);
  CHECK(kGemmStageBytes % 1024 == 0, "GEMM stage %u", kGemmStageBytes);
  if (fails) std::printf("%d rule violations\n", fails);
  else std::printf("all tiling rules hold\n");
  return fails ? 1 : 0;
}
