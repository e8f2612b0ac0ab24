// Host-side check of the scheduling rules that the router and the kernels
// share (compiled with nvcc and run on the CPU, no GPU call): the K parts of
// the tensor-core down units stay inside the workspace's part buffers and
// tickets and give every part of an all-rows unit at least one K-block (a
// part of a gathered unit may have none: it adds zeros); the candidate-group rule
// is the stated threshold; the row-stream stage geometry fits its budget.
// Exits non-zero with the first violated case.
#include <cstdio>
#include <cstdlib>

#include "gemv_common.cuh"
#include "kernels.h"

using namespace moe;

static int fails = 0;
static long long checked = 0;

#define CHECK(cond, ...)                       \
  do {                                         \
    ++checked;                                 \
    if (!(cond)) {                             \
      if (fails++ < 10) {                      \
        std::printf("FAIL %s: ", #cond);       \
        std::printf(__VA_ARGS__);              \
        std::printf("\n");                     \
      }                                        \
    }                                          \
  } while (0)

static void check_ksplit() {
  const int modes[] = {kModeAuto, kModeDense, kModeGemv, kModeTc, kModeTcAll};
  const int ds[] = {256, 512, 2048, 4096, 7168, 8192};
  const int Fs_[] = {128, 384, 768, 1408, 14336, 65536};
  const int Ts[] = {1, 2, 4, 8, 16, 17, 32, 48, 64, 65, 100, 128, 4096};
  const int grids[] = {0, 1, 16, 148, 160, 296, 320, 512};
  const int units_caps[] = {0, 640, 1024};
  for (int mode : modes)
    for (int d : ds)
      for (int F : Fs_)
        for (int S = 0; S <= 2; ++S)
          for (int Fsh : {128, 1408})
            for (int T : Ts)
              for (int grid : grids)
                for (int cap_units : units_caps)
                  for (int gcap : {kGroupMax, kGroupMaxDecode}) {
                  Dims dm = {};
                  dm.gcap = gcap;
                  dm.mode = mode;
                  dm.d = d;
                  dm.F = F;
                  dm.S = S;
                  dm.Fs = S > 0 ? Fsh : 0;
                  dm.T = T;
                  dm.tc_grid = grid;
                  dm.tc_part_units = cap_units;
                  const int nslices = d / kDownSlice;
                  const int tmax = T < gcap ? T : gcap;
                  const int n_max = (tmax + 15) / 16 * 16;
                  for (int n_tc = 0; n_tc <= 700; n_tc += (n_tc < 40 ? 1 : 37)) {
                    const int ks = tc_ksplit(dm, n_tc);
                    const long long base = (long long)n_tc * nslices;
                    CHECK(ks >= 1 && ks <= kTcMaxParts, "ks %d", ks);
                    if (n_max > kTcPartTokens || cap_units == 0 || grid == 0)
                      CHECK(ks == 1, "mode %d n_max %d cap %d grid %d ks %d", mode, n_max,
                            cap_units, grid, ks);
                    if (ks > 1) {
                      CHECK(base * ks <= cap_units, "base %lld ks %d cap %d", base, ks, cap_units);
                      // units are cut only when they fill under 3/4 of the grid, except
                      // forced gathered launches (units as long as their unions)
                      if (mode != kModeTc)
                        CHECK(4 * base < 3LL * grid, "base %lld grid %d", base, grid);
                      // every part of every expert kind has at least one K-block
                      for (int kind = 0; kind < (S > 0 ? 2 : 1); ++kind) {
                        const int nk = (kind ? dm.Fs : F) / kKBlock;
                        for (int p = 0; p < ks; ++p) {
                          const int k0 = nk * p / ks, k1 = nk * (p + 1) / ks;
                          CHECK(k1 - k0 >= 1, "F %d Fs %d ks %d part %d", F, dm.Fs, ks, p);
                        }
                      }
                      // the largest part-buffer element a unit touches
                      const long long last =
                          ((base - 1) * ks + (ks - 1)) * kTcPartTokens * kDownSlice +
                          (long long)(n_max - 1) * kDownSlice + (kDownSlice - 1);
                      CHECK(last < (long long)cap_units * kTcPartTokens * kDownSlice,
                            "part buffer index %lld", last);
                      CHECK(base <= cap_units, "tickets %lld > %d", base, cap_units);
                    }
                  }
                }
}

static void check_candidates() {
  for (int F : {128, 768, 1408, 14336}) {
    for (int passes = 1; passes <= 2; ++passes) {
      bool prev = true;
      for (int u = 0; u <= F; ++u) {
        const bool take = cand_takes_gemv(u, passes, F);
        CHECK(take == ((long long)u * passes * 5 <= 4LL * F), "F %d u %d", F, u);
        CHECK(!take || prev, "not monotone at F %d u %d", F, u);  // once false, stays false
        prev = take;
      }
      CHECK(cand_takes_gemv(0, passes, F), "empty union");
      CHECK(!cand_takes_gemv(F, passes, F), "full union");
    }
  }
}

static void check_geometry() {
  for (int es : {2, 4})
    for (int d = 128; d <= 16384; d += 128) {
      if (es == 2 && d % 256) continue;  // bf16 layers: d_model a multiple of 256
      const int row_bytes = d * es;
      for (int extra : {0, 16, 272, 512}) {
        const Geometry g = geometry(row_bytes, extra);
        CHECK(g.n_stages >= 2 && g.n_stages <= kMaxStages, "d %d es %d stages %d", d, es,
              g.n_stages);
        CHECK((long long)g.n_stages * g.stage <= kSmemBudget, "d %d smem", d);
        CHECK(g.block <= kBlockBytes && g.block % kSliceBytes == 0, "block %d", g.block);
        CHECK(g.stride % 16 == 0 && g.stage % 16 == 0, "alignment d %d", d);
        // the down row stream's wide blocks (bf16 rows of a multiple of 1 KB):
        // up to 8 KB per block, whole 1 KB slices, at least two stages
        if (es == 2 && d % 512 == 0) {
          const Geometry w = geometry(row_bytes, extra, 8192);
          CHECK(w.n_stages >= 2 && w.n_stages <= kMaxStages, "wide d %d stages %d", d, w.n_stages);
          CHECK((long long)w.n_stages * w.stage <= kSmemBudget, "wide d %d smem", d);
          CHECK(w.block <= 8192 && w.block % 1024 == 0, "wide block %d", w.block);
          CHECK(w.stride % 16 == 0 && w.stage % 16 == 0, "wide alignment d %d", d);
        }
      }
    }
}

int main() {
  // group cap: a multiple of the slot block (groups stay inside their
  // expert's slot range), and below kGroupMax only for 33-64 token batches
  // of routed-only tensor-core layers
  static_assert(kGroupMaxDecode % kSlotAlign == 0 && kGroupMax % kSlotAlign == 0, "caps");
  for (int T = 1; T <= 300; ++T)
    for (int E = 1; E <= 256; E *= 2)
      for (int S = 0; S <= 1; ++S)
        for (int no_tc = 0; no_tc <= 1; ++no_tc) {
          Dims cap = {};
          cap.E = E;
          cap.S = S;
          cap.no_tc = no_tc;
          const int g = group_cap(cap, T, 2);
          const bool small = !no_tc && !S && T > 32 && T <= 64 && 4 * T <= 32 * E;
          CHECK(g == (small ? kGroupMaxDecode : kGroupMax), "T %d E %d S %d cap %d", T, E, S, g);
        }

  check_ksplit();
  check_candidates();
  check_geometry();
  std::printf("%s %lld checks, %d failed\n", fails ? "FAIL" : "OK", checked, fails);
  return fails ? 1 : 0;
}
