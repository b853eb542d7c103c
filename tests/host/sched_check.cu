// Host-only check of the GEMM tile scheduler in umma_gemm.cuh (256 x 256 and 256 x 512 tiles): enumerates every
// global tile index through decode_tile() and verifies coverage and uniqueness
// for the dense (band raster), symmetric-upper and causal schedules, over
// ragged sizes and multi-group launches.  Prints "OK" on success.
#include <cstdio>
#include <set>
#include <tuple>
#include <vector>

#include "umma_gemm.cuh"

using namespace mc;

static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { ++fails; if (fails < 20) { std::printf(__VA_ARGS__); std::printf("\n"); } } } while (0)

static GemmGroup mk(int M, int N, int K, int count, int sched, int band, int nshift = 0) {
  GemmGroup G{};
  G.M = M; G.N = N; G.K = K; G.count = count; G.sched = sched; G.band = band; G.nshift = nshift;
  const int tn = MMA_N << nshift;
  G.tiles_m = (M + BM - 1) / BM; G.tiles_n = (N + tn - 1) / tn;
  G.tiles_per_prob = sched_tiles_per_prob(sched, G.tiles_m, G.tiles_n, nshift);
  return G;
}

static void check_groups(std::vector<GemmGroup> gs) {
  long long total = 0;
  for (auto& g : gs) { g.tile_start = total; total += g.tiles_per_prob * g.count; }
  std::vector<std::set<std::tuple<int, int, int>>> seen(gs.size());
  // (prob, tm, tn) of wide symmetric tiles whose first 256-column block is skipped
  std::vector<std::set<std::tuple<int, int, int>>> skipped(gs.size());
  for (long long t = 0; t < total; ++t) {
    TileInfo ti;
    decode_tile(gs.data(), (int)gs.size(), t, ti);
    const GemmGroup& G = gs[ti.g];
    CHECK(t >= G.tile_start && t < G.tile_start + G.tiles_per_prob * G.count, "tile %lld decoded to wrong group", t);
    CHECK(ti.prob >= 0 && ti.prob < G.count, "prob out of range");
    CHECK(ti.tm >= 0 && ti.tm < G.tiles_m && ti.tn >= 0 && ti.tn < G.tiles_n, "tile (%d,%d) out of range M=%d N=%d", ti.tm, ti.tn, G.M, G.N);
    CHECK(ti.num_kb == (G.K + BK - 1) / BK, "num_kb");
    auto key = std::make_tuple(ti.prob, ti.tm, ti.tn);
    CHECK(!seen[ti.g].count(key), "duplicate tile");
    seen[ti.g].insert(key);
    const long long BNt = MMA_N << G.nshift;
    if (G.nshift == 1 && sym_skip_first_block<2>(G, ti)) {
      skipped[ti.g].insert(key);
      // the skipped block must hold no element on or above the diagonal
      CHECK((long long)ti.tn * BNt + MMA_N - 1 < (long long)ti.tm * BM, "skipped block reaches the diagonal");
    }
    if (G.sched == SCHED_SYM) {
      CHECK(ti.tn >= (ti.tm >> G.nshift), "sym tile below diagonal");
      CHECK((long long)ti.tn * BNt + BNt - 1 >= (long long)ti.tm * BM, "sym tile with no upper element");
    }
    if (G.sched == SCHED_CAUSAL) {
      CHECK(ti.tn <= (ti.tm >> G.nshift), "causal tile above diagonal");
      CHECK((long long)ti.tn * BNt <= (long long)ti.tm * BM + BM - 1, "causal tile with no valid element");
    }
  }
  for (size_t gi = 0; gi < gs.size(); ++gi) {
    const GemmGroup& G = gs[gi];
    const int BN = MMA_N << G.nshift;
    for (int p = 0; p < G.count; ++p) {
      if (G.sched == SCHED_DENSE) {
        for (int i = 0; i < G.tiles_m; ++i)
          for (int j = 0; j < G.tiles_n; ++j) CHECK(seen[gi].count({p, i, j}), "dense tile missing");
      } else if (G.sched == SCHED_SYM) {
        // every element (r, c) with c >= r must lie in a computed tile
        // (and not in a skipped first block)
        auto kept = [&](int r, int c) {
          const auto key = std::make_tuple(p, r / BM, c / BN);
          if (!seen[gi].count(key)) return false;
          return !(skipped[gi].count(key) && (c % BN) < MMA_N);
        };
        for (int r = 0; r < G.M; r += 7)
          for (int c = r; c < G.N; c += 5) CHECK(kept(r, c), "sym element (%d,%d) uncovered", r, c);
        for (int r = 0; r < G.M; ++r) CHECK(kept(r, r), "sym diagonal uncovered");
      } else {
        for (int r = 0; r < G.M; r += 3)
          for (int c = 0; c <= r; c += 11) CHECK(seen[gi].count({p, r / BM, c / BN}), "causal element (%d,%d) uncovered", r, c);
        for (int r = 0; r < G.M; ++r) CHECK(seen[gi].count({p, r / BM, r / BN}), "causal diagonal uncovered");
      }
    }
  }
}

int main() {
  const int sizes[] = {1, 7, 64, 100, 128, 129, 255, 256, 257, 300, 384, 511, 640, 1000, 1024, 2048, 4096};
  for (int w = 0; w < 2; ++w) {
    for (int M : sizes)
      for (int N : sizes) {
        check_groups({mk(M, N, 64, 2, SCHED_DENSE, 8, w)});
        check_groups({mk(M, N, 300, 1, SCHED_DENSE, 3, w)});
      }
    for (int m : sizes) {
      check_groups({mk(m, m, 77, 3, SCHED_SYM, 8, w)});
      check_groups({mk(m, m, 128, 2, SCHED_CAUSAL, 8, w)});
    }
    check_groups({mk(4096, 4096, 4096, 3, SCHED_SYM, 8, w), mk(4096, 4096, 14336, 2, SCHED_SYM, 8, w),
                  mk(300, 300, 10, 4, SCHED_SYM, 8, w), mk(129, 129, 1, 1, SCHED_SYM, 8, w)});
  }
  check_groups({mk(4096, 4096, 4096, 3, SCHED_SYM, 8), mk(4096, 4096, 14336, 2, SCHED_SYM, 8),
                mk(300, 300, 10, 4, SCHED_SYM, 8), mk(129, 129, 1, 1, SCHED_SYM, 8)});
  check_groups({mk(4096, 14336, 4096, 2, SCHED_DENSE, 8), mk(14336, 4096, 4096, 1, SCHED_DENSE, 8),
                mk(1024, 1024, 1024, 5, SCHED_DENSE, 8)});
  // the 7B-shaped symmetric launch size
  // 16 x 16 tiles of 256: the upper (or lower) triangle with its diagonal
  GemmGroup a = mk(4096, 4096, 4096, 128, SCHED_SYM, 8);
  CHECK(a.tiles_per_prob == 136, "sym count %lld", a.tiles_per_prob);
  GemmGroup c = mk(4096, 4096, 128, 128, SCHED_CAUSAL, 8);
  CHECK(c.tiles_per_prob == 136, "causal count %lld", c.tiles_per_prob);
  CHECK(BM == 256 && MMA_N == 256, "tile shape");
  // 16 x 8 tiles of 256 x 512: rows i keep j >= i/2 (SYM) or j <= i/2 (CAUSAL)
  GemmGroup aw = mk(4096, 4096, 4096, 1, SCHED_SYM, 8, 1);
  CHECK(aw.tiles_per_prob == 72, "wide sym count %lld", aw.tiles_per_prob);
  GemmGroup cw = mk(4096, 4096, 128, 1, SCHED_CAUSAL, 8, 1);
  CHECK(cw.tiles_per_prob == 72, "wide causal count %lld", cw.tiles_per_prob);
  if (fails) { std::printf("FAILED %d checks\n", fails); return 1; }
  std::printf("OK\n");
  return 0;
}
