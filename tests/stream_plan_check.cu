// Host-only check of the streamed decode kernel's work split (the functions
// the kernel and the host share: stream_block_cols, stream_segments,
// stream_piece).  Built and run by tests/test_stream_plan.py; no GPU.
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "lr_internal.h"

using namespace lr;

static int fails = 0;
#define CHECK(c, ...)                    \
  do {                                   \
    if (!(c)) {                          \
      if (fails < 20) {                  \
        std::printf("FAIL %s: ", #c);    \
        std::printf(__VA_ARGS__);        \
        std::printf("\n");              \
      }                                  \
      ++fails;                           \
    }                                    \
  } while (0)

int main() {
  // Block widths.
  for (int64_t n = 1; n <= 20000; n += (n < 600 ? 1 : 97)) {
    const int cb = stream_block_cols(n);
    const int64_t nb = (n + cb - 1) / cb;
    CHECK(cb % 8 == 0 && cb >= 8 && cb <= 248, "n=%lld cb=%d", (long long)n, cb);
    CHECK(nb == (n + 247) / 248, "n=%lld nb=%lld", (long long)n, (long long)nb);
    CHECK((nb - 1) * cb < n, "n=%lld: last block empty", (long long)n);
  }
  std::mt19937_64 rng(12345);
  for (int trial = 0; trial < 300; ++trial) {
    StreamArgs a{};
    const int pairs = 1 + static_cast<int>(rng() % 7);
    for (int p = 0; p < pairs; ++p) {
      const int K = 1 + static_cast<int>(rng() % (trial % 3 == 0 ? 64 : 16384));
      const int r = 1 + static_cast<int>(rng() % 4000);
      const int N = 1 + static_cast<int>(rng() % (trial % 5 == 0 ? 150000 : 16384));
      StreamJob& j0 = a.job[a.n_jobs++];
      j0.phase = 0; j0.K = K; j0.N = r; j0.cb = stream_block_cols(r);
      j0.unit0 = a.units[0]; a.units[0] += int64_t(K) * r;
      StreamJob& j1 = a.job[a.n_jobs++];
      j1.phase = 1; j1.K = r; j1.N = N; j1.cb = stream_block_cols(N); j1.src = a.n_jobs - 2;
      j1.unit0 = a.units[1]; a.units[1] += int64_t(r) * N;
    }
    const int grids[3] = {148, 132, 7};
    const int G = grids[trial % 3];
    // rows covered per (job, block)
    std::vector<std::vector<std::vector<int>>> cover(a.n_jobs);
    for (int j = 0; j < a.n_jobs; ++j) {
      const int nb = (a.job[j].N + a.job[j].cb - 1) / a.job[j].cb;
      cover[j].assign(nb, std::vector<int>(a.job[j].K, 0));
    }
    std::vector<StreamSeg> buf(4096);
    for (int g = 0; g < G; ++g) {
      const int n = stream_segments(a, g, G, buf.data(), static_cast<int>(buf.size()));
      CHECK(n <= static_cast<int>(buf.size()), "trial %d g %d: %d pieces", trial, g, n);
      int64_t units[2] = {0, 0};
      int last_phase = 0;
      for (int i = 0; i < n && i < static_cast<int>(buf.size()); ++i) {
        const StreamSeg& s = buf[i];
        const StreamJob& J = a.job[s.job];
        CHECK(J.phase >= last_phase, "trial %d g %d: phase-1 piece before a phase-0 piece", trial, g);
        last_phase = J.phase;
        CHECK(0 <= s.k0 && s.k0 < s.k1 && s.k1 <= J.K, "trial %d g %d: rows [%d, %d) of %d", trial,
              g, s.k0, s.k1, J.K);
        const int64_t wb = std::min<int64_t>(J.cb, J.N - int64_t(s.b) * J.cb);
        units[J.phase] += wb * (s.k1 - s.k0);
        for (int k = s.k0; k < s.k1; ++k) ++cover[s.job][s.b][k];
        const StreamSeg p = stream_piece(a, s.job, s.b, g, G);
        CHECK(p.k0 == s.k0 && p.k1 == s.k1, "trial %d g %d: stream_piece differs", trial, g);
      }
      // Balance: a CTA's units are within one row of the widest block of an
      // even share.
      for (int ph = 0; ph < 2; ++ph) {
        const double share = double(a.units[ph]) / G;
        CHECK(std::abs(double(units[ph]) - share) <= 248.0 * 2 + 1e-9,
              "trial %d g %d phase %d: %lld units against %.1f", trial, g, ph,
              (long long)units[ph], share);
      }
    }
    for (int j = 0; j < a.n_jobs; ++j)
      for (size_t b = 0; b < cover[j].size(); ++b)
        for (int k = 0; k < a.job[j].K; ++k)
          CHECK(cover[j][b][k] == 1, "trial %d job %d block %zu row %d covered %d times", trial, j, b,
                k, cover[j][b][k]);
  }
  std::printf(fails ? "FAILED %d\n" : "OK\n", fails);
  return fails ? 1 : 0;
}
