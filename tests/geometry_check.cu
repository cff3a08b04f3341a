// Host-only check of the kernels' index arithmetic (csrc/geometry.cuh), run by tests/test_geometry.py.
// For one grid/window it walks every chunk box of every pass exactly as TMA traverses it (from the
// tensor-map description and the box origin the kernel computes), and checks that
//   * box row r of chunk q of sequence sigma is token token_of(sigma, q, r) of head bh,
//   * rows past the sequence end fall outside the tensor (TMA fills them with zeros),
//   * every token of every head is covered exactly once per pass.
// It prints "ok" plus each pass's token table (one sequence per line) for comparison with the oracle.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "geometry.cuh"

using namespace squad;

static int check_pass(const Grid& g, int kind, int variant, bool print) {
  const PassGeom p = make_geom(g, kind);
  const MapDesc m = describe_pass_map(g, p, variant, 2);
  int errors = 0;
  unsigned cnt[5];
  for (int i = 0; i < 5; ++i) cnt[i] = (m.box[i] + m.es[i] - 1) / m.es[i];
  if (cnt[1] * cnt[2] * cnt[3] * cnt[4] != static_cast<unsigned>(p.chunk_rows)) {
    std::printf("box rows %u != chunk rows %d\n", cnt[1] * cnt[2] * cnt[3] * cnt[4], p.chunk_rows);
    return 1;
  }
  const int BH = g.B * g.h;
  std::vector<int> seen(static_cast<size_t>(BH) * g.n, 0);
  for (int bh = 0; bh < BH; ++bh)
    for (int sigma = 0; sigma < p.n_seq; ++sigma) {
      if (print && bh == 0) std::printf("seq %d %d:", kind, sigma);
      for (int q = 0; q < p.n_chunks; ++q) {
        int c[5];
        chunk_coords(g, p, variant, bh, sigma, q, 0, c);
        const int valid = chunk_valid_rows(p, q);
        for (unsigned i4 = 0; i4 < cnt[4]; ++i4)
          for (unsigned i3 = 0; i3 < cnt[3]; ++i3)
            for (unsigned i2 = 0; i2 < cnt[2]; ++i2)
              for (unsigned i1 = 0; i1 < cnt[1]; ++i1) {
                const int r = static_cast<int>(i1 + cnt[1] * (i2 + cnt[2] * (i3 + cnt[3] * i4)));
                const long long e[5] = {0, c[1] + static_cast<long long>(i1) * m.es[1],
                                        c[2] + static_cast<long long>(i2) * m.es[2],
                                        c[3] + static_cast<long long>(i3) * m.es[3],
                                        c[4] + static_cast<long long>(i4) * m.es[4]};
                bool oob = false;
                unsigned long long off = 0;
                for (int k = 1; k < 5; ++k) {
                  if (e[k] < 0 || static_cast<unsigned long long>(e[k]) >= m.dims[k]) oob = true;
                  off += static_cast<unsigned long long>(e[k]) * m.strides[k - 1];
                }
                const int want = token_of(g, p, sigma, q, r);
                if (r >= valid) {
                  if (want != -1 || !oob) {
                    ++errors;
                    if (errors < 10) std::printf("pad row in bounds: kind %d sigma %d q %d r %d\n", kind, sigma, q, r);
                  }
                  continue;
                }
                const unsigned long long lin = off / (static_cast<unsigned long long>(g.d) * 2);
                const long long got_bh = static_cast<long long>(lin / g.n), got = static_cast<long long>(lin % g.n);
                if (oob || got_bh != bh || got != want || off % (g.d * 2) != 0) {
                  ++errors;
                  if (errors < 10)
                    std::printf("mismatch kind %d var %d bh %d sigma %d q %d r %d: box -> (%lld, %lld) oob %d, token_of %d\n",
                                kind, variant, bh, sigma, q, r, got_bh, got, oob ? 1 : 0, want);
                  continue;
                }
                ++seen[static_cast<size_t>(bh) * g.n + got];
                if (print && bh == 0) std::printf(" %lld", got);
              }
        // Tile rows past the box (the kernel's 128-row tiles) are padding and must map to no token.
        for (int r = p.chunk_rows; r < 128; ++r)
          if (token_of(g, p, sigma, q, r) != -1) {
            ++errors;
            if (errors < 10) std::printf("tile row %d past the box maps to a token (kind %d q %d)\n", r, kind, q);
          }
      }
      if (print && bh == 0) std::printf("\n");
    }
  for (size_t i = 0; i < seen.size(); ++i)
    if (seen[i] != 1) {
      ++errors;
      if (errors < 10) std::printf("token %zu covered %d times in kind %d\n", i, seen[i], kind);
    }
  return errors;
}

// Multiply-shift division against the hardware divide: every divisor up to 4096, numerators at the
// boundaries and a pseudo-random sweep of [0, 2^31).
static int check_fastdiv() {
  int errors = 0;
  unsigned long long x = 88172645463325252ull;
  for (uint32_t d = 1; d <= 4096; ++d) {
    const FastDiv f = make_fastdiv(d);
    const uint32_t edge[] = {0u, 1u, d - 1, d, d + 1, 2 * d - 1, 2 * d, 0x7FFFFFFFu, 0x7FFFFFFEu,
                             0x7FFFFFFFu - (0x7FFFFFFFu % d)};
    for (uint32_t n : edge)
      if (n < 0x80000000u && fdiv(n, f) != n / d) ++errors;
    for (int i = 0; i < 2000; ++i) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      const uint32_t n = static_cast<uint32_t>(x) & 0x7FFFFFFFu;
      if (fdiv(n, f) != n / d) ++errors;
    }
  }
  if (errors) std::printf("fastdiv errors %d\n", errors);
  return errors;
}

int main(int argc, char** argv) {
  if (argc == 2 && argv[1][0] == 'd') {
    const int e = check_fastdiv();
    std::printf(e == 0 ? "ok\n" : "FAILED\n");
    return e == 0 ? 0 : 1;
  }
  if (argc != 8) {
    std::printf("usage: geometry_check B h T H W hw ww\n");
    return 2;
  }
  Grid g{};
  g.B = std::atoi(argv[1]);
  g.h = std::atoi(argv[2]);
  g.d = 128;
  g.T = std::atoi(argv[3]);
  g.H = std::atoi(argv[4]);
  g.W = std::atoi(argv[5]);
  g.hw = std::atoi(argv[6]);
  g.ww = std::atoi(argv[7]);
  g.n = g.T * g.H * g.W;
  g.nwy = g.H / g.hw;
  g.nwx = g.W / g.ww;
  finish_grid(g);
  int errors = 0;
  errors += check_pass(g, kLocal, 0, true);
  errors += check_pass(g, kGlobal, 0, true);
  errors += check_pass(g, kGlobal, 1, false);
  Grid f = g;   // full attention: one sequence of all tokens
  f.hw = f.ww = 1;
  f.nwy = f.H;
  f.nwx = f.W;
  finish_grid(f);
  errors += check_pass(f, kFull, 0, false);
  std::printf(errors == 0 ? "ok\n" : "FAILED %d\n", errors);
  return errors == 0 ? 0 : 1;
}
