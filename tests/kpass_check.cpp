// Host-only check of the k-pass chain schedule (csrc/kpass_plan.h), run by tests/test_kpass_host.py.
// For k = 1 .. SQUAD_KPASS_MAX_LEVELS and both orders it walks the forward and backward steps and checks
// the dataflow the library executes:
//   * forward: every pass reads the previous pass's output as values (v for the first), writes a fresh
//     intermediate (o for the last), and uses its own log-sum-exp slot and work counter;
//   * backward: passes run in reverse execution order with the forward's values and log-sum-exp; each
//     reads the value gradient the pass after it wrote (dout for the last pass), never writes the
//     buffer it reads, starts the dQ/dK shares once, adds to them after, and only the first pass
//     (which writes dv) writes dq and dk;
//   * every buffer index lies inside the workspace, and the levels run in the requested order.
// It prints one line per step and "ok", or the first violation and exits 1.
#include <cstdio>

#include "kpass_plan.h"

using namespace squad;

static int fail(const char* what, int k, int order, int e) {
  std::printf("FAIL k=%d order=%d step=%d: %s\n", k, order, e, what);
  return 1;
}

static int check(int k, int order) {
  squad_kpass_params_t p{};
  p.k = k;
  p.order = order;
  const int ni = kpass_n_inter(k), ng = kpass_n_gbuf(k);
  int prev_out = kBufV;
  bool written[SQUAD_KPASS_MAX_LEVELS] = {false};
  for (int e = 0; e < k; ++e) {
    const KpassFwdStep s = kpass_fwd_step(&p, e);
    std::printf("fwd k=%d order=%d e=%d level=%d values=%d out=%d lse=%d work=%d\n", k, order, e, s.level, s.values,
                s.out, s.lse, s.work);
    if (s.level != (order == SQUAD_KPASS_FORWARD ? e : k - 1 - e)) return fail("level order", k, order, e);
    if (s.values != prev_out) return fail("values are not the previous output", k, order, e);
    if (s.values >= 0 && (s.values >= ni || !written[s.values])) return fail("values not written", k, order, e);
    if (e + 1 == k ? s.out != kBufO : (s.out < 0 || s.out >= ni || written[s.out]))
      return fail("output buffer", k, order, e);
    if (s.out >= 0) written[s.out] = true;
    if (s.lse != e || s.work != 1 + e) return fail("lse slot or work counter", k, order, e);
    prev_out = s.out;
  }
  int prev_g = kBufDout;
  for (int e = k - 1; e >= 0; --e) {
    const KpassBwdStep s = kpass_bwd_step(&p, e);
    const KpassFwdStep f = kpass_fwd_step(&p, e);
    std::printf("bwd k=%d order=%d e=%d level=%d values=%d g_in=%d g_out=%d acc=%d final=%d\n", k, order, e, s.level,
                s.values, s.g_in, s.g_out, s.accumulate ? 1 : 0, s.final_out ? 1 : 0);
    if (s.level != f.level || s.values != f.values || s.lse != f.lse) return fail("not the forward's pass", k, order, e);
    if (s.g_in != prev_g) return fail("upstream is not the later pass's value gradient", k, order, e);
    if (e == 0 ? s.g_out != kBufDv : (s.g_out < 0 || s.g_out >= ng)) return fail("gradient buffer", k, order, e);
    if (s.g_out == s.g_in) return fail("writes the buffer it reads", k, order, e);
    if (s.accumulate != (e + 1 < k) || s.final_out != (e == 0)) return fail("share flags", k, order, e);
    prev_g = s.g_out;
  }
  return 0;
}

int main() {
  for (int k = 1; k <= SQUAD_KPASS_MAX_LEVELS; ++k)
    for (int order = SQUAD_KPASS_FORWARD; order <= SQUAD_KPASS_REVERSE; ++order)
      if (check(k, order) != 0) return 1;
  std::printf("ok\n");
  return 0;
}
