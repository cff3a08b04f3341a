// Planning of k composed passes over nested windows (squad_kpass_* in the header): the levels'
// checks, the single-pass problem each level runs, and the buffer schedule of the forward and the
// backward chains. Host-only and free of CUDA, so that a host build can check it (tests/kpass_check.cpp).
#pragma once

#include <cstdint>
#include <cstring>

#include "squad_attn.h"

namespace squad {

// Buffers of a k-pass chain: the caller's tensors, or index i >= 0 of the workspace's intermediate
// outputs (forward) or value-gradient buffers (backward).
enum KpassBuf : int { kBufV = -1, kBufO = -2, kBufDout = -3, kBufDv = -4 };

struct KpassFwdStep {
  int level;     // level whose pass runs (0 = the innermost window)
  int values;    // kBufV or intermediate output index
  int out;       // kBufO or intermediate output index
  int lse;       // log-sum-exp slot (= the step's position in execution order)
  int work;      // control-block word of the persistent kernel's work counter (1 + step)
};

struct KpassBwdStep {
  int level;
  int values;     // kBufV or intermediate output index (as in the forward)
  int g_in;       // kBufDout or value-gradient buffer index
  int g_out;      // kBufDv or value-gradient buffer index
  int lse;
  bool accumulate;   // add to the fp32 dQ/dK shares of the passes already done
  bool final_out;    // write dq, dk instead of the shares
};

// SQUAD_OK, or why p cannot run: the levels must factor the grid exactly and every pass attends over
// at least two tokens.
inline squad_status_t kpass_check(const squad_kpass_params_t* p) {
  if (p == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (p->k < 1 || p->k > SQUAD_KPASS_MAX_LEVELS) return SQUAD_ERR_INVALID_ARG;
  if (p->order != SQUAD_KPASS_FORWARD && p->order != SQUAD_KPASS_REVERSE) return SQUAD_ERR_INVALID_ARG;
  if (p->B < 1 || p->h < 1 || p->T < 1 || p->H < 1 || p->W < 1) return SQUAD_ERR_INVALID_ARG;
  long long ph = 1, pw = 1;
  for (int l = 0; l < p->k; ++l) {
    if (p->level_h[l] < 1 || p->level_w[l] < 1) return SQUAD_ERR_INVALID_ARG;
    ph *= p->level_h[l];
    pw *= p->level_w[l];
    if (ph > p->H || pw > p->W) return SQUAD_ERR_INVALID_ARG;
  }
  if (ph != p->H || pw != p->W) return SQUAD_ERR_INVALID_ARG;
  if (static_cast<long long>(p->B) * p->h * p->T * p->H > INT32_MAX) return SQUAD_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->T) * p->level_h[0] * p->level_w[0] < 2) return SQUAD_ERR_UNSUPPORTED;
  for (int l = 1; l < p->k; ++l)
    if (static_cast<long long>(p->level_h[l]) * p->level_w[l] < 2) return SQUAD_ERR_UNSUPPORTED;
  return SQUAD_OK;
}

// The single-pass problem of `level` (p checked). Level 0: the windows of h_1 x w_1 tokens over all
// frames, a local pass. Level p >= 1: with hb, wb the products of the levels below and gy, gx the
// number of level-p blocks along H and W, the rows of one (b, head, frame, block row) form a grid
// (1, hb h_p gx, wb w_p) whose window (1, hb gx, wb) has exactly h_p x w_p windows; its slots are the
// level-p sequences, a global pass. A token's linear row (b h n + token) is the same in every view.
inline void kpass_level_params(const squad_kpass_params_t* p, int level, squad_params_t* s) {
  std::memset(s, 0, sizeof(*s));
  s->d = p->d;
  s->dtype = p->dtype;
  s->scale = p->scale;
  if (level == 0) {
    s->B = p->B;
    s->h = p->h;
    s->T = p->T;
    s->H = p->H;
    s->W = p->W;
    s->tw = p->T;
    s->hw = p->level_h[0];
    s->ww = p->level_w[0];
    s->order = SQUAD_LOCAL_ONLY;
    return;
  }
  long long hb = 1, wb = 1;
  for (int q = 0; q < level; ++q) {
    hb *= p->level_h[q];
    wb *= p->level_w[q];
  }
  const long long hu = hb * p->level_h[level], wu = wb * p->level_w[level];
  const long long gy = p->H / hu, gx = p->W / wu;
  s->B = static_cast<int>(static_cast<long long>(p->B) * p->h * p->T * gy);
  s->h = 1;
  s->T = 1;
  s->H = static_cast<int>(hu * gx);
  s->W = static_cast<int>(wu);
  s->tw = 1;
  s->hw = static_cast<int>(hb * gx);
  s->ww = static_cast<int>(wb);
  s->order = SQUAD_GLOBAL_ONLY;
}

// Level of the pass at position e of the execution order.
inline int kpass_exec_level(const squad_kpass_params_t* p, int e) {
  return p->order == SQUAD_KPASS_FORWARD ? e : p->k - 1 - e;
}

// Intermediate outputs of the forward (k - 1) and value-gradient buffers of the backward.
inline int kpass_n_inter(int k) { return k - 1; }
inline int kpass_n_gbuf(int k) { return k - 1 < 2 ? k - 1 : 2; }

// Forward step e (0 <= e < k): values are v or the previous step's output; the last step writes o.
inline KpassFwdStep kpass_fwd_step(const squad_kpass_params_t* p, int e) {
  KpassFwdStep s;
  s.level = kpass_exec_level(p, e);
  s.values = e == 0 ? kBufV : e - 1;
  s.out = e + 1 == p->k ? kBufO : e;
  s.lse = e;
  s.work = 1 + e;
  return s;
}

// Backward step for executed pass e, run for e = k-1 down to 0: the last executed pass starts from
// dout; every pass hands the gradient of its values to the pass before it, alternating between the
// two buffers counting from the last pass (k - 1 - e = 0, 1, 0, ...), and the first writes dv. The
// first step done starts the fp32 dQ/dK shares, the last (e = 0) writes dq and dk.
inline KpassBwdStep kpass_bwd_step(const squad_kpass_params_t* p, int e) {
  KpassBwdStep s;
  s.level = kpass_exec_level(p, e);
  s.values = e == 0 ? kBufV : e - 1;
  s.g_in = e + 1 == p->k ? kBufDout : (p->k - 2 - e) % 2;
  s.g_out = e == 0 ? kBufDv : (p->k - 1 - e) % 2;
  s.lse = e;
  s.accumulate = e + 1 < p->k;
  s.final_out = e == 0;
  return s;
}

}  // namespace squad
