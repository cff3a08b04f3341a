// C ABI of the SQuad-Attention library (include/squad_attn.h): argument validation, TMA tensor maps
// for the window and slot views, and the launch sequence of the two passes.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "squad_attn.h"
#include "geometry.cuh"
#include "host_util.h"
#include "kpass_plan.h"
#include "bwd_pass.h"
#include "bwd_stream.h"
#include "pack_pass.h"
#include "pad.h"
#include "short_pass.h"
#include "simt_pass.h"
#include "tc_pass.h"

using namespace squad;

namespace {

constexpr int kAbiVersion = 1;
// Control block at the start of a workspace (zeroed by every call): word 0 the device status, words
// 1-3 work counters of the persistent kernels, then one counter per (b, head) for the fused passes.
constexpr size_t kCtrlFixedWords = 4;
// Run both passes of a short-sequence problem in one persistent launch (second pass trailing the first
// by two heads, reading it from L2); otherwise one launch per pass.
constexpr bool kFusePasses = true;
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;   // 1 s per device-side wait

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void* p, size_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The caller's grid when the window does not divide it: the kernels run on the padded grid.
struct PadDims {
  int H0 = 0, W0 = 0;   // original extents
  bool padded = false;
};

// Validates the parameters and fills the grid description. `windowed` = SQuad call (window fields
// and order are used); false = full attention (only B, h, d, T, H, W, dtype, scale). For a window
// that does not divide H x W, *g is the grid reflect-padded at the bottom and right up to multiples
// of the window (SQuad paper appendix, "Conformance to the theoretical curves is quantitative"), and
// *pd keeps the original extents.
squad_status_t validate(const squad_params_t* p, bool windowed, Grid* g, float* scale, PadDims* pd = nullptr) {
  if (p == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (p->B < 1 || p->h < 1 || p->T < 1 || p->H < 1 || p->W < 1) return SQUAD_ERR_INVALID_ARG;
  if (p->dtype != SQUAD_BF16 && p->dtype != SQUAD_FP32) return SQUAD_ERR_INVALID_ARG;
  if (p->d < 1) return SQUAD_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SQUAD_ERR_UNSUPPORTED;
  if (!(p->scale >= 0.f) || !std::isfinite(p->scale)) return SQUAD_ERR_INVALID_ARG;
  int H = p->H, W = p->W;
  if (windowed && p->hw >= 1 && p->ww >= 1) {   // padded extents (reflect padding is shorter than the extent
    H = (p->H + p->hw - 1) / p->hw * p->hw;     // whenever hw <= H and ww <= W, checked below)
    W = (p->W + p->ww - 1) / p->ww * p->ww;
  }
  const long long n = static_cast<long long>(p->T) * H * W;
  if (n > (1ll << 30)) return SQUAD_ERR_UNSUPPORTED;
  const long long bhn = static_cast<long long>(p->B) * p->h * n;
  if (bhn > (1ll << 31) - 1) return SQUAD_ERR_UNSUPPORTED;
  Grid gg{};
  gg.B = p->B;
  gg.h = p->h;
  gg.d = p->d;
  gg.T = p->T;
  gg.H = H;
  gg.W = W;
  gg.n = static_cast<int>(n);
  if (windowed) {
    if (p->order < SQUAD_LOCAL_THEN_GLOBAL || p->order > SQUAD_GLOBAL_ONLY) return SQUAD_ERR_INVALID_ARG;
    if (p->tw < 1 || p->hw < 1 || p->ww < 1) return SQUAD_ERR_INVALID_ARG;
    if (p->tw > p->T || p->hw > p->H || p->ww > p->W) return SQUAD_ERR_INVALID_ARG;
    // The window covers every frame (tw < T is outside the method); space is tiled by the window over
    // the (padded) grid.
    if (p->tw != p->T) return SQUAD_ERR_UNSUPPORTED;
    gg.hw = p->hw;
    gg.ww = p->ww;
    gg.nwy = H / p->hw;
    gg.nwx = W / p->ww;
  } else {
    gg.hw = 1;
    gg.ww = 1;
    gg.nwy = p->H;
    gg.nwx = p->W;
  }
  finish_grid(gg);
  *g = gg;
  if (pd != nullptr) {
    pd->H0 = p->H;
    pd->W0 = p->W;
    pd->padded = H != p->H || W != p->W;
  }
  *scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->d));
  return SQUAD_OK;
}

size_t elem_bytes(const squad_params_t* p) { return p->dtype == SQUAD_BF16 ? 2 : 4; }

size_t ctrl_bytes(const Grid& g) {
  return align256(4 * (kCtrlFixedWords + static_cast<size_t>(g.B) * g.h));
}

struct FwdWorkspace {
  uint32_t* status;   // control block (ctrl_bytes)
  void* o1;
  float* lse1;
  float* lse2;
  void *qp, *kp, *vp, *op;   // padded grids only: the padded q, k, v (kept for the backward) and output
};

size_t fwd_ws_bytes(const Grid& g, size_t eb, bool padded) {
  const size_t bhn = static_cast<size_t>(g.B) * g.h * g.n;
  const size_t t = align256(bhn * g.d * eb);
  return ctrl_bytes(g) + t + 2 * align256(bhn * 4) + (padded ? 4 * t : 0);
}

FwdWorkspace carve_fwd(void* ws, const Grid& g, size_t eb, bool padded) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t bhn = static_cast<size_t>(g.B) * g.h * g.n;
  const size_t t = align256(bhn * g.d * eb);
  FwdWorkspace w;
  w.status = reinterpret_cast<uint32_t*>(b);
  b += ctrl_bytes(g);
  w.o1 = b;
  b += t;
  w.lse1 = reinterpret_cast<float*>(b);
  b += align256(bhn * 4);
  w.lse2 = reinterpret_cast<float*>(b);
  b += align256(bhn * 4);
  w.qp = w.kp = w.vp = w.op = nullptr;
  if (padded) {
    w.qp = b;
    w.kp = b + t;
    w.vp = b + 2 * t;
    w.op = b + 3 * t;
  }
  return w;
}

struct BwdWorkspace {
  uint32_t* status;
  float* dq_acc;
  float* dk_acc;
  float* do1;
  float* drow;
  void *dop, *dqp, *dkp, *dvp;   // padded grids only: dout zero-padded, gradients on the padded grid
  uint8_t* pds;                  // the whole-sequence kernel's P/dS scratch slots (last; may be empty)
};

size_t bwd_ws_bytes(const Grid& g, size_t eb, bool padded) {
  const size_t bhn = static_cast<size_t>(g.B) * g.h * g.n;
  return ctrl_bytes(g) + 3 * align256(bhn * g.d * 4) + align256(bhn * 4) + (padded ? 4 * align256(bhn * g.d * eb) : 0);
}

size_t pds_bytes(const squad_params_t* sp, const Grid& g);

BwdWorkspace carve_bwd(void* ws, const Grid& g, size_t eb, bool padded) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t bhn = static_cast<size_t>(g.B) * g.h * g.n;
  BwdWorkspace w;
  w.status = reinterpret_cast<uint32_t*>(b);
  b += ctrl_bytes(g);
  w.dq_acc = reinterpret_cast<float*>(b);
  b += align256(bhn * g.d * 4);
  w.dk_acc = reinterpret_cast<float*>(b);
  b += align256(bhn * g.d * 4);
  w.do1 = reinterpret_cast<float*>(b);
  b += align256(bhn * g.d * 4);
  w.drow = reinterpret_cast<float*>(b);
  b += align256(bhn * 4);
  w.dop = w.dqp = w.dkp = w.dvp = nullptr;
  if (padded) {
    const size_t t = align256(bhn * g.d * eb);
    w.dop = b;
    w.dqp = b + t;
    w.dkp = b + 2 * t;
    w.dvp = b + 3 * t;
    b += 4 * t;
  }
  w.pds = b;
  return w;
}

PadShape pad_shape(const Grid& g, const PadDims& pd, size_t eb) {
  PadShape s;
  s.BH = g.B * g.h;
  s.T = g.T;
  s.H = pd.H0;
  s.W = pd.W0;
  s.Hp = g.H;
  s.Wp = g.W;
  s.d = g.d;
  s.vec = static_cast<int>(g.d * eb / 16);
  return s;
}

// ------------------------------------------------------------------------------------------------
// TMA tensor maps: each pass's sequences are boxes of the caller's [B, h, n, d] tensor
// ------------------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Slot-box encoding for the GLOBAL pass: a view with dims (d, wx, wy, dx, (bh*T+t)*H+dy) whose box
// has unit element strides (geometry.cuh, variant 1). Tiled TMA stores use the same maps, and they
// are only defined for unit element strides.
constexpr int kSlotBoxVariant = 1;

bool encode_pass_map(CUtensorMap* m, const void* base, const Grid& g, const PassGeom& p, int variant) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const MapDesc d = describe_pass_map(g, p, variant, 2);
  for (int i = 0; i < 5; ++i)
    if (d.box[i] < 1 || d.box[i] > 256 || d.es[i] < 1 || d.es[i] > 8) return false;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5], es[5];
  for (int i = 0; i < 5; ++i) {
    dims[i] = d.dims[i];
    box[i] = d.box[i];
    es[i] = d.es[i];
  }
  for (int i = 0; i < 4; ++i) strides[i] = d.strides[i];
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The tensor-core kernel handles bf16, d = 128, and chunks of whole lines of at most 128 rows.
bool tc_eligible(const squad_params_t* prm, const Grid& g, const PassGeom& p) {
  if (prm->dtype != SQUAD_BF16 || g.d != 128) return false;
  if (p.line_len > 128 || p.chunk_rows < 1 || p.chunk_rows > 128) return false;
  if (p.kind == kGlobal && (g.W > 256 || p.lines_per_chunk * g.hw > 256)) return false;
  return true;
}


// Sequences of at most 256 tokens run whole (one TMA box, one K/V block) in the short-sequence kernel.
bool short_eligible(const squad_params_t* prm, const Grid& g, const PassGeom& p) {
  return prm->dtype == SQUAD_BF16 && g.d == 128 && p.kind != kFull && p.seq_len <= 256 && p.n_chunks == 1;
}

bool fill_short_pass(ShortPass& sp, const Grid& g, int kind, const void* q, const void* k, const void* v, void* out,
                     float* lse) {
  sp.p = make_geom(g, kind, 256);
  sp.variant = kind == kGlobal ? kSlotBoxVariant : 0;
  sp.lse = lse;
  return encode_pass_map(&sp.tm_q, q, g, sp.p, sp.variant) && encode_pass_map(&sp.tm_k, k, g, sp.p, sp.variant) &&
         encode_pass_map(&sp.tm_v, v, g, sp.p, sp.variant) && encode_pass_map(&sp.tm_o, out, g, sp.p, sp.variant);
}

squad_status_t launch_short_args(ShortArgs& a, float scale, uint32_t* status, uint32_t* work, uint32_t* done,
                                 cudaStream_t stream) {
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = status;
  a.work = work;
  a.done = done;
  a.timeout_ns = kWaitTimeoutNs;
  const int sms = num_sms_current();
  if (sms <= 0) return SQUAD_ERR_CUDA;
  return launch_short(a, sms, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}

// One attention pass: out = softmax(scale q k^T) v over the sequences of `kind`. `work` is a zeroed
// counter for the persistent short-sequence kernel.
squad_status_t run_pass(const squad_params_t* prm, const Grid& g, int kind, float scale, const void* q,
                        const void* k, const void* v, bool v_bf16, void* out, float* lse, uint32_t* status,
                        uint32_t* work, cudaStream_t stream) {
  if (prm->dtype == SQUAD_BF16 && v_bf16) {
    // sequences of at most 64 tokens: several per 128-row tile
    PackFwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.g = g;
    a.p = make_geom(g, kind, 256);
    if (pack_eligible(g, a.p)) {
      a.variant = kind == kGlobal ? kSlotBoxVariant : 0;
      if (!encode_pass_map(&a.tm_q, q, g, a.p, a.variant) || !encode_pass_map(&a.tm_k, k, g, a.p, a.variant) ||
          !encode_pass_map(&a.tm_v, v, g, a.p, a.variant))
        return SQUAD_ERR_CUDA;
      pack_plan(a);
      a.out = static_cast<__nv_bfloat16*>(out);
      a.lse = lse;
      a.scale_log2 = scale * 1.4426950408889634f;
      a.status = status;
      a.timeout_ns = kWaitTimeoutNs;
      return launch_pack_fwd(a, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
    }
  }
  if (short_eligible(prm, g, make_geom(g, kind, 256)) && v_bf16 && work != nullptr) {
    ShortArgs a;
    std::memset(&a, 0, sizeof(a));
    a.g = g;
    a.n_passes = 1;
    if (!fill_short_pass(a.pass[0], g, kind, q, k, v, out, lse)) return SQUAD_ERR_CUDA;
    if (short_plan(a)) return launch_short_args(a, scale, status, work, nullptr, stream);
  }
  const PassGeom p = make_geom(g, kind);
  if (tc_eligible(prm, g, p) && v_bf16) {
    TcPassArgs a;
    std::memset(&a, 0, sizeof(a));
    const int variant = kind == kGlobal ? kSlotBoxVariant : 0;
    if (!encode_pass_map(&a.tm_q, q, g, p, variant) || !encode_pass_map(&a.tm_k, k, g, p, variant) ||
        !encode_pass_map(&a.tm_v, v, g, p, variant) || !encode_pass_map(&a.tm_o, out, g, p, variant))
      return SQUAD_ERR_CUDA;
    a.g = g;
    a.p = p;
    a.global_variant = variant;
    a.lse = lse;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.status = status;
    a.timeout_ns = kWaitTimeoutNs;
    const int sms = num_sms_current();
    if (sms <= 0) return SQUAD_ERR_CUDA;
    return launch_tc_pass(a, sms, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
  }
  SimtFwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.g = g;
  a.p = p;
  a.scale = scale;
  a.in_bf16 = prm->dtype == SQUAD_BF16;
  a.v_bf16 = v_bf16;
  a.out_bf16 = prm->dtype == SQUAD_BF16;
  return launch_simt_fwd(a, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}

}  // namespace

extern "C" {

int squad_attn_abi_version(void) { return kAbiVersion; }

const char* squad_status_string(squad_status_t s) {
  switch (s) {
    case SQUAD_OK: return "ok";
    case SQUAD_ERR_INVALID_ARG: return "invalid argument";
    case SQUAD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SQUAD_ERR_CUDA: return "CUDA error";
    case SQUAD_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

double squad_attn_flops(const squad_params_t* p) {
  Grid g;
  float sc;
  if (validate(p, true, &g, &sc) != SQUAD_OK) return 0.0;
  const double w = static_cast<double>(p->tw) * p->hw * p->ww;
  const double n = g.n;
  const double local = n * w, global = n * n / w;   // per (b, head, d): n rows x sequence length
  const double terms = p->order == SQUAD_LOCAL_ONLY ? local : p->order == SQUAD_GLOBAL_ONLY ? global : local + global;
  return 4.0 * p->B * p->h * p->d * terms;
}

squad_status_t squad_window_solve(int T, int H, int W, int* tw, int* hw, int* ww) {
  if (T < 1 || H < 1 || W < 1 || tw == nullptr || hw == nullptr || ww == nullptr) return SQUAD_ERR_INVALID_ARG;
  double best = 0.0;
  int best_h = 0, best_w = 0;
  for (int h = 1; h <= H; ++h) {
    // the width whose ratio h:w is closest to H:W (log ratio), of the two around h*W/H
    const int lo = std::max(1, static_cast<int>(std::floor(static_cast<double>(h) * W / H)));
    const double target = std::log(static_cast<double>(H) / W);
    const double e_lo = std::fabs(std::log(static_cast<double>(h) / lo) - target);
    const double e_hi = std::fabs(std::log(static_cast<double>(h) / (lo + 1)) - target);
    const int w = e_hi < e_lo ? lo + 1 : lo;
    if (w > W) continue;
    const double hp = static_cast<double>((H + h - 1) / h * h), wp = static_cast<double>((W + w - 1) / w * w);
    const double np = static_cast<double>(T) * hp * wp, m = static_cast<double>(T) * h * w;
    const double cost = np * m + np * np / m;
    if (best_h == 0 || cost < best) {
      best = cost;
      best_h = h;
      best_w = w;
    }
  }
  *tw = T;
  *hw = best_h;
  *ww = best_w;
  return SQUAD_OK;
}

double full_attn_flops(const squad_params_t* p) {
  Grid g;
  float sc;
  if (validate(p, false, &g, &sc) != SQUAD_OK) return 0.0;
  const double n = g.n;
  return 4.0 * p->B * p->h * p->d * n * n;
}

size_t squad_attn_fwd_workspace_bytes(const squad_params_t* p) {
  Grid g;
  float sc;
  PadDims pd;
  if (validate(p, true, &g, &sc, &pd) != SQUAD_OK) return 0;
  return fwd_ws_bytes(g, elem_bytes(p), pd.padded);
}

size_t squad_attn_bwd_workspace_bytes(const squad_params_t* p) {
  Grid g;
  float sc;
  PadDims pd;
  if (validate(p, true, &g, &sc, &pd) != SQUAD_OK) return 0;
  return bwd_ws_bytes(g, elem_bytes(p), pd.padded) + pds_bytes(p, g);
}

}  // extern "C"

namespace {

// The forward on the kernels' grid g (already padded where needed); the control block is zeroed.
squad_status_t fwd_core(const squad_params_t* p, const Grid& g, float scale, const void* q, const void* k,
                        const void* v, void* o, const FwdWorkspace& ws, cudaStream_t stream) {
  squad_status_t st;
  const bool bf16 = p->dtype == SQUAD_BF16;
  uint32_t* ctrl = ws.status;
  if (p->order == SQUAD_LOCAL_ONLY || p->order == SQUAD_GLOBAL_ONLY) {
    // one pass straight into o; its LSE goes where the first pass's would (the backward reads it there)
    const int kind = p->order == SQUAD_LOCAL_ONLY ? kLocal : kGlobal;
    return run_pass(p, g, kind, scale, q, k, v, bf16, o, ws.lse1, ctrl, ctrl + 2, stream);
  }
  const int first = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kLocal : kGlobal;
  const int second = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kGlobal : kLocal;
  if (kFusePasses && short_eligible(p, g, make_geom(g, first, 256)) && short_eligible(p, g, make_geom(g, second, 256))) {
    // Both passes in one persistent launch; the second pass reads each head's first-pass output
    // (its values) once all of that head's first-pass units are stored.
    ShortArgs a;
    std::memset(&a, 0, sizeof(a));
    a.g = g;
    a.n_passes = 2;
    if (!fill_short_pass(a.pass[0], g, first, q, k, v, ws.o1, ws.lse1) ||
        !fill_short_pass(a.pass[1], g, second, q, k, ws.o1, o, ws.lse2))
      return SQUAD_ERR_CUDA;
    if (short_plan(a)) return launch_short_args(a, scale, ctrl, ctrl + 1, ctrl + kCtrlFixedWords, stream);
  }
  st = run_pass(p, g, first, scale, q, k, v, bf16, ws.o1, ws.lse1, ctrl, ctrl + 2, stream);
  if (st != SQUAD_OK) return st;
  return run_pass(p, g, second, scale, q, k, ws.o1, bf16, o, ws.lse2, ctrl, ctrl + 3, stream);
}

}  // namespace

extern "C" {

squad_status_t squad_attn_fwd(const squad_params_t* p, const void* q, const void* k, const void* v, void* o,
                              void* workspace, squad_stream_t stream_) {
  Grid g;
  float scale;
  PadDims pd;
  squad_status_t st = validate(p, true, &g, &scale, &pd);
  if (st != SQUAD_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(workspace, 256))
    return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const size_t eb = elem_bytes(p);
  FwdWorkspace ws = carve_fwd(workspace, g, eb, pd.padded);
  if (cudaMemsetAsync(ws.status, 0, ctrl_bytes(g), stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  if (!pd.padded) return fwd_core(p, g, scale, q, k, v, o, ws, stream);
  // Reflect-pad q, k, v into the workspace, run on the padded grid, crop the output into o.
  const PadShape ps = pad_shape(g, pd, eb);
  if (launch_reflect_pad(q, ws.qp, ps, false, stream) != cudaSuccess ||
      launch_reflect_pad(k, ws.kp, ps, false, stream) != cudaSuccess ||
      launch_reflect_pad(v, ws.vp, ps, false, stream) != cudaSuccess)
    return SQUAD_ERR_CUDA;
  st = fwd_core(p, g, scale, ws.qp, ws.kp, ws.vp, ws.op, ws, stream);
  if (st != SQUAD_OK) return st;
  return launch_crop(ws.op, o, ps, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}

squad_status_t squad_attn_fwd_status(const squad_params_t* p, const void* workspace, squad_stream_t stream_) {
  Grid g;
  float scale;
  squad_status_t st = validate(p, true, &g, &scale);
  if (st != SQUAD_OK) return st;
  if (!aligned(workspace, 256)) return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return SQUAD_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  return word == 0 ? SQUAD_OK : SQUAD_ERR_TIMEOUT;
}

}  // extern "C"

namespace {

// The backward kernel of one pass (SQUAD_BWD_*): whole sequences on the tensor cores where the
// shared-memory plan fits, else chunks of whole lines on the tensor cores, else the CUDA cores.
int bwd_kernel_of(const squad_params_t* sp, const Grid& g, int kind) {
  if (sp->dtype == SQUAD_BF16) {
    BwdTcArgs b;
    std::memset(&b, 0, sizeof(b));
    b.g = g;
    b.p = make_geom(g, kind, 256);
    if (short_eligible(sp, g, b.p) && bwd_tc_plan(b)) return SQUAD_BWD_TC_WHOLE;
    if (g.d == 128 && bwd_stream_eligible(g, make_geom(g, kind))) return SQUAD_BWD_TC_CHUNKED;
  }
  return SQUAD_BWD_CUDA_CORE;
}

// Bytes of P/dS scratch the whole-sequence backward kernel needs for either pass of this problem (0
// when no pass of more than 128 tokens runs on it).
size_t pds_bytes(const squad_params_t* sp, const Grid& g) {
  size_t m = 0;
  if (sp->dtype != SQUAD_BF16) return 0;
  for (const int kind : {kLocal, kGlobal}) {
    if ((kind == kLocal && sp->order == SQUAD_GLOBAL_ONLY) || (kind == kGlobal && sp->order == SQUAD_LOCAL_ONLY))
      continue;   // a pass this order does not run
    BwdTcArgs b;
    std::memset(&b, 0, sizeof(b));
    b.g = g;
    b.p = make_geom(g, kind, 256);
    if (short_eligible(sp, g, b.p) && bwd_tc_plan(b) && !b.single)
      m = std::max(m, static_cast<size_t>(kBwdPdsSlots) * b.pds_slot_bytes);
  }
  return align256(m);
}

// One pass's backward inside a chain of passes. accumulate: add the fp32 dQ/dK shares already in the
// accumulators; final_out: write dq, dk (input dtype) instead of the accumulators. dv_out receives the
// gradient of this pass's values in the input dtype; out is this pass's forward output (the chunked
// kernels form D from it).
squad_status_t bwd_one_pass(const squad_params_t* sp, const Grid& g, int kind, float scale, const void* q,
                            const void* k, const void* values, const void* out, const void* dout, const float* lse,
                            uint32_t* status, float* dq_acc, float* dk_acc, float* drow, void* dq, void* dk,
                            void* dv_out, bool accumulate, bool final_out, uint8_t* pds, cudaStream_t stream) {
  const bool bf16 = sp->dtype == SQUAD_BF16;
  const int kernel = bwd_kernel_of(sp, g, kind);
  if (kernel == SQUAD_BWD_TC_WHOLE) {
    BwdTcArgs b;
    std::memset(&b, 0, sizeof(b));
    b.g = g;
    b.p = make_geom(g, kind, 256);
    if (bwd_tc_plan(b)) {
      b.variant = kind == kGlobal ? kSlotBoxVariant : 0;
      if (!encode_pass_map(&b.tm_q, q, g, b.p, b.variant) || !encode_pass_map(&b.tm_k, k, g, b.p, b.variant) ||
          !encode_pass_map(&b.tm_v, values, g, b.p, b.variant) || !encode_pass_map(&b.tm_do, dout, g, b.p, b.variant))
        return SQUAD_ERR_CUDA;
      b.lse = lse;
      b.o = static_cast<const __nv_bfloat16*>(out);
      b.dq_acc = dq_acc;
      b.dk_acc = dk_acc;
      b.dq_out = static_cast<__nv_bfloat16*>(dq);
      b.dk_out = static_cast<__nv_bfloat16*>(dk);
      b.dv_out = static_cast<__nv_bfloat16*>(dv_out);
      b.final_out = final_out ? 1 : 0;
      b.accumulate = accumulate ? 1 : 0;
      b.scale = scale;
      b.scale_log2 = scale * 1.4426950408889634f;
      b.status = status;
      b.timeout_ns = kWaitTimeoutNs;
      b.pds = pds;
      return launch_bwd_tc(b, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
    }
  }
  if (kernel == SQUAD_BWD_TC_CHUNKED) {
    // Longer sequences: the chunked tensor-core kernels (D from the pass output `out`).
    BwdStreamArgs s;
    std::memset(&s, 0, sizeof(s));
    s.g = g;
    s.p = make_geom(g, kind);
    s.variant = kind == kGlobal ? kSlotBoxVariant : 0;
    if (!encode_pass_map(&s.tm_q, q, g, s.p, s.variant) || !encode_pass_map(&s.tm_k, k, g, s.p, s.variant) ||
        !encode_pass_map(&s.tm_v, values, g, s.p, s.variant) ||
        !encode_pass_map(&s.tm_do, dout, g, s.p, s.variant) || !encode_pass_map(&s.tm_o, out, g, s.p, s.variant))
      return SQUAD_ERR_CUDA;
    s.lse = lse;
    s.drow = drow;
    s.dq_acc = dq_acc;
    s.dk_acc = dk_acc;
    s.dq_out = static_cast<__nv_bfloat16*>(dq);
    s.dk_out = static_cast<__nv_bfloat16*>(dk);
    s.dv_out = static_cast<__nv_bfloat16*>(dv_out);
    s.final_out = final_out ? 1 : 0;
    s.accumulate = accumulate ? 1 : 0;
    s.scale = scale;
    s.scale_log2 = scale * 1.4426950408889634f;
    s.status = status;
    s.timeout_ns = kWaitTimeoutNs;
    return launch_bwd_stream(s, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
  }
  SimtBwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = values;
  a.dout = dout;
  a.lse = lse;
  a.Drow = drow;
  a.dq_acc = dq_acc;
  a.dk_acc = dk_acc;
  a.dq_out = dq;
  a.dk_out = dk;
  a.dv_out = dv_out;
  a.g = g;
  a.p = make_geom(g, kind);
  a.scale = scale;
  a.in_bf16 = bf16;
  a.v_bf16 = bf16;
  a.dout_bf16 = bf16;
  a.grad_bf16 = bf16;
  a.dv_bf16 = bf16;
  a.accumulate = accumulate ? 1 : 0;
  a.final_out = final_out ? 1 : 0;
  return launch_simt_bwd(a, stream) == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}

// The backward on the kernels' grid g (already padded where needed); the control block is zeroed.
squad_status_t bwd_core(const squad_params_t* p, const Grid& g, float scale, const void* q, const void* k,
                        const void* v, const void* o, const void* dout, const FwdWorkspace& fw,
                        const BwdWorkspace& bw, void* dq, void* dk, void* dv, cudaStream_t stream) {
  const bool bf16 = p->dtype == SQUAD_BF16;
  if (p->order == SQUAD_LOCAL_ONLY || p->order == SQUAD_GLOBAL_ONLY) {
    // One pass: values v, upstream dout, the pass's LSE in the first slot; no share to add.
    const int kind = p->order == SQUAD_LOCAL_ONLY ? kLocal : kGlobal;
    return bwd_one_pass(p, g, kind, scale, q, k, v, o, dout, fw.lse1, bw.status, bw.dq_acc, bw.dk_acc, bw.drow,
                        dq, dk, dv, /*accumulate=*/false, /*final_out=*/true, bw.pds, stream);
  }
  const int first = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kLocal : kGlobal;
  const int second = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kGlobal : kLocal;

  if (bf16) {
    // Tensor-core kernels when every sequence of both passes fits one CTA: pass 2 first (values O1,
    // upstream dout; gives the dQ, dK shares and dO1 in bf16), then pass 1 (values v, upstream dO1;
    // completes dQ, dK and gives dV).
    BwdTcArgs b2, b1;
    std::memset(&b2, 0, sizeof(b2));
    b2.g = g;
    b2.p = make_geom(g, second, 256);
    b1 = b2;
    b1.p = make_geom(g, first, 256);
    if (short_eligible(p, g, b2.p) && short_eligible(p, g, b1.p) && bwd_tc_plan(b2) && bwd_tc_plan(b1)) {
      __nv_bfloat16* do1 = reinterpret_cast<__nv_bfloat16*>(bw.do1);
      b2.variant = second == kGlobal ? kSlotBoxVariant : 0;
      b1.variant = first == kGlobal ? kSlotBoxVariant : 0;
      if (!encode_pass_map(&b2.tm_q, q, g, b2.p, b2.variant) || !encode_pass_map(&b2.tm_k, k, g, b2.p, b2.variant) ||
          !encode_pass_map(&b2.tm_v, fw.o1, g, b2.p, b2.variant) ||
          !encode_pass_map(&b2.tm_do, dout, g, b2.p, b2.variant) ||
          !encode_pass_map(&b1.tm_q, q, g, b1.p, b1.variant) || !encode_pass_map(&b1.tm_k, k, g, b1.p, b1.variant) ||
          !encode_pass_map(&b1.tm_v, v, g, b1.p, b1.variant) || !encode_pass_map(&b1.tm_do, do1, g, b1.p, b1.variant))
        return SQUAD_ERR_CUDA;
      for (BwdTcArgs* b : {&b2, &b1}) {
        b->dq_acc = bw.dq_acc;
        b->dk_acc = bw.dk_acc;
        b->scale = scale;
        b->scale_log2 = scale * 1.4426950408889634f;
        b->status = bw.status;
        b->timeout_ns = kWaitTimeoutNs;
        b->pds = bw.pds;
      }
      b2.lse = fw.lse2;
      b2.o = static_cast<const __nv_bfloat16*>(o);
      b2.dv_out = do1;
      b2.final_out = 0;
      b1.lse = fw.lse1;
      b1.o = static_cast<const __nv_bfloat16*>(fw.o1);
      b1.dq_out = static_cast<__nv_bfloat16*>(dq);
      b1.dk_out = static_cast<__nv_bfloat16*>(dk);
      b1.dv_out = static_cast<__nv_bfloat16*>(dv);
      b1.final_out = 1;
      b1.accumulate = 1;
      if (launch_bwd_tc(b2, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
      if (launch_bwd_tc(b1, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
      return SQUAD_OK;
    }
    if (bwd_kernel_of(p, g, second) != SQUAD_BWD_CUDA_CORE || bwd_kernel_of(p, g, first) != SQUAD_BWD_CUDA_CORE) {
      // Pass by pass, each on the kernel that takes its sequences (whole-sequence or chunked tensor
      // cores); dO1 is bf16 as in the fused pair.
      squad_status_t st = bwd_one_pass(p, g, second, scale, q, k, fw.o1, o, dout, fw.lse2, bw.status, bw.dq_acc,
                                       bw.dk_acc, bw.drow, dq, dk, bw.do1, /*accumulate=*/false,
                                       /*final_out=*/false, bw.pds, stream);
      if (st != SQUAD_OK) return st;
      return bwd_one_pass(p, g, first, scale, q, k, v, fw.o1, bw.do1, fw.lse1, bw.status, bw.dq_acc, bw.dk_acc,
                          bw.drow, dq, dk, dv, /*accumulate=*/true, /*final_out=*/true, bw.pds, stream);
    }
  }

  // Pass 2 backward: values = O1 (pass-1 output), upstream = dout. Gives dQ, dK shares and dO1.
  SimtBwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = fw.o1;
  a.dout = dout;
  a.lse = fw.lse2;
  a.Drow = bw.drow;
  a.dq_acc = bw.dq_acc;
  a.dk_acc = bw.dk_acc;
  a.dq_out = dq;
  a.dk_out = dk;
  a.dv_out = bw.do1;
  a.g = g;
  a.p = make_geom(g, second);
  a.scale = scale;
  a.in_bf16 = bf16;
  a.v_bf16 = bf16;
  a.dout_bf16 = bf16;
  a.grad_bf16 = bf16;
  a.dv_bf16 = 0;
  a.accumulate = 0;
  a.final_out = 0;
  if (launch_simt_bwd(a, stream) != cudaSuccess) return SQUAD_ERR_CUDA;

  // Pass 1 backward: values = v, upstream = dO1. Adds its dQ, dK shares and gives dV.
  a.v = v;
  a.dout = bw.do1;
  a.lse = fw.lse1;
  a.dv_out = dv;
  a.p = make_geom(g, first);
  a.dout_bf16 = 0;
  a.dv_bf16 = bf16;
  a.accumulate = 1;
  a.final_out = 1;
  if (launch_simt_bwd(a, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  return SQUAD_OK;
}

}  // namespace

extern "C" {

squad_status_t squad_attn_bwd(const squad_params_t* p, const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const void* fwd_workspace, void* dq, void* dk, void* dv,
                              void* bwd_workspace, squad_stream_t stream_) {
  Grid g;
  float scale;
  PadDims pd;
  squad_status_t st = validate(p, true, &g, &scale, &pd);
  if (st != SQUAD_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(fwd_workspace, 256) ||
      !aligned(bwd_workspace, 256))
    return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const size_t eb = elem_bytes(p);
  FwdWorkspace fw = carve_fwd(const_cast<void*>(fwd_workspace), g, eb, pd.padded);
  BwdWorkspace bw = carve_bwd(bwd_workspace, g, eb, pd.padded);
  if (cudaMemsetAsync(bw.status, 0, ctrl_bytes(g), stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  if (!pd.padded) return bwd_core(p, g, scale, q, k, v, o, dout, fw, bw, dq, dk, dv, stream);
  // The padded method: dout is zero on the padded tokens (the adjoint of the crop); the padded q, k, v
  // and output are the forward workspace's; each input token's gradient sums over its padded copies.
  const PadShape ps = pad_shape(g, pd, eb);
  if (launch_reflect_pad(dout, bw.dop, ps, true, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  st = bwd_core(p, g, scale, fw.qp, fw.kp, fw.vp, fw.op, bw.dop, fw, bw, bw.dqp, bw.dkp, bw.dvp, stream);
  if (st != SQUAD_OK) return st;
  const bool bf16 = p->dtype == SQUAD_BF16;
  if (launch_fold(bw.dqp, dq, ps, bf16, stream) != cudaSuccess || launch_fold(bw.dkp, dk, ps, bf16, stream) != cudaSuccess ||
      launch_fold(bw.dvp, dv, ps, bf16, stream) != cudaSuccess)
    return SQUAD_ERR_CUDA;
  return SQUAD_OK;
}

squad_status_t squad_attn_bwd_kernels(const squad_params_t* p, int kernels[2]) {
  Grid g;
  float scale;
  PadDims pd;
  const squad_status_t st = validate(p, true, &g, &scale, &pd);
  if (st != SQUAD_OK) return st;
  if (kernels == nullptr) return SQUAD_ERR_INVALID_ARG;
  kernels[0] = kernels[1] = 0;
  if (p->order == SQUAD_LOCAL_ONLY || p->order == SQUAD_GLOBAL_ONLY) {
    kernels[0] = bwd_kernel_of(p, g, p->order == SQUAD_LOCAL_ONLY ? kLocal : kGlobal);
    return SQUAD_OK;
  }
  const int first = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kLocal : kGlobal;
  const int second = p->order == SQUAD_LOCAL_THEN_GLOBAL ? kGlobal : kLocal;
  kernels[0] = bwd_kernel_of(p, g, first);
  kernels[1] = bwd_kernel_of(p, g, second);
  return SQUAD_OK;
}

squad_status_t full_attn_fwd(const squad_params_t* p, const void* q, const void* k, const void* v, void* o,
                             float* lse_or_null, squad_stream_t stream_) {
  Grid g;
  float scale;
  squad_status_t st = validate(p, false, &g, &scale);
  if (st != SQUAD_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return SQUAD_ERR_INVALID_ARG;
  if (lse_or_null != nullptr && !aligned(lse_or_null, 4)) return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const bool bf16 = p->dtype == SQUAD_BF16;
  return run_pass(p, g, kFull, scale, q, k, v, bf16, o, lse_or_null, nullptr, nullptr, stream);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// k composed passes over nested windows. Each pass is one single-pass problem on a reinterpretation
// of the caller's contiguous [B, h, n, d] buffers: a token's linear row (b h n + token) is the same in
// every view, so outputs, log-sum-exps and the fp32 dQ/dK shares of all passes line up.
// ------------------------------------------------------------------------------------------------

namespace {

constexpr size_t kKpassCtrlBytes = 256;   // word 0 the status, words 1..k the passes' work counters

struct KpassPlan {
  int k;
  squad_params_t sub[SQUAD_KPASS_MAX_LEVELS];   // the single-pass problem of each level
  Grid g[SQUAD_KPASS_MAX_LEVELS];
  int kind[SQUAD_KPASS_MAX_LEVELS];
  float scale;
  size_t eb;                                    // element bytes of the input dtype
  size_t bhn;                                   // B * h * n rows
};

squad_status_t kpass_plan(const squad_kpass_params_t* p, KpassPlan* pl) {
  squad_status_t st = kpass_check(p);
  if (st != SQUAD_OK) return st;
  pl->k = p->k;
  for (int l = 0; l < p->k; ++l) {
    kpass_level_params(p, l, &pl->sub[l]);
    PadDims pd;
    st = validate(&pl->sub[l], true, &pl->g[l], &pl->scale, &pd);
    if (st != SQUAD_OK) return st;
    if (pd.padded) return SQUAD_ERR_INVALID_ARG;   // unreachable: each view's window divides its grid
    pl->kind[l] = l == 0 ? kLocal : kGlobal;
  }
  pl->eb = elem_bytes(&pl->sub[0]);
  pl->bhn = static_cast<size_t>(p->B) * p->h * p->T * p->H * p->W;
  return SQUAD_OK;
}

struct KpassFwdWs {
  uint32_t* ctrl;
  void* inter[SQUAD_KPASS_MAX_LEVELS];   // outputs of executed passes 0 .. k-2 (input dtype)
  float* lse[SQUAD_KPASS_MAX_LEVELS];    // log-sum-exp of executed pass e
};

size_t kpass_fwd_bytes(const KpassPlan& pl) {
  const size_t t = align256(pl.bhn * pl.sub[0].d * pl.eb), l = align256(pl.bhn * 4);
  return kKpassCtrlBytes + static_cast<size_t>(kpass_n_inter(pl.k)) * t + static_cast<size_t>(pl.k) * l;
}

KpassFwdWs carve_kpass_fwd(void* ws, const KpassPlan& pl) {
  const size_t t = align256(pl.bhn * pl.sub[0].d * pl.eb), l = align256(pl.bhn * 4);
  uint8_t* b = static_cast<uint8_t*>(ws);
  KpassFwdWs w{};
  w.ctrl = reinterpret_cast<uint32_t*>(b);
  b += kKpassCtrlBytes;
  for (int e = 0; e < kpass_n_inter(pl.k); ++e, b += t) w.inter[e] = b;
  for (int e = 0; e < pl.k; ++e, b += l) w.lse[e] = reinterpret_cast<float*>(b);
  return w;
}

struct KpassBwdWs {
  uint32_t* ctrl;
  float* dq_acc;    // fp32 dQ and dK shares [B, h, n, d]
  float* dk_acc;
  float* drow;      // [B, h, n] per-row softmax-Jacobian terms (CUDA-core kernels)
  void* gbuf[2];    // value gradients passed between consecutive passes (input dtype)
  uint8_t* pds;     // the whole-sequence kernel's P/dS scratch slots (last; may be empty)
};

// P/dS scratch of the largest whole-sequence level of the chain (0 if none runs on that kernel).
size_t kpass_pds_bytes(const KpassPlan& pl) {
  size_t m = 0;
  for (int l = 0; l < pl.k; ++l) m = std::max(m, pds_bytes(&pl.sub[l], pl.g[l]));
  return m;
}

size_t kpass_bwd_bytes(const KpassPlan& pl) {
  const size_t d = static_cast<size_t>(pl.sub[0].d);
  const size_t t = align256(pl.bhn * d * pl.eb), f = align256(pl.bhn * d * 4), l = align256(pl.bhn * 4);
  return kKpassCtrlBytes + 2 * f + l + static_cast<size_t>(kpass_n_gbuf(pl.k)) * t + kpass_pds_bytes(pl);
}

KpassBwdWs carve_kpass_bwd(void* ws, const KpassPlan& pl) {
  const size_t d = static_cast<size_t>(pl.sub[0].d);
  const size_t t = align256(pl.bhn * d * pl.eb), f = align256(pl.bhn * d * 4), l = align256(pl.bhn * 4);
  uint8_t* b = static_cast<uint8_t*>(ws);
  KpassBwdWs w{};
  w.ctrl = reinterpret_cast<uint32_t*>(b);
  b += kKpassCtrlBytes;
  w.dq_acc = reinterpret_cast<float*>(b);
  b += f;
  w.dk_acc = reinterpret_cast<float*>(b);
  b += f;
  w.drow = reinterpret_cast<float*>(b);
  b += l;
  w.gbuf[0] = kpass_n_gbuf(pl.k) > 0 ? b : nullptr;
  w.gbuf[1] = kpass_n_gbuf(pl.k) > 1 ? b + t : nullptr;
  w.pds = b + static_cast<size_t>(kpass_n_gbuf(pl.k)) * t;
  return w;
}

}  // namespace

extern "C" {

squad_status_t squad_kpass_pass_params(const squad_kpass_params_t* p, int level, squad_params_t* out) {
  if (out == nullptr) return SQUAD_ERR_INVALID_ARG;
  const squad_status_t st = kpass_check(p);
  if (st != SQUAD_OK) return st;
  if (level < 0 || level >= p->k) return SQUAD_ERR_INVALID_ARG;
  squad_params_t s;
  kpass_level_params(p, level, &s);
  Grid g;
  float sc;
  PadDims pd;
  const squad_status_t vs = validate(&s, true, &g, &sc, &pd);
  if (vs != SQUAD_OK) return vs;
  *out = s;
  return SQUAD_OK;
}

size_t squad_kpass_fwd_workspace_bytes(const squad_kpass_params_t* p) {
  KpassPlan pl;
  if (kpass_plan(p, &pl) != SQUAD_OK) return 0;
  return kpass_fwd_bytes(pl);
}

size_t squad_kpass_bwd_workspace_bytes(const squad_kpass_params_t* p) {
  KpassPlan pl;
  if (kpass_plan(p, &pl) != SQUAD_OK) return 0;
  return kpass_bwd_bytes(pl);
}

double squad_kpass_flops(const squad_kpass_params_t* p) {
  KpassPlan pl;
  if (kpass_plan(p, &pl) != SQUAD_OK) return 0.0;
  double total = 0.0;
  for (int l = 0; l < pl.k; ++l) total += squad_attn_flops(&pl.sub[l]);
  return total;
}

squad_status_t squad_kpass_fwd(const squad_kpass_params_t* p, const void* q, const void* k, const void* v, void* o,
                               void* workspace, squad_stream_t stream_) {
  KpassPlan pl;
  const squad_status_t st = kpass_plan(p, &pl);
  if (st != SQUAD_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(workspace, 256))
    return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const KpassFwdWs ws = carve_kpass_fwd(workspace, pl);
  if (cudaMemsetAsync(ws.ctrl, 0, kKpassCtrlBytes, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  const bool bf16 = p->dtype == SQUAD_BF16;
  for (int e = 0; e < pl.k; ++e) {
    const KpassFwdStep st = kpass_fwd_step(p, e);
    const int l = st.level;
    const void* values = st.values == kBufV ? v : ws.inter[st.values];
    void* out = st.out == kBufO ? o : ws.inter[st.out];
    const squad_status_t ps = run_pass(&pl.sub[l], pl.g[l], pl.kind[l], pl.scale, q, k, values, bf16, out,
                                       ws.lse[st.lse], ws.ctrl, ws.ctrl + st.work, stream);
    if (ps != SQUAD_OK) return ps;
  }
  return SQUAD_OK;
}

squad_status_t squad_kpass_bwd(const squad_kpass_params_t* p, const void* q, const void* k, const void* v,
                               const void* o, const void* dout, const void* fwd_workspace, void* dq, void* dk,
                               void* dv, void* bwd_workspace, squad_stream_t stream_) {
  KpassPlan pl;
  const squad_status_t st = kpass_plan(p, &pl);
  if (st != SQUAD_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(fwd_workspace, 256) ||
      !aligned(bwd_workspace, 256))
    return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const KpassFwdWs fw = carve_kpass_fwd(const_cast<void*>(fwd_workspace), pl);
  const KpassBwdWs bw = carve_kpass_bwd(bwd_workspace, pl);
  if (cudaMemsetAsync(bw.ctrl, 0, kKpassCtrlBytes, stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  // Last executed pass first (the schedule of kpass_bwd_step).
  for (int e = pl.k - 1; e >= 0; --e) {
    const KpassBwdStep st = kpass_bwd_step(p, e);
    const int l = st.level;
    const void* values = st.values == kBufV ? v : fw.inter[st.values];
    const void* g_in = st.g_in == kBufDout ? dout : bw.gbuf[st.g_in];
    void* g_out = st.g_out == kBufDv ? dv : bw.gbuf[st.g_out];
    const void* out = e + 1 == p->k ? o : fw.inter[e];   // this pass's output: the next pass's values
    const squad_status_t ps = bwd_one_pass(&pl.sub[l], pl.g[l], pl.kind[l], pl.scale, q, k, values, out, g_in,
                                           fw.lse[st.lse], bw.ctrl, bw.dq_acc, bw.dk_acc, bw.drow, dq, dk, g_out,
                                           st.accumulate, st.final_out, bw.pds, stream);
    if (ps != SQUAD_OK) return ps;
  }
  return SQUAD_OK;
}

squad_status_t squad_kpass_status(const squad_kpass_params_t* p, const void* workspace, squad_stream_t stream_) {
  KpassPlan pl;
  const squad_status_t st = kpass_plan(p, &pl);
  if (st != SQUAD_OK) return st;
  if (!aligned(workspace, 256)) return SQUAD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return SQUAD_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SQUAD_ERR_CUDA;
  return word == 0 ? SQUAD_OK : SQUAD_ERR_TIMEOUT;
}

}  // extern "C"
