// Sequence geometry of one attention pass: which tokens form each sequence, and how a sequence is cut
// into chunks of at most 128 rows (one tensor-core tile of queries, or one block of keys/values).
//
// SQuad re-indexes the [B, h, n, d] token grid in two ways (paper §3.2 "Construction of the local and
// global token views"; agihunt.info digest: each pass takes the axis it attends over as its sequence
// and merges the remaining index into the batch of heads):
//   LOCAL  sequence sigma = window c = (wy, wx), rows ordered (t, dy, dx): "lines" are frames t,
//          each line is the hw x ww block of one frame.
//   GLOBAL sequence sigma = slot j = (t, dy, dx), rows ordered (wy, wx): "lines" are window rows wy,
//          each line is the W/ww windows of that row.
//   FULL   one sequence of all n tokens in order (plain softmax attention, paper eq. 5); lines are
//          single tokens.
// A chunk is L whole lines (L * line_len <= 128, or <= 256 for the short-sequence kernel), so every
// chunk of a sequence is one rectangular TMA box of the tensor, and lines past the end of the
// sequence fall outside the tensor (zero fill).
#pragma once

#include <cstdint>

namespace squad {

// Division by a divisor fixed at launch, as one high multiply and a shift: for d >= 2 with
// L = ceil(log2 d), m = ceil(2^(31+L) / d) and s = L - 1, floor(n / d) = floor(n * m / 2^(31+L)) for
// every 0 <= n < 2^31 (m / 2^(31+L) exceeds 1/d by less than 2^-(31+L), so n times the excess stays
// below 2^-L <= 1/d and cannot carry floor(n/d) past the next integer). d == 1 is stored as m = 0.
struct FastDiv {
  uint32_t d, m, s;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  if (d <= 1) return f;
  uint32_t L = 0;
  while ((1ull << L) < d) ++L;
  f.m = static_cast<uint32_t>(((1ull << (31 + L)) + d - 1) / d);
  f.s = L - 1;
  return f;
}

__host__ __device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  if (f.m == 0) return n;
#ifdef __CUDA_ARCH__
  return __umulhi(n, f.m) >> f.s;
#else
  return static_cast<uint32_t>((static_cast<unsigned long long>(n) * f.m) >> 32) >> f.s;
#endif
}

enum PassKind : int { kLocal = 0, kGlobal = 1, kFull = 2 };

struct Grid {
  int B, h, d;
  int T, H, W;
  int hw, ww;           // window (tw == T)
  int n;                // T*H*W
  int nwy, nwx;         // H/hw, W/ww
  FastDiv f_nwx, f_ww, f_hwww;   // divisions by nwx, ww and hw*ww
};

__host__ __device__ inline void finish_grid(Grid& g) {
  g.f_nwx = make_fastdiv(static_cast<uint32_t>(g.nwx));
  g.f_ww = make_fastdiv(static_cast<uint32_t>(g.ww));
  g.f_hwww = make_fastdiv(static_cast<uint32_t>(g.hw * g.ww));
}

struct PassGeom {
  int kind;
  int n_seq;            // sequences per (b, head)
  int seq_len;          // tokens per sequence
  int line_len;         // tokens per line
  int n_lines;          // lines per sequence
  int lines_per_chunk;  // L
  int n_chunks;         // ceil(n_lines / L)
  int chunk_rows;       // L * line_len  (rows of one TMA box, <= 128)
  FastDiv f_line, f_chunks, f_per_bh;   // divisions by line_len, n_chunks and n_seq * n_chunks
};

// max_rows: most rows per chunk (128 for the chunked kernels; 256 makes a sequence of up to 256 tokens
// one chunk).
__host__ __device__ inline PassGeom make_geom(const Grid& g, int kind, int max_rows = 128) {
  PassGeom p{};
  p.kind = kind;
  if (kind == kLocal) {
    p.n_seq = g.nwy * g.nwx;
    p.line_len = g.hw * g.ww;
    p.n_lines = g.T;
  } else if (kind == kGlobal) {
    p.n_seq = g.T * g.hw * g.ww;
    p.line_len = g.nwx;
    p.n_lines = g.nwy;
  } else {
    p.n_seq = 1;
    p.line_len = 1;
    p.n_lines = g.n;
  }
  p.seq_len = p.line_len * p.n_lines;
  // Whole lines per chunk, at most 128 rows; a line longer than 128 rows is one chunk by itself (only
  // the CUDA-core kernels accept such chunks).
  p.lines_per_chunk = p.line_len > max_rows ? 1 : max_rows / p.line_len;
  if (p.lines_per_chunk > p.n_lines) p.lines_per_chunk = p.n_lines;
  p.n_chunks = (p.n_lines + p.lines_per_chunk - 1) / p.lines_per_chunk;
  p.chunk_rows = p.lines_per_chunk * p.line_len;
  p.f_line = make_fastdiv(static_cast<uint32_t>(p.line_len));
  p.f_chunks = make_fastdiv(static_cast<uint32_t>(p.n_chunks));
  p.f_per_bh = make_fastdiv(static_cast<uint32_t>(p.n_seq * p.n_chunks));
  return p;
}

// Token index (within one (b, head)) of row `r` of chunk `q` of sequence `sigma`; -1 when the row is
// padding: past the chunk's box, or past the end of the sequence.
__host__ __device__ inline int token_of(const Grid& g, const PassGeom& p, int sigma, int q, int r) {
  if (r >= p.chunk_rows) return -1;
  const int rl = static_cast<int>(fdiv(static_cast<uint32_t>(r), p.f_line));
  const int line = q * p.lines_per_chunk + rl;
  if (line >= p.n_lines) return -1;
  const int pos = r - rl * p.line_len;
  if (p.kind == kFull) return line;
  int t, y, x;
  if (p.kind == kLocal) {
    const int wy = static_cast<int>(fdiv(static_cast<uint32_t>(sigma), g.f_nwx)), wx = sigma - wy * g.nwx;
    const int dy = static_cast<int>(fdiv(static_cast<uint32_t>(pos), g.f_ww)), dx = pos - dy * g.ww;
    t = line;
    y = wy * g.hw + dy;
    x = wx * g.ww + dx;
  } else {
    t = static_cast<int>(fdiv(static_cast<uint32_t>(sigma), g.f_hwww));
    const int rem = sigma - t * g.hw * g.ww;
    const int dy = static_cast<int>(fdiv(static_cast<uint32_t>(rem), g.f_ww)), dx = rem - dy * g.ww;
    y = line * g.hw + dy;
    x = pos * g.ww + dx;
  }
  return (t * g.H + y) * g.W + x;
}

// TMA view of a [B, h, n, d] bf16 tensor for one pass: dims/strides/box/element strides as given to
// cuTensorMapEncodeTiled (innermost first). The box of chunk q of a sequence holds its rows in order.
// LOCAL  : view (d, W, H, T, BH), box (64, ww, hw, L, 1).
// GLOBAL : variant 0, view (d, W, H, T, BH), box (64, W, L*hw, 1, 1) traversed every ww-th x and
//          every hw-th y (element strides), i.e. one token per window of L window rows.
//          variant 1, view (d, W/ww, H/hw, ww, BH*T*H) with strides (ww d, hw W d, d, W d) elements,
//          box (64, W/ww, L, 1, 1) with unit element strides.
// FULL   : view (d, n, BH, 1, 1), box (64, L, 1, 1, 1).
struct MapDesc {
  unsigned long long dims[5];
  unsigned long long strides[4];   // bytes, for dims 1..4
  unsigned int box[5];
  unsigned int es[5];
};

inline MapDesc describe_pass_map(const Grid& g, const PassGeom& p, int variant, unsigned long long elem_bytes) {
  MapDesc m{};
  const unsigned long long d = g.d, eb = elem_bytes, BH = static_cast<unsigned long long>(g.B) * g.h;
  for (int i = 0; i < 5; ++i) m.es[i] = 1;
  if (p.kind == kLocal || (p.kind == kGlobal && variant == 0)) {
    m.dims[0] = d; m.dims[1] = g.W; m.dims[2] = g.H; m.dims[3] = g.T; m.dims[4] = BH;
    m.strides[0] = d * eb;
    m.strides[1] = static_cast<unsigned long long>(g.W) * d * eb;
    m.strides[2] = static_cast<unsigned long long>(g.H) * g.W * d * eb;
    m.strides[3] = static_cast<unsigned long long>(g.n) * d * eb;
    if (p.kind == kLocal) {
      m.box[0] = 64; m.box[1] = g.ww; m.box[2] = g.hw; m.box[3] = p.lines_per_chunk; m.box[4] = 1;
    } else {
      m.box[0] = 64; m.box[1] = g.nwx * g.ww; m.box[2] = p.lines_per_chunk * g.hw; m.box[3] = 1; m.box[4] = 1;
      m.es[1] = g.ww;
      m.es[2] = g.hw;
    }
  } else if (p.kind == kGlobal) {
    m.dims[0] = d; m.dims[1] = g.nwx; m.dims[2] = g.nwy; m.dims[3] = g.ww;
    m.dims[4] = BH * g.T * g.H;
    m.strides[0] = static_cast<unsigned long long>(g.ww) * d * eb;
    m.strides[1] = static_cast<unsigned long long>(g.hw) * g.W * d * eb;
    m.strides[2] = d * eb;
    m.strides[3] = static_cast<unsigned long long>(g.W) * d * eb;
    m.box[0] = 64; m.box[1] = g.nwx; m.box[2] = p.lines_per_chunk; m.box[3] = 1; m.box[4] = 1;
  } else {
    m.dims[0] = d; m.dims[1] = g.n; m.dims[2] = BH; m.dims[3] = 1; m.dims[4] = 1;
    m.strides[0] = d * eb;
    m.strides[1] = static_cast<unsigned long long>(g.n) * d * eb;
    m.strides[2] = BH * g.n * d * eb;
    m.strides[3] = m.strides[2];
    m.box[0] = 64; m.box[1] = p.lines_per_chunk; m.box[2] = 1; m.box[3] = 1; m.box[4] = 1;
  }
  return m;
}

// TMA box origin of chunk `chunk` of sequence `sigma` of head `bh`, d-panel `panel` (64 columns).
__host__ __device__ inline void chunk_coords(const Grid& g, const PassGeom& p, int variant, int bh, int sigma,
                                             int chunk, int panel, int c[5]) {
  c[0] = panel * 64;
  if (p.kind == kLocal) {
    const int wy = static_cast<int>(fdiv(static_cast<uint32_t>(sigma), g.f_nwx)), wx = sigma - wy * g.nwx;
    c[1] = wx * g.ww;
    c[2] = wy * g.hw;
    c[3] = chunk * p.lines_per_chunk;
    c[4] = bh;
  } else if (p.kind == kGlobal) {
    const int tt = static_cast<int>(fdiv(static_cast<uint32_t>(sigma), g.f_hwww));
    const int rem = sigma - tt * g.hw * g.ww;
    const int dy = static_cast<int>(fdiv(static_cast<uint32_t>(rem), g.f_ww)), dx = rem - dy * g.ww;
    if (variant == 0) {
      c[1] = dx;
      c[2] = dy + chunk * p.lines_per_chunk * g.hw;
      c[3] = tt;
      c[4] = bh;
    } else {
      c[1] = 0;
      c[2] = chunk * p.lines_per_chunk;
      c[3] = dx;
      c[4] = (bh * g.T + tt) * g.H + dy;
    }
  } else {
    c[1] = chunk * p.lines_per_chunk;
    c[2] = bh;
    c[3] = 0;
    c[4] = 0;
  }
}

// Number of valid rows of chunk q (rows past the sequence end are padding).
__host__ __device__ inline int chunk_valid_rows(const PassGeom& p, int q) {
  int lines = p.n_lines - q * p.lines_per_chunk;
  if (lines > p.lines_per_chunk) lines = p.lines_per_chunk;
  return lines * p.line_len;
}

}  // namespace squad
