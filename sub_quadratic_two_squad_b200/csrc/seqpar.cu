// squad_seqpar_reorder: the block reorderings of the sequence split around its all-to-all exchanges.
//
// Both passes of SQuad-Attention attend inside groups that one re-indexing of the tokens makes
// contiguous (agihunt.info digest, the paragraph that defines the operator: the axis a pass does not
// attend over is folded into the batch of heads), so a block's tokens can be split over R ranks with one
// exchange between the passes. A tensor of the split is a stack of blocks of Hb*W*d contiguous elements
// (Hb = H/R latent rows of one frame of one head), indexed by (b, head, r, tg), r < R, tg < Tg = T/R:
//   band   [B, h, R, Tg]  the rows [rank*Hb, (rank+1)*Hb) of every frame t = r*Tg + tg (the local pass)
//   frames [B, h, Tg, R]  every row band r of the frames [rank*Tg, (rank+1)*Tg) (the global pass)
//   chunks [R, B, h, Tg]  the all-to-all buffer: chunk r goes to (or came from) rank r
// A reordering moves whole blocks; with `add`, each element is the sum of the moved value and add's
// element at the same output position, in fp32, rounded once to the tensor dtype.
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "squad_attn.h"

namespace {

struct ReorderShape {
  int B, h, R, Tg;
  int from, to;
  uint32_t vec;   // 16-byte pieces per block
};

// Index of block (b, hd, r, tg) in a layout.
__device__ __forceinline__ size_t block_index(const ReorderShape& s, int layout, int b, int hd, int r, int tg) {
  if (layout == SQUAD_SP_BAND) return ((static_cast<size_t>(b) * s.h + hd) * s.R + r) * s.Tg + tg;
  if (layout == SQUAD_SP_FRAMES) return ((static_cast<size_t>(b) * s.h + hd) * s.Tg + tg) * s.R + r;
  return ((static_cast<size_t>(r) * s.B + b) * s.h + hd) * s.Tg + tg;   // chunks
}

// (b, hd, r, tg) of block `i` of a layout.
__device__ __forceinline__ void block_coords(const ReorderShape& s, int layout, size_t i, int& b, int& hd, int& r,
                                             int& tg) {
  if (layout == SQUAD_SP_BAND) {
    tg = static_cast<int>(i % s.Tg); i /= s.Tg;
    r = static_cast<int>(i % s.R); i /= s.R;
    hd = static_cast<int>(i % s.h); b = static_cast<int>(i / s.h);
  } else if (layout == SQUAD_SP_FRAMES) {
    r = static_cast<int>(i % s.R); i /= s.R;
    tg = static_cast<int>(i % s.Tg); i /= s.Tg;
    hd = static_cast<int>(i % s.h); b = static_cast<int>(i / s.h);
  } else {
    tg = static_cast<int>(i % s.Tg); i /= s.Tg;
    hd = static_cast<int>(i % s.h); i /= s.h;
    b = static_cast<int>(i % s.B); r = static_cast<int>(i / s.B);
  }
}

__device__ __forceinline__ uint32_t add_bf16x2(uint32_t x, uint32_t a) {
  const float lo = __uint_as_float(x << 16) + __uint_as_float(a << 16);
  const float hi = __uint_as_float(x & 0xFFFF0000u) + __uint_as_float(a & 0xFFFF0000u);
  const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// kAdd: 0 copy, 1 bf16 sum, 2 fp32 sum. A work item is a segment of kSegPieces 16-byte pieces of one
// output block; CTAs take items in turn, each thread loads its kPer pieces of the segment before storing
// them (consecutive threads, consecutive pieces: coalesced on both sides).
constexpr int kThreads = 256, kPer = 4;
constexpr uint32_t kSegPieces = kThreads * kPer;

__device__ __forceinline__ uint4 sum_pieces(uint4 v, uint4 a, int kind) {
  if (kind == 1)
    return make_uint4(add_bf16x2(v.x, a.x), add_bf16x2(v.y, a.y), add_bf16x2(v.z, a.z), add_bf16x2(v.w, a.w));
  return make_uint4(__float_as_uint(__uint_as_float(v.x) + __uint_as_float(a.x)),
                    __float_as_uint(__uint_as_float(v.y) + __uint_as_float(a.y)),
                    __float_as_uint(__uint_as_float(v.z) + __uint_as_float(a.z)),
                    __float_as_uint(__uint_as_float(v.w) + __uint_as_float(a.w)));
}

template <int kAdd>
__global__ void __launch_bounds__(kThreads) reorder_kernel(const uint4* __restrict__ x, const uint4* __restrict__ add,
                                                           uint4* __restrict__ y, ReorderShape s) {
  const size_t nblk = static_cast<size_t>(s.B) * s.h * s.R * s.Tg;
  const uint32_t segs = (s.vec + kSegPieces - 1) / kSegPieces;
  const size_t items = nblk * segs;
  for (size_t item = blockIdx.x; item < items; item += gridDim.x) {
    const size_t blk = item / segs;
    const uint32_t v0 = static_cast<uint32_t>(item - blk * segs) * kSegPieces + threadIdx.x;
    int b, hd, r, tg;
    block_coords(s, s.to, blk, b, hd, r, tg);
    const uint4* src = x + block_index(s, s.from, b, hd, r, tg) * s.vec;
    uint4 val[kPer], a[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t v = v0 + j * kThreads;
      if (v < s.vec) {
        val[j] = src[v];
        if constexpr (kAdd != 0) a[j] = add[blk * s.vec + v];
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t v = v0 + j * kThreads;
      if (v < s.vec) y[blk * s.vec + v] = kAdd != 0 ? sum_pieces(val[j], a[j], kAdd) : val[j];
    }
  }
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" squad_status_t squad_seqpar_reorder(const squad_params_t* p, int R, int from, int to, const void* x,
                                               const void* add, void* y, squad_stream_t stream) {
  if (p == nullptr || R < 1 || p->B < 1 || p->h < 1 || p->T < 1 || p->H < 1 || p->W < 1) return SQUAD_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SQUAD_ERR_INVALID_ARG;
  if (p->dtype != SQUAD_BF16 && p->dtype != SQUAD_FP32) return SQUAD_ERR_INVALID_ARG;
  if (p->T % R != 0 || p->H % R != 0) return SQUAD_ERR_INVALID_ARG;
  if (from < SQUAD_SP_BAND || from > SQUAD_SP_CHUNKS || to < SQUAD_SP_BAND || to > SQUAD_SP_CHUNKS)
    return SQUAD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || x == y || add == y || (add != nullptr && !aligned16(add)))
    return SQUAD_ERR_INVALID_ARG;
  const size_t esize = p->dtype == SQUAD_BF16 ? 2u : 4u;
  const size_t block_bytes = static_cast<size_t>(p->H / R) * p->W * p->d * esize;   // a multiple of 128
  if (block_bytes / 16u > 0x7FFFFFFFull) return SQUAD_ERR_UNSUPPORTED;   // piece indices stay 32-bit
  ReorderShape s{p->B, p->h, R, p->T / R, from, to, static_cast<uint32_t>(block_bytes / 16u)};
  const size_t items = static_cast<size_t>(p->B) * p->h * p->T *   // R * Tg blocks per (b, head), in segments
                       ((s.vec + kSegPieces - 1) / kSegPieces);
  const unsigned grid = static_cast<unsigned>(items < 148u * 4u ? items : 148u * 4u);   // 4 CTAs per SM fit
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint4* xs = static_cast<const uint4*>(x);
  const uint4* as = static_cast<const uint4*>(add);
  uint4* ys = static_cast<uint4*>(y);
  if (add == nullptr)
    reorder_kernel<0><<<grid, kThreads, 0, st>>>(xs, nullptr, ys, s);
  else if (p->dtype == SQUAD_BF16)
    reorder_kernel<1><<<grid, kThreads, 0, st>>>(xs, as, ys, s);
  else
    reorder_kernel<2><<<grid, kThreads, 0, st>>>(xs, as, ys, s);
  return cudaGetLastError() == cudaSuccess ? SQUAD_OK : SQUAD_ERR_CUDA;
}
