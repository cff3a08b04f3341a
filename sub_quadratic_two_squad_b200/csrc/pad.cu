// Reflect padding of the latent grid for windows that do not divide it, and its adjoints (SQuad paper,
// appendix "Conformance to the theoretical curves is quantitative", which names reflect padding as the
// way such grids are handled). Each frame is padded at the bottom (H) and the right
// (W) end up to a multiple of the window; reflect = the edge token is not repeated, so padded index
// i >= size reads index 2 (size - 1) - i. Tensors are [B*h, T, H, W, d] rows of d elements.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "pad.h"

namespace squad {

namespace {

__device__ __forceinline__ int reflect_src(int i, int size) { return i < size ? i : 2 * (size - 1) - i; }

// dst (padded grid) <- src: every 16-byte piece of every padded token row. zero_fill: padded tokens
// become zeros instead of reflected copies (the adjoint of cropping).
__global__ void pad_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, PadShape s, int zero_fill) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.Hp * s.Wp * s.vec;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int v = static_cast<int>(i % s.vec);
    size_t tok = i / s.vec;
    const int xp = static_cast<int>(tok % s.Wp);
    tok /= s.Wp;
    const int yp = static_cast<int>(tok % s.Hp);
    const size_t frame = tok / s.Hp;   // bh * T + t
    if (zero_fill && (yp >= s.H || xp >= s.W)) {
      dst[i] = make_uint4(0, 0, 0, 0);
    } else {
      const size_t st = (frame * s.H + reflect_src(yp, s.H)) * s.W + reflect_src(xp, s.W);
      dst[i] = src[st * s.vec + v];
    }
  }
}

// dst (original grid) <- the original tokens of src (padded grid).
__global__ void crop_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, PadShape s) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.H * s.W * s.vec;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int v = static_cast<int>(i % s.vec);
    size_t tok = i / s.vec;
    const int x = static_cast<int>(tok % s.W);
    tok /= s.W;
    const int y = static_cast<int>(tok % s.H);
    const size_t frame = tok / s.H;
    dst[i] = src[((frame * s.Hp + y) * s.Wp + x) * s.vec + v];
  }
}

__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_elem(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, size_t i, float x) { p[i] = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elem(float* p, size_t i, float x) { p[i] = x; }

// Adjoint of the reflect padding: an original token's gradient is the sum over the padded tokens that
// copy it (itself, its reflection below the bottom edge, right of the right edge, and both), in fp32.
template <typename E>
__global__ void fold_kernel(const E* __restrict__ src, E* __restrict__ dst, PadShape s) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.H * s.W * s.d;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % s.d);
    size_t tok = i / s.d;
    const int x = static_cast<int>(tok % s.W);
    tok /= s.W;
    const int y = static_cast<int>(tok % s.H);
    const size_t frame = tok / s.H;
    const int yr = 2 * (s.H - 1) - y, xr = 2 * (s.W - 1) - x;   // the padded indices that reflect onto y, x
    const bool has_y = yr >= s.H && yr < s.Hp, has_x = xr >= s.W && xr < s.Wp;
    auto at = [&](int yy, int xx) { return load_elem(src, ((frame * s.Hp + yy) * s.Wp + xx) * s.d + c); };
    float acc = at(y, x);
    if (has_y) acc += at(yr, x);
    if (has_x) acc += at(y, xr);
    if (has_y && has_x) acc += at(yr, xr);
    store_elem(dst, i, acc);
  }
}

unsigned blocks_for(size_t work) {
  const size_t b = (work + 255) / 256;
  return static_cast<unsigned>(b < 148u * 16u ? (b == 0 ? 1 : b) : 148u * 16u);
}

}  // namespace

cudaError_t launch_reflect_pad(const void* src, void* dst, const PadShape& s, bool zero_fill, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.Hp * s.Wp * s.vec;
  pad_kernel<<<blocks_for(total), 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), s,
                                                    zero_fill ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_crop(const void* src, void* dst, const PadShape& s, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.H * s.W * s.vec;
  crop_kernel<<<blocks_for(total), 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), s);
  return cudaGetLastError();
}

cudaError_t launch_fold(const void* src, void* dst, const PadShape& s, bool bf16, cudaStream_t stream) {
  const size_t total = static_cast<size_t>(s.BH) * s.T * s.H * s.W * s.d;
  if (bf16)
    fold_kernel<<<blocks_for(total), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(src),
                                                       static_cast<__nv_bfloat16*>(dst), s);
  else
    fold_kernel<<<blocks_for(total), 256, 0, stream>>>(static_cast<const float*>(src), static_cast<float*>(dst), s);
  return cudaGetLastError();
}

}  // namespace squad
