// Reflect padding of the latent grid and its adjoints (pad.cu).
#pragma once

#include <cuda_runtime.h>

namespace squad {

struct PadShape {
  int BH, T;      // frames = BH * T
  int H, W;       // original grid
  int Hp, Wp;     // padded grid (multiples of the window)
  int d;          // elements per token row
  int vec;        // 16-byte pieces per token row (d * element bytes / 16)
};

// dst [BH, T, Hp, Wp, d] from src [BH, T, H, W, d]: reflected copies at the padded tokens, or zeros
// there when zero_fill (the adjoint of cropping). Whole 16-byte pieces; both buffers 16-byte aligned.
cudaError_t launch_reflect_pad(const void* src, void* dst, const PadShape& s, bool zero_fill, cudaStream_t stream);
// dst [BH, T, H, W, d] <- the original tokens of src [BH, T, Hp, Wp, d].
cudaError_t launch_crop(const void* src, void* dst, const PadShape& s, cudaStream_t stream);
// dst [BH, T, H, W, d] <- each original token's sum over its padded copies in src (bf16 or fp32 both ways).
cudaError_t launch_fold(const void* src, void* dst, const PadShape& s, bool bf16, cudaStream_t stream);

}  // namespace squad
