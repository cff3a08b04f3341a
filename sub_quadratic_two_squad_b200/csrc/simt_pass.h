// Arguments and launchers of the CUDA-core attention kernels (attn_simt.cu).
#pragma once

#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct SimtFwdArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;        // [B, h, n] natural-log LSE, or null
  Grid g;
  PassGeom p;
  float scale;
  int in_bf16;       // q, k are bf16 (else fp32)
  int v_bf16;        // v is bf16
  int out_bf16;      // out is bf16
};

struct SimtBwdArgs {
  const void* q;
  const void* k;
  const void* v;     // this pass's values
  const void* dout;  // upstream gradient of this pass's output
  const float* lse;  // this pass's forward LSE
  float* Drow;       // [B, h, n] scratch: D_i = sum_j P_ij dP_ij
  float* dq_acc;     // fp32 accumulators of dQ and dK across the two passes
  float* dk_acc;
  void* dq_out;      // final gradients (written when final_out)
  void* dk_out;
  void* dv_out;      // gradient of this pass's values
  Grid g;
  PassGeom p;
  float scale;
  int in_bf16, v_bf16, dout_bf16, grad_bf16, dv_bf16;
  int accumulate;    // add the accumulators' contents (the other pass's share)
  int final_out;     // write dq/dk to dq_out/dk_out in the gradient dtype instead of the accumulators
};

cudaError_t launch_simt_fwd(const SimtFwdArgs& a, cudaStream_t stream);
cudaError_t launch_simt_bwd(const SimtBwdArgs& a, cudaStream_t stream);

}  // namespace squad
