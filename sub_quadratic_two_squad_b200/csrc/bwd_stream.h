// Arguments and launcher of the chunked tensor-core backward (bwd_stream.cu): one SQuad pass's
// gradients for sequences of any length, cut into chunks of at most 128 rows, persistent CTAs taking
// the chunks in turn.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct BwdStreamArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_o;   // bf16 maps whose box is one chunk (SWIZZLE_128B); tm_o is
                                               // this pass's output (for D = rowsum(dO o O))
  Grid g;
  PassGeom p;                 // chunks of at most 128 rows (make_geom(..., 128))
  int variant;                // slot-box encoding (GLOBAL pass)
  const float* lse;           // [B, h, n] natural-log LSE of this pass's forward
  float* drow;                // [B, h, n] fp32: D of each query, written by the rows kernel
  float* dq_acc;              // [B, h, n, d] fp32 shares of dQ and dK, as for the whole-sequence kernel
  float* dk_acc;
  __nv_bfloat16* dq_out;      // final dQ, dK (final_out only)
  __nv_bfloat16* dk_out;
  __nv_bfloat16* dv_out;      // gradient of this pass's values
  float scale, scale_log2;
  int final_out;              // write dq_out / dk_out (bf16) instead of the fp32 shares
  int accumulate;             // add the fp32 shares already in dq_acc / dk_acc first
  uint32_t* status;           // device status word (0 = ok, 4 = a wait timed out)
  unsigned long long timeout_ns;
};

// True if the chunked kernels take this pass (bf16 operands assumed by the caller).
bool bwd_stream_eligible(const Grid& g, const PassGeom& p);
// One pass's gradients: the rows kernel (dQ, D), then the columns kernel (dK, dV).
cudaError_t launch_bwd_stream(const BwdStreamArgs& a, cudaStream_t stream);

}  // namespace squad
