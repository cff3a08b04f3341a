// Arguments and launcher of the packed forward pass (attn_pack.cu): one SQuad pass over sequences of
// at most 64 tokens, several sequences per CTA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct PackFwdArgs {
  CUtensorMap tm_q, tm_k, tm_v;   // bf16 maps whose box is one whole sequence (SWIZZLE_128B)
  Grid g;
  PassGeom p;                     // one chunk per sequence (make_geom(..., 256))
  int variant;                    // slot-box encoding (GLOBAL pass)
  int pack;                       // sequences per CTA: 128 / seg_rows
  int seg_rows;                   // rows of one sequence's band (the length rounded up to 8)
  __nv_bfloat16* out;             // [B, h, n, d] pass output
  float* lse;                     // [B, h, n] natural-log LSE, or null
  float scale_log2;               // softmax scale * log2(e)
  uint32_t* status;               // device status word (0 = ok, 4 = a wait timed out)
  unsigned long long timeout_ns;  // limit of every device-side wait
};

// True if the packed kernel takes this pass (bf16 operands, checked by the caller): d = 128 and
// sequences of at most 64 tokens (two or more per 128-row tile).
bool pack_eligible(const Grid& g, const PassGeom& p);
// Fills pack / seg_rows of `a` from a.p.
void pack_plan(PackFwdArgs& a);
cudaError_t launch_pack_fwd(const PackFwdArgs& a, cudaStream_t stream);

}  // namespace squad
