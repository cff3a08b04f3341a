// Arguments and launcher of the short-sequence attention kernel (attn_short.cu): one attention pass
// over sequences of at most 256 tokens, each loaded whole as one TMA box.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct ShortPassArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_o;   // bf16 maps whose box is one whole sequence (SWIZZLE_128B)
  Grid g;
  PassGeom p;                           // one chunk per sequence (make_geom(..., 256))
  int global_variant;
  float* lse;                           // [B, h, n] natural-log LSE, or null
  float scale_log2;                     // softmax scale * log2(e)
  uint32_t* status;                     // device status word (0 = ok, 4 = a wait timed out)
  unsigned long long timeout_ns;
  // shared-memory plan (short_pass_plan)
  int n_slots;
  uint32_t panel_bytes;                 // rows (rounded to 8) x 128 bytes
  uint32_t slot_bytes;                  // 2 panels
  uint32_t guard_bytes;                 // readable slack past the ring for tile reads past a slot
  uint32_t smem_bytes;
};

// Fills the shared-memory plan of `a` for sequences of a.p.seq_len tokens; false if they do not fit.
bool short_pass_plan(ShortPassArgs& a);
cudaError_t launch_short_pass(const ShortPassArgs& args, int num_sms, cudaStream_t stream);

}  // namespace squad
