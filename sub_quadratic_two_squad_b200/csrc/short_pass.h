// Arguments and launcher of the fused short-sequence attention kernel (attn_short.cu): one or both
// SQuad passes over sequences of at most 256 tokens in one persistent launch, each sequence loaded
// whole as one TMA box.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct ShortPass {
  CUtensorMap tm_q, tm_k, tm_v, tm_o;   // bf16 maps whose box is one whole sequence (SWIZZLE_128B)
  PassGeom p;                           // one chunk per sequence (make_geom(..., 256))
  int variant;                          // slot-box encoding (GLOBAL pass)
  float* lse;                           // [B, h, n] natural-log LSE of this pass, or null
  uint32_t panel_bytes;                 // rows (rounded to 8) x 128 bytes
  uint32_t alloc_bytes;                 // one ring allocation: 2 panels
  int units_per_head;                   // sequences (>128 tokens) or sequence pairs (<=128) per head
};

struct ShortArgs {
  ShortPass pass[2];
  Grid g;
  int n_passes;        // 1, or 2: pass[1] reads pass[0]'s output as its values
  int lag;             // heads by which a head's second-pass units trail its first-pass units
  FastDiv f_u0, f_u1, f_u01;   // divisions by the per-head unit counts (pass 0, pass 1, both)
  float scale_log2;    // softmax scale * log2(e)
  uint32_t* status;    // device status word (0 = ok, 4 = a wait timed out)
  uint32_t* work;      // work counter, zero before the launch
  uint32_t* done;      // [B*h] first-pass units of each head whose output is in memory, zero before
                       // the launch (two passes only)
  unsigned long long timeout_ns;
  uint32_t ring_bytes, guard_bytes, smem_bytes;
};

// Fills the unit counts and shared-memory plan of `a` (pass geometries and n_passes set); false if
// the sequences do not fit.
bool short_plan(ShortArgs& a);
cudaError_t launch_short(const ShortArgs& args, int num_sms, cudaStream_t stream);

}  // namespace squad
