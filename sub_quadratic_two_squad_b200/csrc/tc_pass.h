// Arguments and launcher of the tensor-core attention pass kernel (attn_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "geometry.cuh"

namespace squad {

struct TcPassArgs {
  CUtensorMap tm_q, tm_k, tm_v;   // bf16 tensor maps with the pass's chunk box (SWIZZLE_128B)
  CUtensorMap tm_o;               // the same box over the output (tiled TMA stores)
  Grid g;
  PassGeom p;
  int global_variant;             // slot-box encoding used for the GLOBAL pass maps (see tmap.cpp)
  float* lse;                     // [B, h, n] natural-log LSE, or null
  float scale_log2;               // softmax scale * log2(e)
  uint32_t* status;               // device status word (0 = ok, 4 = a wait timed out)
  unsigned long long timeout_ns;  // limit of every device-side wait
};

cudaError_t launch_tc_pass(const TcPassArgs& args, int num_sms, cudaStream_t stream);

}  // namespace squad
