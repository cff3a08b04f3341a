// Arguments and launchers of the tensor-core backward kernels (bwd_tc.cu): one SQuad pass's gradients
// over sequences of at most 208 tokens, each sequence loaded whole (Q, K, V, dO) as TMA boxes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "geometry.cuh"

namespace squad {

struct BwdTcArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // bf16 maps whose box is one whole sequence (SWIZZLE_128B)
  Grid g;
  PassGeom p;                 // one chunk per sequence (make_geom(..., 256))
  int variant;                // slot-box encoding (GLOBAL pass)
  const float* lse;           // [B, h, n] natural-log LSE of this pass's forward
  const __nv_bfloat16* o;     // [B, h, n, d] this pass's output (D_i = dO_i . O_i)
  float* dq_acc;              // [B, h, n, d] fp32 share of dQ: written, added to (accumulate), or read
                              // and completed (final_out with accumulate)
  float* dk_acc;              // [B, h, n, d] fp32 share of dK (likewise)
  __nv_bfloat16* dq_out;      // final dQ (final_out only)
  __nv_bfloat16* dk_out;      // final dK (final_out only)
  __nv_bfloat16* dv_out;      // gradient of this pass's values
  float scale, scale_log2;
  int final_out;              // write dq_out / dk_out (bf16) instead of the fp32 shares
  int accumulate;             // add the fp32 shares already in dq_acc / dk_acc (earlier passes') first
  int single;                 // sequences of at most 128 tokens: the one-tile kernel (no recomputation)
  int pack;                   // sequences per CTA of the one-tile kernel (128 / seg_rows)
  int seg_rows;               // rows of one sequence's band in its tiles (the length rounded up to 8)
  uint32_t panel_bytes;       // rows (rounded to 8) x 128 bytes
  uint32_t guard_bytes, smem_bytes;
  uint32_t* status;           // device status word (0 = ok, 4 = a wait timed out)
  unsigned long long timeout_ns;
  uint8_t* pds;               // whole-sequence kernel: kBwdPdsSlots slots of pds_slot_bytes (P and dS of
                              // one sequence, bf16, written in the row phase, read by the column phase)
  uint32_t pds_slot_bytes;
};

// Scratch of the whole-sequence backward: one slot per resident CTA, each holding a sequence's P and dS
// (bf16) in the layout of two 128-key operand tiles (two 64-key panels of at most 208 rows, 128-byte
// swizzle): 8 panels of at most 208 x 128 bytes.
constexpr int kBwdPdsSlots = 160;
constexpr size_t kBwdPdsSlotMaxBytes = 8u * 208u * 128u;
constexpr size_t kBwdPdsScratchBytes = static_cast<size_t>(kBwdPdsSlots) * kBwdPdsSlotMaxBytes;

// Fills the shared-memory plan of `a` (p and g set); false if the sequences do not fit.
bool bwd_tc_plan(BwdTcArgs& a);
// One pass's gradients: dQ, then dK and dV, in one persistent launch (the two-tile kernel needs `pds`).
cudaError_t launch_bwd_tc(const BwdTcArgs& a, cudaStream_t stream);

}  // namespace squad
