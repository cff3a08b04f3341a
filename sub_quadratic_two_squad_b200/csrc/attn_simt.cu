// CUDA-core (fp32 FMA) attention kernels: the exact fp32 path of SQuad-Attention and the backward pass.
//
// Forward: one warp per query row; the lanes split the head dimension, every score is a warp-reduced
// dot product, softmax is online in fp32 with expf. Used for SQUAD_FP32 (where tensor cores cannot
// reach 1e-5 relative error) and for shapes outside the tensor-core tiling.
//
// Backward of one softmax pass with values V and upstream gradient dO (chain rule; the pages print no
// formula): with P = softmax(scale Q K^T) recomputed from the saved log-sum-exp,
//   dP = dO V^T,  D_i = sum_j P_ij dP_ij,  dS = P o (dP - D),  dQ = scale dS K,  dK = scale dS^T Q,
//   dV = P^T dO.
// Row kernel: dQ and D (one warp per query row). Column kernel: dK and dV (one warp per key row).
// Every token belongs to exactly one sequence per pass, so no atomics are needed; the two passes'
// contributions to dQ and dK are summed through fp32 accumulators.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "geometry.cuh"
#include "simt_pass.h"

namespace squad {

namespace {

__device__ __forceinline__ float ldf(const void* p, size_t i, int bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]) : reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void stf(void* p, size_t i, float v, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[i] = v;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ int seq_token(const Grid& g, const PassGeom& p, int sigma, int j) {
  return token_of(g, p, sigma, j / p.chunk_rows, j - (j / p.chunk_rows) * p.chunk_rows);
}

constexpr int kMaxPer = 4;   // d <= 128 -> at most 4 elements per lane

struct RowRef {
  int bh, sigma, j, tok;
  bool valid;
};
__device__ __forceinline__ RowRef row_ref(const Grid& g, const PassGeom& p) {
  RowRef r;
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long total = static_cast<long long>(g.B) * g.h * p.n_seq * p.seq_len;
  r.valid = w < total;
  if (!r.valid) return r;
  r.j = static_cast<int>(w % p.seq_len);
  r.sigma = static_cast<int>((w / p.seq_len) % p.n_seq);
  r.bh = static_cast<int>(w / (static_cast<long long>(p.seq_len) * p.n_seq));
  r.tok = seq_token(g, p, r.sigma, r.j);
  return r;
}

}  // namespace

__global__ void __launch_bounds__(256) simt_pass_fwd_kernel(SimtFwdArgs a) {
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const RowRef r = row_ref(g, p);
  if (!r.valid) return;
  const int lane = threadIdx.x & 31;
  const int per = g.d / 32;
  const size_t head = static_cast<size_t>(r.bh) * g.n;
  float qv[kMaxPer], acc[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    qv[i] = i < per ? ldf(a.q, (head + r.tok) * g.d + lane + 32 * i, a.in_bf16) : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int jj = 0; jj < p.seq_len; ++jj) {
    const size_t kt = (head + seq_token(g, p, r.sigma, jj)) * g.d;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
      if (i < per) dot = fmaf(qv[i], ldf(a.k, kt + lane + 32 * i, a.in_bf16), dot);
    const float sc = warp_sum(dot) * a.scale;
    const float m_new = fmaxf(m, sc);
    const float corr = expf(m - m_new);
    const float pj = expf(sc - m_new);
    l = fmaf(l, corr, pj);
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
      if (i < per) acc[i] = fmaf(acc[i], corr, pj * ldf(a.v, kt + lane + 32 * i, a.v_bf16));
    m = m_new;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i)
    if (i < per) stf(a.out, (head + r.tok) * g.d + lane + 32 * i, acc[i] * inv, a.out_bf16);
  if (a.lse != nullptr && lane == 0) a.lse[head + r.tok] = m + logf(l);
}

// Row kernel of one pass's backward: dQ (this pass's share, times `scale`) and D_i.
__global__ void __launch_bounds__(256) simt_pass_bwd_rows_kernel(SimtBwdArgs a) {
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const RowRef r = row_ref(g, p);
  if (!r.valid) return;
  const int lane = threadIdx.x & 31;
  const int per = g.d / 32;
  const size_t head = static_cast<size_t>(r.bh) * g.n;
  const size_t row = (head + r.tok) * g.d;
  const float lse = a.lse[head + r.tok];
  float qv[kMaxPer], dov[kMaxPer], dq[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    qv[i] = i < per ? ldf(a.q, row + lane + 32 * i, a.in_bf16) : 0.f;
    dov[i] = i < per ? ldf(a.dout, row + lane + 32 * i, a.dout_bf16) : 0.f;
    dq[i] = 0.f;
  }
  // D_i = sum_j P_ij dP_ij
  float D = 0.f;
  for (int jj = 0; jj < p.seq_len; ++jj) {
    const size_t kt = (head + seq_token(g, p, r.sigma, jj)) * g.d;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
      if (i < per) {
        s = fmaf(qv[i], ldf(a.k, kt + lane + 32 * i, a.in_bf16), s);
        dp = fmaf(dov[i], ldf(a.v, kt + lane + 32 * i, a.v_bf16), dp);
      }
    s = warp_sum(s);
    dp = warp_sum(dp);
    D = fmaf(expf(s * a.scale - lse), dp, D);
  }
  for (int jj = 0; jj < p.seq_len; ++jj) {
    const size_t kt = (head + seq_token(g, p, r.sigma, jj)) * g.d;
    float s = 0.f, dp = 0.f;
    float kv[kMaxPer];
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      kv[i] = i < per ? ldf(a.k, kt + lane + 32 * i, a.in_bf16) : 0.f;
      if (i < per) {
        s = fmaf(qv[i], kv[i], s);
        dp = fmaf(dov[i], ldf(a.v, kt + lane + 32 * i, a.v_bf16), dp);
      }
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float ds = expf(s * a.scale - lse) * (dp - D);
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) dq[i] = fmaf(ds, kv[i], dq[i]);
  }
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    if (i >= per) continue;
    const size_t e = row + lane + 32 * i;
    float v = dq[i] * a.scale;
    if (a.accumulate) v += a.dq_acc[e];
    if (a.final_out)
      stf(a.dq_out, e, v, a.grad_bf16);
    else
      a.dq_acc[e] = v;
  }
  if (lane == 0) a.Drow[head + r.tok] = D;
}

// Column kernel of one pass's backward: dK (this pass's share) and dV for key row `j`.
__global__ void __launch_bounds__(256) simt_pass_bwd_cols_kernel(SimtBwdArgs a) {
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const RowRef r = row_ref(g, p);
  if (!r.valid) return;
  const int lane = threadIdx.x & 31;
  const int per = g.d / 32;
  const size_t head = static_cast<size_t>(r.bh) * g.n;
  const size_t col = (head + r.tok) * g.d;
  float kv[kMaxPer], vv[kMaxPer], dk[kMaxPer], dv[kMaxPer];
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    kv[i] = i < per ? ldf(a.k, col + lane + 32 * i, a.in_bf16) : 0.f;
    vv[i] = i < per ? ldf(a.v, col + lane + 32 * i, a.v_bf16) : 0.f;
    dk[i] = 0.f;
    dv[i] = 0.f;
  }
  for (int ii = 0; ii < p.seq_len; ++ii) {
    const int qt = seq_token(g, p, r.sigma, ii);
    const size_t qrow = (head + qt) * g.d;
    float qv[kMaxPer], dov[kMaxPer];
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      qv[i] = i < per ? ldf(a.q, qrow + lane + 32 * i, a.in_bf16) : 0.f;
      dov[i] = i < per ? ldf(a.dout, qrow + lane + 32 * i, a.dout_bf16) : 0.f;
      s = fmaf(qv[i], kv[i], s);
      dp = fmaf(dov[i], vv[i], dp);
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float pij = expf(s * a.scale - a.lse[head + qt]);
    const float ds = pij * (dp - a.Drow[head + qt]);
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      dk[i] = fmaf(ds, qv[i], dk[i]);
      dv[i] = fmaf(pij, dov[i], dv[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    if (i >= per) continue;
    const size_t e = col + lane + 32 * i;
    float v = dk[i] * a.scale;
    if (a.accumulate) v += a.dk_acc[e];
    if (a.final_out)
      stf(a.dk_out, e, v, a.grad_bf16);
    else
      a.dk_acc[e] = v;
    stf(a.dv_out, e, dv[i], a.dv_bf16);
  }
}

static unsigned rows_grid(const Grid& g, const PassGeom& p) {
  const long long rows = static_cast<long long>(g.B) * g.h * p.n_seq * p.seq_len;
  return static_cast<unsigned>((rows + 7) / 8);
}

cudaError_t launch_simt_fwd(const SimtFwdArgs& a, cudaStream_t stream) {
  const unsigned grid = rows_grid(a.g, a.p);
  if (grid == 0) return cudaSuccess;
  simt_pass_fwd_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_simt_bwd(const SimtBwdArgs& a, cudaStream_t stream) {
  const unsigned grid = rows_grid(a.g, a.p);
  if (grid == 0) return cudaSuccess;
  simt_pass_bwd_rows_kernel<<<grid, 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt_pass_bwd_cols_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace squad
