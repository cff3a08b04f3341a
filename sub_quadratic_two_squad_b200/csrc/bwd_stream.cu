// Tensor-core backward of one SQuad pass for sequences of any length, sm_100a: the sequences are cut
// into chunks of whole lines of at most 128 rows (geometry.cuh), and each CTA keeps one chunk resident
// while the others stream through a double buffer, so shared memory does not grow with the sequence.
//
// Each pass of SQuad-Attention is ordinary softmax attention inside each sequence (a window for the
// local pass, a slot across windows for the global pass; SQuad paper §3.2), so its gradients are those
// of softmax attention, sequence by sequence. With P = softmax(scale Q K^T) recomputed from the
// forward's LSE, O the pass output and dO the gradient of it:
//   D_i = sum_j P_ij dP_ij = dO_i . O_i,  dP = dO V^T,  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
//
// rows kernel, per item (sequence, query chunk i): Q_i, dO_i and O_i resident; D_i from dO_i and
//   O_i; the key chunks j stream through: S = Q_i K_j^T and dP = dO_i V_j^T in tensor memory, the
//   row-owner warps form dS (bf16, packed over S), dQ_i += dS K_j accumulates in tensor memory (in one
//   of two column sets, items alternating). Writes dQ_i (or its fp32 share) and D_i.
// columns kernel, per item (sequence, key chunk j): K_j and V_j resident; the query chunks i stream
//   through with their LSE and D: S^T = K_j Q_i^T and dP^T = V_j dO_i^T, the warps form P^T and dS^T,
//   dV_j += P^T dO_i and dK_j += dS^T Q_i accumulate in tensor memory. Writes dV_j and dK_j.
// Both persistent, one CTA per SM taking items in turn, 288 threads: warps 0-3 own one TMEM lane
// (row) per thread, warps 4-7 write the accumulated gradients out (warp 4 + w reads the lanes of warp
// w), warp 8 issues the TMA loads and the tcgen05 MMAs. The stream of chunks runs on across items, and
// the next item's resident chunks are loaded as soon as the last products that read them complete,
// so loads, products, the owners' work and the write-out of the previous item overlap. Rows past a
// chunk are computed and dropped; columns past it are masked to zero. The rows kernel runs first (the
// columns kernel reads its D).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "host_util.h"
#include "ptx.cuh"
#include "geometry.cuh"
#include "bwd_stream.h"

namespace squad {

namespace {

constexpr int kThreads = 288;   // 4 row-owner warps, 4 epilogue warps, 1 load/MMA warp
constexpr uint32_t kPanel = 16384;           // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kTile = 2 * kPanel;       // a 128-row chunk of one tensor, both 64-column panels
constexpr float kLog2e = 1.4426950408889634f;

// rows kernel: Q_i, dO_i, O_i, then two buffers of (K_j, V_j)
constexpr uint32_t kRowQ = 0, kRowDO = kTile, kRowO = 2 * kTile, kRowKV = 3 * kTile;
constexpr uint32_t kRowBar = kRowKV + 4 * kTile;
// columns kernel: K_j, V_j, then two buffers of (Q_i, dO_i), then two slots of per-query LSE and D
constexpr uint32_t kColK = 0, kColV = kTile, kColQD = 2 * kTile;
constexpr uint32_t kColVec = kColQD + 4 * kTile;
constexpr uint32_t kColBar = kColVec + 2 * 2 * 128 * 4;
constexpr uint32_t kBarBytes = 256;
constexpr uint32_t kRowSmem = kRowBar + kBarBytes + 1024;
constexpr uint32_t kColSmem = kColBar + kBarBytes + 1024;
static_assert(kRowSmem <= 232448 && kColSmem <= 232448, "shared memory budget");

struct Bars {
  uint64_t first[2];       // an item's resident chunk(s) landed (items alternate)
  uint64_t full[2];        // a streamed buffer landed
  uint64_t empty[2];       // the MMAs that read a streamed buffer are done
  uint64_t s_full, p_full;
  uint64_t o_full[2];      // an item's accumulated gradients are complete (rows: per dQ column set)
  uint64_t o_free[2];      // ... and have been read out of tensor memory by the epilogue warps
  uint64_t vec_full[2], vec_empty[2];   // columns kernel: LSE / D of a streamed query chunk
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block");

__device__ __forceinline__ int round16s(int x) { return (x + 15) & ~15; }

// K-major descriptor of K step kk (16 elements) of a 128-row chunk tile at `addr`.
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, int kk) {
  return sw128_desc(addr + static_cast<uint32_t>(kk >> 2) * kPanel + static_cast<uint32_t>(kk & 3) * 32u, 16, 1024);
}
// MN-major descriptor (the 128 d columns wide) of rows [16 kk, 16 kk + 16) of a chunk tile at `addr`.
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, int kk) {
  return sw128_desc(addr + static_cast<uint32_t>(kk) * 2048u, kPanel, 1024);
}

// (head, sequence, chunk) of CTA `blk` (chunks of a sequence are consecutive).
__device__ __forceinline__ void decode_blk(const PassGeom& p, int blk, int& bh, int& sigma, int& chunk) {
  const int per_bh = p.n_seq * p.n_chunks;
  bh = static_cast<int>(fdiv(static_cast<uint32_t>(blk), p.f_per_bh));
  const int rem = blk - bh * per_bh;
  sigma = static_cast<int>(fdiv(static_cast<uint32_t>(rem), p.f_chunks));
  chunk = rem - sigma * p.n_chunks;
}

// One chunk of `m` (both panels) into `dst`, completing on `bar` (bytes counted by the caller).
__device__ __forceinline__ void load_chunk(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, const Grid& g,
                                           const PassGeom& p, int variant, int bh, int sigma, int chunk) {
  int c[5];
  chunk_coords(g, p, variant, bh, sigma, chunk, 0, c);
  tma_load_5d(dst, m, bar, c[0], c[1], c[2], c[3], c[4]);
  tma_load_5d(dst + kPanel, m, bar, c[0] + 64, c[1], c[2], c[3], c[4]);
}

// Dot product of row r of two chunk tiles (bf16, 128-byte swizzle) in fp32.
__device__ __forceinline__ float row_dot(const uint8_t* a, const uint8_t* b, int r) {
  float acc = 0.f;
#pragma unroll
  for (int pnl = 0; pnl < 2; ++pnl) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t off = static_cast<uint32_t>(pnl) * kPanel + static_cast<uint32_t>(r) * 128u +
                           ((static_cast<uint32_t>(c) ^ static_cast<uint32_t>(r & 7)) << 4);
      const uint4 x = *reinterpret_cast<const uint4*>(a + off);
      const uint4 y = *reinterpret_cast<const uint4*>(b + off);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc = fmaf(__uint_as_float(xs[k] << 16), __uint_as_float(ys[k] << 16), acc);
        acc = fmaf(__uint_as_float(xs[k] & 0xFFFF0000u), __uint_as_float(ys[k] & 0xFFFF0000u), acc);
      }
    }
  }
  return acc;
}

// The 128 fp32 values of this thread's row in TMEM columns [col, col + 128), written to global memory
// when `store`: times `mul`, plus `acc` (fp32 row) if given, as bf16 to `out16` or as fp32 to `out32`
// (acc and out32 rows are 32-byte aligned: workspace rows of 512 bytes, read and written 32 bytes at a
// time).
// Every thread of the warp calls it (tcgen05.ld is warp-wide); only the stores depend on `store`.
__device__ __forceinline__ void write_row(uint32_t taddr, bool store, float mul, const float* acc,
                                          __nv_bfloat16* out16, float* out32) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t r[64];
    tmem_ld64(taddr + 64 * h, r);
    if (!store) continue;
    float v[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]) * mul;
    if (acc != nullptr) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float x[8];
        ldg_v8(acc + 64 * h + 8 * i, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * i + j] += x[j];
      }
    }
    if (out16 != nullptr) {
      uint4* o4 = reinterpret_cast<uint4*>(out16 + 64 * h);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o4[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                           pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) stg_v8(out32 + 64 * h + 8 * i, &v[8 * i]);
    }
  }
}

// Common set-up: zero the operand tiles once (rows past a chunk are read by the MMAs and must be
// finite; every chunk's boxes write the same rows), initialise the barriers, allocate all of tensor
// memory.
__device__ __forceinline__ void setup(uint8_t* base, uint32_t tiles_bytes, Bars* bars, int warp) {
  for (uint32_t i = threadIdx.x; i < tiles_bytes / 16u; i += kThreads)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 256) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->first[s], 1);
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
      mbar_init(&bars->vec_full[s], 128);
      mbar_init(&bars->vec_empty[s], 128);
      mbar_init(&bars->o_full[s], 1);
      mbar_init(&bars->o_free[s], 128);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

__device__ __forceinline__ void teardown(uint32_t tmem, int warp) {
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// rows: dQ and D of query chunks (persistent: this CTA takes items blockIdx.x, + gridDim.x, ...)
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) bwd_rows_kernel(const __grid_constant__ BwdStreamArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(base + kRowBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const int nb = p.n_chunks;
  const int items = g.B * g.h * p.n_seq * nb;
  const int mine = static_cast<int>(blockIdx.x) < items
                       ? (items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
  setup(base, kRowBar, bars, warp);
  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};
  const uint32_t tile_tx = 2u * static_cast<uint32_t>(p.chunk_rows) * 128u;   // one chunk, both panels
  auto item_of = [&](int k) { return static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x); };

  if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads + MMA issue
      prefetch_tmap(&a.tm_q);
      prefetch_tmap(&a.tm_k);
      prefetch_tmap(&a.tm_v);
      prefetch_tmap(&a.tm_do);
      prefetch_tmap(&a.tm_o);
      // Q_i, dO_i, O_i of this CTA's k-th item
      auto load_res = [&](int k) {
        int bh, sigma, qc;
        decode_blk(p, item_of(k), bh, sigma, qc);
        uint64_t* bar = &bars->first[k & 1];
        mbar_arrive_expect_tx(bar, 3u * tile_tx);
        load_chunk(base + kRowQ, &a.tm_q, bar, g, p, a.variant, bh, sigma, qc);
        load_chunk(base + kRowDO, &a.tm_do, bar, g, p, a.variant, bh, sigma, qc);
        load_chunk(base + kRowO, &a.tm_o, bar, g, p, a.variant, bh, sigma, qc);
      };
      // stream entry e = k nb + j: the key chunk j of item k's sequence, into buffer e & 1
      auto load_kv = [&](int e) {
        int bh, sigma, qc;
        decode_blk(p, item_of(e / nb), bh, sigma, qc);
        const int j = e % nb;
        uint8_t* dst = base + kRowKV + static_cast<uint32_t>(e & 1) * 2u * kTile;
        mbar_arrive_expect_tx(&bars->full[e & 1], 2u * tile_tx);
        load_chunk(dst, &a.tm_k, &bars->full[e & 1], g, p, a.variant, bh, sigma, j);
        load_chunk(dst + kTile, &a.tm_v, &bars->full[e & 1], g, p, a.variant, bh, sigma, j);
      };
      const int n_entries = mine * nb;
      int res_issued = 0, kv_issued = 0;
      if (mine > 0) {
        load_res(0);
        res_issued = 1;
        for (; kv_issued < 2 && kv_issued < n_entries; ++kv_issued) load_kv(kv_issued);
      }
      const uint32_t aq = smem_u32(base + kRowQ), ado = smem_u32(base + kRowDO);
      const uint32_t idesc_o = idesc_bf16(128, 128, true);
      bool ok = true;
      for (int k = 0; k < mine && ok; ++k) {
        const uint32_t dq_col = 256u + 128u * static_cast<uint32_t>(k & 1);   // alternating dQ columns
        ok = mbar_wait(&bars->first[k & 1], (k >> 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < nb && ok; ++j) {
          const int e = k * nb + j;
          const int nk = chunk_valid_rows(p, j);
          const int N = round16s(nk);
          const uint32_t ak = smem_u32(base + kRowKV + static_cast<uint32_t>(e & 1) * 2u * kTile);
          const uint32_t av = ak + kTile;
          ok = mbar_wait(&bars->full[e & 1], (e >> 1) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t idesc_s = idesc_bf16(128, N, false);
          for (int kk = 0; kk < 8; ++kk)   // S = Q_i K_j^T -> [0, N)
            umma_bf16_ss(tmem, kdesc(aq, kk), kdesc(ak, kk), idesc_s, kk > 0);
          for (int kk = 0; kk < 8; ++kk)   // dP = dO_i V_j^T -> [128, 128 + N)
            umma_bf16_ss(tmem + 128, kdesc(ado, kk), kdesc(av, kk), idesc_s, kk > 0);
          umma_commit(&bars->s_full);
          ok = mbar_wait(&bars->p_full, e & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          if (j == nb - 1 && k + 1 < mine) {
            // this item's S and dP are done and the owners have formed its D: load the next item's
            // resident chunks while its last dQ product runs
            load_res(k + 1);
            ++res_issued;
          }
          if (j == 0 && k >= 2) {   // these dQ columns were last used two items ago: read out by now
            ok = mbar_wait(&bars->o_free[k & 1], ((k >> 1) - 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
          }
          for (int kk = 0; kk < N / 16; ++kk)   // dQ += dS K_j
            umma_bf16_ts(tmem + dq_col, tmem + kk * 8, mndesc(ak, kk), idesc_o, j > 0 || kk > 0);
          umma_commit(&bars->empty[e & 1]);
          if (j == nb - 1) umma_commit(&bars->o_full[k & 1]);
          if (kv_issued < n_entries) {   // refill this buffer once the products that read it are done
            ok = mbar_wait(&bars->empty[e & 1], (e >> 1) & 1, ctl);
            if (ok) load_kv(kv_issued++);
          }
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
      // every load issued has landed before the CTA can exit (bounded)
      if (res_issued > 0) mbar_wait_drain(&bars->first[(res_issued - 1) & 1], ((res_issued - 1) >> 1) & 1, 20000000ull);
      for (int e = (kv_issued > 2 ? kv_issued - 2 : 0); e < kv_issued; ++e)
        mbar_wait_drain(&bars->full[e & 1], (e >> 1) & 1, 20000000ull);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- row owners
    const int rl = warp * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int k = 0; k < mine && ok; ++k) {
      int bh, sigma, qc;
      decode_blk(p, item_of(k), bh, sigma, qc);
      const int nq = chunk_valid_rows(p, qc);
      const int tok = rl < nq ? token_of(g, p, sigma, qc, rl) : -1;
      const size_t gi = static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok);
      const float lse2 = tok >= 0 ? a.lse[gi] * kLog2e : 0.f;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->first[k & 1], (k >> 1) & 1, ctl));
      if (!ok) break;
      const float D = row_dot(base + kRowDO, base + kRowO, rl);   // D_i = dO_i . O_i
      if (tok >= 0) a.drow[gi] = D;
      for (int j = 0; j < nb && ok; ++j) {
        const int e = k * nb + j;
        const int nk = chunk_valid_rows(p, j);
        const int N = round16s(nk);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full, e & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        // dS = P o (dP - D) with P = 2^(S scale log2e - LSE log2e), packed two per column over S
#pragma unroll 1
        for (int c = 0; c < N / 32 + ((N & 31) ? 1 : 0); ++c) {
          uint32_t sr[32], dr[32], pk[16];
          tmem_ld32(t_row + 32 * c, sr);
          tmem_ld32(t_row + 128 + 32 * c, dr);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k0 = 32 * c + 2 * i;
            float e0, e1, d0, d1, s0, s1;
            ffma2(e0, e1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), sl2, sl2, -lse2, -lse2);
            ffma2(d0, d1, __uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]), 1.f, 1.f, -D, -D);
            fmul2(s0, s1, ex2_approx(e0), ex2_approx(e1), d0, d1);
            // columns past the chunk hold unwritten tensor memory: whatever was formed there is dropped
            pk[i] = pack_bf16x2(k0 < nk ? s0 : 0.f, k0 + 1 < nk ? s1 : 0.f);
          }
          tmem_st16_nowait(t_row + 16 * c, pk);   // over scores already read; waited for below
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue: dQ of each item
    const int rl = (warp - 4) * 32 + lane;   // the row of owner warp (warp - 4), lane `lane`
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    bool ok = true;
    for (int k = 0; k < mine && ok; ++k) {
      int bh, sigma, qc;
      decode_blk(p, item_of(k), bh, sigma, qc);
      const int nq = chunk_valid_rows(p, qc);
      const int tok = rl < nq ? token_of(g, p, sigma, qc, rl) : -1;
      const size_t ro = (static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok)) * 128;
      if (a.accumulate && tok >= 0) prefetch_l2(a.dq_acc + ro, 512u);   // the earlier passes' share: into L2
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_full[k & 1], (k >> 1) & 1, ctl));
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_dq = t_lane + 256u + 128u * static_cast<uint32_t>(k & 1);
      if (a.final_out)
        write_row(t_dq, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, a.dq_out + ro, nullptr);
      else
        write_row(t_dq, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, nullptr, a.dq_acc + ro);
      tc_fence_before();
      mbar_arrive(&bars->o_free[k & 1]);
    }
  }
  teardown(tmem, warp);
}

// ------------------------------------------------------------------------------------------------
// columns: dK and dV of key chunks (persistent: this CTA takes items blockIdx.x, + gridDim.x, ...)
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) bwd_cols_kernel(const __grid_constant__ BwdStreamArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(base + kColBar);
  float* lse_s = reinterpret_cast<float*>(base + kColVec);   // [2][128] per query, log2 units
  float* d_s = lse_s + 256;                                   // [2][128] per query D
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const int nb = p.n_chunks;
  const int items = g.B * g.h * p.n_seq * nb;
  const int mine = static_cast<int>(blockIdx.x) < items
                       ? (items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
  setup(base, kColVec, bars, warp);
  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};
  const uint32_t tile_tx = 2u * static_cast<uint32_t>(p.chunk_rows) * 128u;
  auto item_of = [&](int k) { return static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x); };

  if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads + MMA issue
      prefetch_tmap(&a.tm_q);
      prefetch_tmap(&a.tm_k);
      prefetch_tmap(&a.tm_v);
      prefetch_tmap(&a.tm_do);
      auto load_res = [&](int k) {   // K_j, V_j of this CTA's k-th item
        int bh, sigma, kc;
        decode_blk(p, item_of(k), bh, sigma, kc);
        uint64_t* bar = &bars->first[k & 1];
        mbar_arrive_expect_tx(bar, 2u * tile_tx);
        load_chunk(base + kColK, &a.tm_k, bar, g, p, a.variant, bh, sigma, kc);
        load_chunk(base + kColV, &a.tm_v, bar, g, p, a.variant, bh, sigma, kc);
      };
      auto load_qd = [&](int e) {    // stream entry e = k nb + i: query chunk i of item k's sequence
        int bh, sigma, kc;
        decode_blk(p, item_of(e / nb), bh, sigma, kc);
        const int i = e % nb;
        uint8_t* dst = base + kColQD + static_cast<uint32_t>(e & 1) * 2u * kTile;
        mbar_arrive_expect_tx(&bars->full[e & 1], 2u * tile_tx);
        load_chunk(dst, &a.tm_q, &bars->full[e & 1], g, p, a.variant, bh, sigma, i);
        load_chunk(dst + kTile, &a.tm_do, &bars->full[e & 1], g, p, a.variant, bh, sigma, i);
      };
      const int n_entries = mine * nb;
      int res_issued = 0, qd_issued = 0;
      if (mine > 0) {
        load_res(0);
        res_issued = 1;
        for (; qd_issued < 2 && qd_issued < n_entries; ++qd_issued) load_qd(qd_issued);
      }
      const uint32_t ak = smem_u32(base + kColK), av = smem_u32(base + kColV);
      const uint32_t idesc_o = idesc_bf16(128, 128, true);
      bool ok = true;
      for (int k = 0; k < mine && ok; ++k) {
        ok = mbar_wait(&bars->first[k & 1], (k >> 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        for (int i = 0; i < nb && ok; ++i) {
          const int e = k * nb + i;
          const int nq = chunk_valid_rows(p, i);
          const int Nq = round16s(nq);
          const uint32_t aq = smem_u32(base + kColQD + static_cast<uint32_t>(e & 1) * 2u * kTile);
          const uint32_t ado = aq + kTile;
          ok = mbar_wait(&bars->full[e & 1], (e >> 1) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t idesc_c = idesc_bf16(128, Nq, false);
          for (int kk = 0; kk < 8; ++kk)   // S^T = K_j Q_i^T -> [0, Nq)
            umma_bf16_ss(tmem, kdesc(ak, kk), kdesc(aq, kk), idesc_c, kk > 0);
          for (int kk = 0; kk < 8; ++kk)   // dP^T = V_j dO_i^T -> [128, 128 + Nq)
            umma_bf16_ss(tmem + 128, kdesc(av, kk), kdesc(ado, kk), idesc_c, kk > 0);
          umma_commit(&bars->s_full);
          if (i == nb - 1 && k + 1 < mine) {
            // K_j and V_j are read by this item's last S^T and dP^T only: once those complete, load
            // the next item's
            ok = mbar_wait(&bars->s_full, e & 1, ctl);
            if (!ok) break;
            load_res(k + 1);
            ++res_issued;
          }
          ok = mbar_wait(&bars->p_full, e & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          if (i == 0 && k >= 1) {   // the previous item's dV and dK read out of their columns
            ok = mbar_wait(&bars->o_free[0], (k - 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
          }
          for (int kk = 0; kk < Nq / 16; ++kk)   // dV += P^T dO_i -> [256, 384)
            umma_bf16_ts(tmem + 256, tmem + kk * 8, mndesc(ado, kk), idesc_o, i > 0 || kk > 0);
          for (int kk = 0; kk < Nq / 16; ++kk)   // dK += dS^T Q_i -> [384, 512)
            umma_bf16_ts(tmem + 384, tmem + 128 + kk * 8, mndesc(aq, kk), idesc_o, i > 0 || kk > 0);
          umma_commit(&bars->empty[e & 1]);
          if (i == nb - 1) umma_commit(&bars->o_full[0]);
          if (qd_issued < n_entries) {
            ok = mbar_wait(&bars->empty[e & 1], (e >> 1) & 1, ctl);
            if (ok) load_qd(qd_issued++);
          }
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
      if (res_issued > 0) mbar_wait_drain(&bars->first[(res_issued - 1) & 1], ((res_issued - 1) >> 1) & 1, 20000000ull);
      for (int e = (qd_issued > 2 ? qd_issued - 2 : 0); e < qd_issued; ++e)
        mbar_wait_drain(&bars->full[e & 1], (e >> 1) & 1, 20000000ull);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- key-row owners
    const int rl = warp * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int k = 0; k < mine && ok; ++k) {
      int bh, sigma, kc;
      decode_blk(p, item_of(k), bh, sigma, kc);
      for (int i = 0; i < nb && ok; ++i) {
        const int e = k * nb + i;
        const int nq = chunk_valid_rows(p, i);
        const int Nq = round16s(nq);
        const int slot = e & 1;
        // this query chunk's LSE (log2 units; +inf past the chunk: P = 0 there) and D, one per thread
        if (e >= 2) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->vec_empty[slot], ((e >> 1) - 1) & 1, ctl));
        if (!ok) break;
        {
          const int qt = rl < nq ? token_of(g, p, sigma, i, rl) : -1;
          const size_t qi = static_cast<size_t>(bh) * g.n + (qt < 0 ? 0 : qt);
          lse_s[slot * 128 + rl] = qt >= 0 ? a.lse[qi] * kLog2e : INFINITY;
          d_s[slot * 128 + rl] = qt >= 0 ? a.drow[qi] : 0.f;
        }
        mbar_arrive(&bars->vec_full[slot]);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->vec_full[slot], (e >> 1) & 1, ctl));
        if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full, e & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        const float* ls = lse_s + slot * 128;
        const float* dd = d_s + slot * 128;
        // P^T over S^T and dS^T over dP^T, both bf16 packed two per column
#pragma unroll 1
        for (int c = 0; c < Nq / 32 + ((Nq & 31) ? 1 : 0); ++c) {
          uint32_t sr[32], dr[32], pp[16], ps[16];
          tmem_ld32(t_row + 32 * c, sr);
          tmem_ld32(t_row + 128 + 32 * c, dr);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int j0 = 32 * c + 2 * q;   // query column within the chunk
            const bool v0 = j0 < nq, v1 = j0 + 1 < nq;
            float e0, e1, d0, d1, s0, s1;
            ffma2(e0, e1, __uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1]), sl2, sl2, -ls[j0], -ls[j0 + 1]);
            ffma2(d0, d1, __uint_as_float(dr[2 * q]), __uint_as_float(dr[2 * q + 1]), 1.f, 1.f, -dd[j0], -dd[j0 + 1]);
            const float p0 = v0 ? ex2_approx(e0) : 0.f, p1 = v1 ? ex2_approx(e1) : 0.f;
            fmul2(s0, s1, p0, p1, d0, d1);
            pp[q] = pack_bf16x2(p0, p1);
            ps[q] = pack_bf16x2(v0 ? s0 : 0.f, v1 ? s1 : 0.f);
          }
          tmem_st16_nowait(t_row + 16 * c, pp);
          tmem_st16_nowait(t_row + 128 + 16 * c, ps);
        }
        tmem_wait_st();
        mbar_arrive(&bars->vec_empty[slot]);   // this chunk's LSE and D are no longer read
        tc_fence_before();
        mbar_arrive(&bars->p_full);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue: dV and dK of each item
    const int rl = (warp - 4) * 32 + lane;   // the key row of owner warp (warp - 4), lane `lane`
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    bool ok = true;
    for (int k = 0; k < mine && ok; ++k) {
      int bh, sigma, kc;
      decode_blk(p, item_of(k), bh, sigma, kc);
      const int nk = chunk_valid_rows(p, kc);
      const int tok = rl < nk ? token_of(g, p, sigma, kc, rl) : -1;
      const size_t ro = (static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok)) * 128;
      if (a.accumulate && tok >= 0) prefetch_l2(a.dk_acc + ro, 512u);   // the earlier passes' share: into L2
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_full[0], k & 1, ctl));
      if (!ok) break;
      tc_fence_after();
      write_row(t_lane + 256, tok >= 0, 1.f, nullptr, a.dv_out + ro, nullptr);
      if (a.final_out)
        write_row(t_lane + 384, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, a.dk_out + ro, nullptr);
      else
        write_row(t_lane + 384, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, nullptr, a.dk_acc + ro);
      tc_fence_before();
      mbar_arrive(&bars->o_free[0]);
    }
  }
  teardown(tmem, warp);
}

}  // namespace

bool bwd_stream_eligible(const Grid& g, const PassGeom& p) {
  return g.d == 128 && p.kind != kFull && p.chunk_rows >= 1 && p.chunk_rows <= 128 && p.line_len <= 128;
}

cudaError_t launch_bwd_stream(const BwdStreamArgs& a, cudaStream_t stream) {
  static std::atomic<unsigned long long> set_r{0}, set_c{0};
  cudaError_t e = max_dyn_smem_once(bwd_rows_kernel, kRowSmem, set_r);
  if (e != cudaSuccess) return e;
  e = max_dyn_smem_once(bwd_cols_kernel, kColSmem, set_c);
  if (e != cudaSuccess) return e;
  const int items = a.g.B * a.g.h * a.p.n_seq * a.p.n_chunks;
  if (items == 0) return cudaSuccess;
  // persistent: one CTA per SM (each takes most of an SM's shared memory)
  const int sms = num_sms_current();
  const unsigned grid = static_cast<unsigned>(sms > 0 && sms < items ? sms : items);
  bwd_rows_kernel<<<grid, kThreads, kRowSmem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_cols_kernel<<<grid, kThreads, kColSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace squad
