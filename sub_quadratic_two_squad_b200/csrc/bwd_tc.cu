// Tensor-core backward of one SQuad pass over sequences of at most 208 tokens, sm_100a.
//
// Each pass of SQuad-Attention is ordinary softmax attention inside each sequence (a window for the
// local pass, a slot across windows for the global pass; SQuad paper §3.2), so its gradients are those
// of softmax attention, sequence by sequence (agihunt.info digest, the paragraph that defines the
// operator; the chain rule through both passes is applied by the caller). With
// P = softmax(scale Q K^T) recomputed from the forward's LSE, O the pass output and dO its gradient:
//   dP = dO V^T,  D_i = sum_j P_ij dP_ij = dO_i . O_i,  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
//
// One kernel per pass, persistent (one CTA per SM, sequences taken in turn), 288 threads: warps 0-3 own
// one TMEM lane (one row) per thread, warps 4-7 write the gradients out (warp 4 + w reads the lanes of
// warp w), warp 8 loads each sequence's Q, K (first) and V, dO once as whole TMA boxes and issues the
// tcgen05 MMAs. A sequence's loads are issued once the previous sequence's products have completed,
// so they land while its last gradients are written out.
// Sequences of 129-208 tokens (bwd_tc_kernel):
//   rows, per 128-query tile: each warp forms D from its rows of dO (shared memory) and O (global)
//     while S = Q K^T and dP = dO V^T go into TMEM; then P and dS = P o (dP - D) in one pass over the
//     scores (bf16): dS packed two per column over S for dQ = dS K (A from TMEM), and P and dS of the
//     row written to the CTA's scratch slot in global memory, in the layout of 128-key operand
//     tiles. Where tensor memory has room, dQ has columns of its own, so the next tile's S and dP are
//     computed while it is written out.
//   columns, per 128-key tile: that tile's P and dS come back from the slot (L2) into the K and V
//     allocations, free once the row products are done, by bulk copies, and dV = P^T dO and
//     dK = dS^T Q are two products over all queries (P^T and dS^T as MN-major A operands). No score
//     is computed twice.
// Sequences of at most 128 tokens (bwd_tc1_kernel): one tile each way, P and dS through shared memory.
// Rows past the sequence are computed and dropped; columns past it are masked to P = dS = 0, and the
// shared-memory rows past each box are zeroed so every MMA operand is finite.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "host_util.h"
#include "ptx.cuh"
#include "geometry.cuh"
#include "bwd_pass.h"

namespace squad {

namespace {

constexpr int kBwdThreads = 288;   // 4 row-owner warps, 4 epilogue warps, 1 load/MMA warp
constexpr uint32_t kBwdSmemLimit = 232448;
// Each CTA takes all 512 TMEM columns, so it also takes more than half of an SM's shared memory:
// no second CTA is ever resident beside it waiting for tensor memory.
constexpr uint32_t kBwdSmemMin = 120u * 1024u;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdBars {
  uint64_t load_qk, load_vd, s_full, p_full, o_full, o_free, drain, epi_free;
  uint64_t pds_ready, pds_full, pds_empty;   // whole-sequence kernel: P and dS through the scratch slot
  uint32_t tmem_base;
  uint32_t abort;
};
constexpr uint32_t kBwdBarBytes = 128;
static_assert(sizeof(BwdBars) <= kBwdBarBytes, "barrier block");
constexpr uint32_t kBwdVecBytes = 2u * 256u * 4u;   // per-query LSE (log2 units) and D, column kernel

__device__ __forceinline__ int round16b(int x) { return (x + 15) & ~15; }

// dQ gets tensor-memory columns of its own, [384, 512), where S and dP ([0, 2N)) leave them free;
// they are also clear of the column phase's S^T and dP^T ([0, 256)).
__device__ __forceinline__ bool dq_own_columns(int N) { return 2 * N <= 384; }

// D = dO_r . O_r in fp32: row r of the dO tile (bf16, 128-byte swizzle, two 64-column panels `panel`
// bytes apart) against the row's output held as 16 x 8 bf16 (columns 8i .. 8i + 7 in o[i]).
__device__ __forceinline__ float row_dot_out(const uint8_t* sdo, uint32_t panel, int r, const uint4 (&o)[16]) {
  float acc[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t pnl = static_cast<uint32_t>(i >> 3), c = static_cast<uint32_t>(i & 7);
    const uint4 x = *reinterpret_cast<const uint4*>(sdo + pnl * panel + static_cast<uint32_t>(r) * 128u +
                                                    ((c ^ static_cast<uint32_t>(r & 7)) << 4));
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {o[i].x, o[i].y, o[i].z, o[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[k & 1] = fmaf(__uint_as_float(xs[k] << 16), __uint_as_float(ys[k] << 16), acc[k & 1]);
      acc[k & 1] = fmaf(__uint_as_float(xs[k] & 0xFFFF0000u), __uint_as_float(ys[k] & 0xFFFF0000u), acc[k & 1]);
    }
  }
  return acc[0] + acc[1];
}

__device__ __forceinline__ uint32_t pack2_rn(float lo, float hi) { return pack_bf16x2(lo, hi); }

// K-major descriptor of a 128-row operand tile starting at `addr` (panel 0; panel 1 at +panel).
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, int kk, uint32_t panel) {
  return sw128_desc(addr + static_cast<uint32_t>(kk >> 2) * panel + static_cast<uint32_t>(kk & 3) * 32u, 16, 1024);
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
        o4[i] = make_uint4(pack2_rn(v[8 * i], v[8 * i + 1]), pack2_rn(v[8 * i + 2], v[8 * i + 3]),
                           pack2_rn(v[8 * i + 4], v[8 * i + 5]), pack2_rn(v[8 * i + 6], v[8 * i + 7]));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) stg_v8(out32 + 64 * h + 8 * i, &v[8 * i]);
    }
  }
}

__global__ void __launch_bounds__(kBwdThreads, 1) bwd_tc_kernel(const __grid_constant__ BwdTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t panel = a.panel_bytes, alloc = 2u * panel;
  uint8_t* const sq = base;
  uint8_t* const sk = base + alloc;
  uint8_t* const sv = base + 2 * alloc;
  uint8_t* const sdo = base + 3 * alloc;
  BwdBars* const bars = reinterpret_cast<BwdBars*>(base + 4 * alloc + a.guard_bytes + kBwdVecBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const int s = p.seq_len;
  const int N = round16b(s);
  const int ntiles = (s + 127) / 128;
  const int seqs = g.B * g.h * p.n_seq;

  // Rows past the sequence in each allocation, and the guard past the last one, are read by the MMAs:
  // zero them once (the TMA boxes write exactly s rows per panel, sequence after sequence).
  {
    const uint32_t tail = panel - static_cast<uint32_t>(s) * 128u;   // bytes per panel
    const uint32_t tail16 = tail / 16u;
    for (uint32_t i = threadIdx.x; i < 8u * tail16; i += kBwdThreads) {
      const uint32_t pnl = i / tail16, j = i - pnl * tail16;
      reinterpret_cast<uint4*>(base + pnl * panel + static_cast<uint32_t>(s) * 128u)[j] = make_uint4(0, 0, 0, 0);
    }
    for (uint32_t i = threadIdx.x; i < a.guard_bytes / 16u; i += kBwdThreads)
      reinterpret_cast<uint4*>(base + 4 * alloc)[i] = make_uint4(0, 0, 0, 0);
  }
  // This CTA's scratch slot starts zeroed: its parts that no row writes (keys past the last column
  // chunk) are read by the column products.
  uint8_t* const pds = a.pds + static_cast<size_t>(blockIdx.x) * a.pds_slot_bytes;
  for (uint32_t i = threadIdx.x; i < a.pds_slot_bytes / 16u; i += kBwdThreads)
    reinterpret_cast<uint4*>(pds)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_global();   // ... visible to the bulk copies (async proxy)
  if (threadIdx.x == 256) {
    mbar_init(&bars->load_qk, 1);
    mbar_init(&bars->load_vd, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->pds_ready, 128);   // the owners' P and dS rows of the sequence are in the slot
    mbar_init(&bars->pds_full, 1);      // a key tile's P and dS landed in the K and V allocations
    mbar_init(&bars->pds_empty, 1);     // ... and the products that read them are done
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();   // zeroed rows -> visible to the MMAs (async proxy)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};
  // All 512 columns were requested, so the allocation starts at lane 0, column 0: anything else is
  // an error, reported through the status word, and no tensor-memory access is made.
  const bool tmem_ok = tmem == 0u;
  if (!tmem_ok && threadIdx.x == 0 && a.status != nullptr) atomicCAS(a.status, 0u, kStatusTimeout);
  const uint32_t idesc_o = idesc_bf16(128, 128, true);   // [128 x 128] += A(TMEM) x B(MN-major, d wide)

  if (!tmem_ok) {
    // nothing issued: fall through to the release below
  } else if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads + MMA issue
      prefetch_tmap(&a.tm_q);
      prefetch_tmap(&a.tm_k);
      prefetch_tmap(&a.tm_v);
      prefetch_tmap(&a.tm_do);
      const uint32_t tx_half = 4u * static_cast<uint32_t>(s) * 128u;   // two tensors, both panels
      const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv), ado = smem_u32(sdo);
      uint32_t p_cnt = 0, f_cnt = 0, oc = 0, issued = 0, pf = 0, pe = 0;
      // the epilogue warps have read the previous results (dQ, or dV and dK) out of tensor memory
      auto wait_free = [&]() -> bool {
        const bool r = mbar_wait(&bars->o_free, f_cnt & 1, ctl);
        ++f_cnt;
        if (r) tc_fence_after();
        return r;
      };
      // rows: per 128-query tile, S and dP, then dQ = dS K into [qcol, qcol + 128)
      const uint32_t idesc_s = idesc_bf16(128, N, false);
      const bool own_dq = dq_own_columns(N);
      const uint32_t qcol = own_dq ? 384u : static_cast<uint32_t>(N);
      bool ok = true;
      bool pending = false;   // an o_full whose o_free has not been waited for
      uint32_t it = 0;
      for (int seq = static_cast<int>(blockIdx.x); ok && seq < seqs; seq += static_cast<int>(gridDim.x), ++it) {
        if (it > 0) {
          // the previous sequence's products have read all of its operand tiles
          ok = mbar_wait(&bars->o_full, (oc - 1) & 1u, ctl);
          if (!ok) break;
        }
        {
          const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(seq), p.f_per_bh));
          int c[5];
          chunk_coords(g, p, a.variant, bh, seq - bh * p.n_seq, 0, 0, c);
          mbar_arrive_expect_tx(&bars->load_qk, tx_half);
          mbar_arrive_expect_tx(&bars->load_vd, tx_half);
          const CUtensorMap* maps[4] = {&a.tm_q, &a.tm_k, &a.tm_v, &a.tm_do};
          uint8_t* dsts[4] = {sq, sk, sv, sdo};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint64_t* bar = i < 2 ? &bars->load_qk : &bars->load_vd;
            tma_load_5d(dsts[i], maps[i], bar, c[0], c[1], c[2], c[3], c[4]);
            tma_load_5d(dsts[i] + panel, maps[i], bar, c[0] + 64, c[1], c[2], c[3], c[4]);
          }
          ++issued;
        }
        ok = mbar_wait(&bars->load_qk, it & 1u, ctl);
        if (!ok) break;
        tc_fence_after();
      for (int t = 0; t < ntiles && ok; ++t) {
        // dQ over dP's columns: the previous tile's dQ must have been read before S and dP are written
        if (t > 0 && !own_dq && !(ok = wait_free())) break;
        const uint32_t row_off = static_cast<uint32_t>(t) * 16384u;
        for (int kk = 0; kk < 8; ++kk)   // S = Q_t K^T -> [0, N)
          umma_bf16_ss(tmem, kdesc(aq + row_off, kk, panel), kdesc(ak, kk, panel), idesc_s, kk > 0);
        if (t == 0) {
          ok = mbar_wait(&bars->load_vd, it & 1u, ctl);
          if (!ok) break;
          tc_fence_after();
          // dP (and dQ) reach the columns of the previous sequence's dV and dK: read out by now
          if (pending) {
            if (!(ok = wait_free())) break;
            pending = false;
          }
        }
        for (int kk = 0; kk < 8; ++kk)   // dP = dO_t V^T -> [N, 2N)
          umma_bf16_ss(tmem + N, kdesc(ado + row_off, kk, panel), kdesc(av, kk, panel), idesc_s, kk > 0);
        umma_commit(&bars->s_full);
        ok = mbar_wait(&bars->p_full, p_cnt & 1, ctl);
        ++p_cnt;
        if (!ok) break;
        tc_fence_after();
        // dQ in columns of its own: only the previous tile's dQ must have been read
        if (t > 0 && own_dq && !(ok = wait_free())) break;
        for (int kk = 0; kk < N / 16; ++kk)   // dQ = dS K
          umma_bf16_ts(tmem + qcol, tmem + kk * 8, sw128_desc(ak + kk * 2048, panel, 1024), idesc_o, kk > 0);
        umma_commit(&bars->o_full);
        ++oc;
      }
      // columns, per 128-key tile kt: the owners' P and dS of the whole sequence (bf16, in this CTA's
      // scratch slot) come into the K and V allocations, which the row phase's last products free, and
      // dV += P^T dO and dK += dS^T Q run over all queries (P^T and dS^T as MN-major A operands) into
      // [256, 384) and [384, 512), once the epilogue has read the last dQ, or the previous key tile's dV
      // and dK, out of those columns. No scores are recomputed.
      pending = ok;
      if (ok) ok = mbar_wait(&bars->pds_ready, it & 1u, ctl);
      if (ok) ok = mbar_wait(&bars->o_full, (oc - 1) & 1u, ctl);   // the last dQ product has read K
      const int Ns = round16b(s);
      for (int kt = 0; kt < ntiles && ok; ++kt) {
        if (kt > 0 && !(ok = mbar_wait(&bars->pds_empty, (pe - 1) & 1u, ctl))) break;
        mbar_arrive_expect_tx(&bars->pds_full, 4u * panel);
        bulk_load(sk, pds + static_cast<size_t>(4 * kt) * panel, 2u * panel, &bars->pds_full);       // P, keys of kt
        bulk_load(sv, pds + static_cast<size_t>(4 * kt + 2) * panel, 2u * panel, &bars->pds_full);   // dS
        ok = mbar_wait(&bars->pds_full, pf & 1u, ctl);
        ++pf;
        if (!ok) break;
        if (pending) {
          if (!(ok = wait_free())) break;
          pending = false;
        }
        tc_fence_after();
        const uint32_t idesc_t = idesc_bf16_a_mn(128, 128);   // A = P^T / dS^T, B = dO / Q (MN-major)
        for (int kk = 0; kk < Ns / 16; ++kk)   // dV = P^T dO -> [256, 384)
          umma_bf16_ss(tmem + 256, sw128_desc(ak + kk * 2048, panel, 1024), sw128_desc(ado + kk * 2048, panel, 1024),
                       idesc_t, kk > 0);
        for (int kk = 0; kk < Ns / 16; ++kk)   // dK = dS^T Q -> [384, 512)
          umma_bf16_ss(tmem + 384, sw128_desc(av + kk * 2048, panel, 1024), sw128_desc(aq + kk * 2048, panel, 1024),
                       idesc_t, kk > 0);
        umma_commit(&bars->pds_empty);
        ++pe;
        umma_commit(&bars->o_full);
        ++oc;
        pending = true;
      }
      }
      // every MMA issued has completed before the CTA frees tensor memory, and every load issued has
      // landed before it exits
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
      if (issued > 0) {
        mbar_wait_drain(&bars->load_qk, (issued - 1) & 1u, 20000000ull);
        mbar_wait_drain(&bars->load_vd, (issued - 1) & 1u, 20000000ull);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ row-owner warps
    const int rl = warp * 32 + lane;   // TMEM lane of this thread
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0;
    bool ok = true;
    uint32_t it = 0;
    for (int seq = static_cast<int>(blockIdx.x); ok && seq < seqs; seq += static_cast<int>(gridDim.x), ++it) {
    const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(seq), p.f_per_bh));
    const int sigma = seq - bh * p.n_seq;
    // rows: D, then P and dS of each 128-query tile; dS packed over S for dQ = dS K, and P and dS of
    // every row also written to this CTA's scratch slot for the column products
    const int rows = static_cast<int>(panel / 128u);   // rows of a scratch panel (the sequence rounded to 16)
    for (int t = 1; t < ntiles; ++t) {   // the output rows of the later tiles (for D): into L2 now
      const int r = 128 * t + rl;
      const int tok = r < s ? token_of(g, p, sigma, 0, r) : -1;
      if (tok >= 0) prefetch_l2(a.o + (static_cast<size_t>(bh) * g.n + tok) * 128, 256u);
    }
    for (int t = 0; t < ntiles && ok; ++t) {
      const int r = 128 * t + rl;
      const int tok = r < s ? token_of(g, p, sigma, 0, r) : -1;
      const size_t gi = static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok);
      const float lse2 = tok >= 0 ? a.lse[gi] * kLog2e : 0.f;
      // D_i = dO_i . O_i: the row's output from global memory, its dO row from shared memory
      uint4 orow[16];
      {
        const uint4* src = reinterpret_cast<const uint4*>(a.o + gi * 128);
#pragma unroll
        for (int i = 0; i < 16; ++i) orow[i] = tok >= 0 ? src[i] : make_uint4(0, 0, 0, 0);
      }
      if (t == 0) {
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->load_vd, it & 1u, ctl));
        if (!ok) break;
      }
      const float D = tok >= 0 ? row_dot_out(sdo, panel, r, orow) : 0.f;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full, s_cnt & 1, ctl));   // warp-uniform exit
      ++s_cnt;
      if (!ok) break;
      tc_fence_after();
      const bool put = r < rows;   // this row is one of the scratch tiles' rows
      uint8_t* const row_p = pds + static_cast<size_t>(r) * 128u;
      const uint32_t sw = static_cast<uint32_t>(r & 7);
      // P = 2^(S scale log2e - LSE log2e) recomputed from S and the LSE, dS = P o (dP - D); both bf16,
      // zero outside the sequence
#pragma unroll 1
      for (int c = 0; c < (N + 31) / 32; ++c) {
        uint32_t sr[32], dr[32], pp[16], pk[16];
        tmem_ld32(t_row + 32 * c, sr);
        tmem_ld32(t_row + N + 32 * c, dr);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = 32 * c + 2 * i;
          const bool v0 = tok >= 0 && j < s, v1 = tok >= 0 && j + 1 < s;
          float e0, e1, d0, d1, s0, s1;
          ffma2(e0, e1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), sl2, sl2, -lse2, -lse2);
          ffma2(d0, d1, __uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]), 1.f, 1.f, -D, -D);
          const float p0 = v0 ? ex2_approx(e0) : 0.f, p1 = v1 ? ex2_approx(e1) : 0.f;
          fmul2(s0, s1, p0, p1, d0, d1);
          pp[i] = pack2_rn(p0, p1);
          pk[i] = pack2_rn(v0 ? s0 : 0.f, v1 ? s1 : 0.f);
        }
        tmem_st16_nowait(t_row + 16 * c, pk);   // waited for below, before the MMA reads dS
        if (put) {
          // keys [32 c, 32 c + 32): key tile c / 4, its 64-key panel (c / 2) % 2, 16-byte chunks
          // 4 (c % 2) .. + 3 of the row (128-byte swizzle)
          const size_t pnl = static_cast<size_t>(4 * (c >> 2) + ((c >> 1) & 1)) * panel;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t off = ((static_cast<uint32_t>(4 * (c & 1) + q)) ^ sw) << 4;
            *reinterpret_cast<uint4*>(row_p + pnl + off) = make_uint4(pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
            *reinterpret_cast<uint4*>(row_p + pnl + 2 * static_cast<size_t>(panel) + off) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    if (!ok) break;
    // the sequence's P and dS rows are in the slot: visible to the bulk copies of the column phase
    fence_proxy_async_global();
    mbar_arrive(&bars->pds_ready);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    // dQ of each row tile, then dV and dK of each key tile, as the products complete; warp 4 + w reads
    // the TMEM lanes of owner warp w.
    const int rl = (warp - 4) * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    const uint32_t qcol = dq_own_columns(N) ? 384u : static_cast<uint32_t>(N);
    uint32_t o_cnt = 0;
    bool ok = true;
    for (int seq = static_cast<int>(blockIdx.x); ok && seq < seqs; seq += static_cast<int>(gridDim.x)) {
      const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(seq), p.f_per_bh));
      const int sigma = seq - bh * p.n_seq;
      if (a.accumulate) {
        // the earlier passes' fp32 shares of this sequence's rows, added below: into L2 now
        for (int t = 0; t < ntiles; ++t) {
          const int r = 128 * t + rl;
          const int tok = r < s ? token_of(g, p, sigma, 0, r) : -1;
          if (tok >= 0) {
            const size_t ro = (static_cast<size_t>(bh) * g.n + tok) * 128;
            prefetch_l2(a.dq_acc + ro, 512u);
            prefetch_l2(a.dk_acc + ro, 512u);
          }
        }
      }
      for (int t = 0; t < 2 * ntiles && ok; ++t) {   // row tiles, then key tiles
        const int r = 128 * (t < ntiles ? t : t - ntiles) + rl;
        const int tok = r < s ? token_of(g, p, sigma, 0, r) : -1;
        const size_t ro = (static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok)) * 128;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_full, o_cnt & 1, ctl));
        ++o_cnt;
        if (!ok) break;
        tc_fence_after();
        if (t < ntiles) {
          if (a.final_out)
            write_row(t_row + qcol, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, a.dq_out + ro, nullptr);
          else
            write_row(t_row + qcol, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, nullptr, a.dq_acc + ro);
        } else {
          write_row(t_row + 256, tok >= 0, 1.f, nullptr, a.dv_out + ro, nullptr);
          if (a.final_out)
            write_row(t_row + 384, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, a.dk_out + ro, nullptr);
          else
            write_row(t_row + 384, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, nullptr, a.dk_acc + ro);
        }
        tc_fence_before();
        mbar_arrive(&bars->o_free);
      }
    }
  }
  // tcgen05.dealloc is warp-wide and aligned: reconverge warp 8 (lane 0 arrives from the issue loop)
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
// Sequences of at most 128 tokens: one query tile and one key tile. A work item is `pack` consecutive
// sequences (of all B h n_seq), each in its own band of `seg` rows (the length rounded up to 8) of
// every tile; S and dP are computed once over the whole tile, and a score counts only where query and
// key lie in the same band (P = dS = 0 elsewhere, so the products stay block-diagonal). The
// row-owner warps write P and dS (bf16) to shared memory, and dQ = dS K, dV = P^T dO and dK = dS^T Q
// are three products read from there (P^T and dS^T as MN-major A operands of the same tiles).
//
// Persistent: one CTA per SM takes items blockIdx.x, blockIdx.x + gridDim.x, ... 288 threads: warps
// 0-3 own the rows (D, P and dS), warps 4-7 write the gradients out (a thread per row again: warp
// 4 + w reads the TMEM lanes of warp w), warp 8 loads and issues the MMAs. Once the three products of
// an item have completed its operand tiles are dead, so the next item's loads are issued while the
// epilogue warps write this item's gradients out; the next dP is computed meanwhile, the next S as
// soon as dK has been read out of the columns S reuses, and the owners form the next P and dS while
// dQ and dV are still being written.
// ------------------------------------------------------------------------------------------------
constexpr uint32_t kPdsPanel = 16384;   // 128 query rows x 64 keys (bf16), 128-byte swizzle

// kPacked: several sequences per item (128-row operand tiles, a band per sequence). Otherwise one
// sequence per item, its operand tiles as long as the sequence (rounded to 8 rows) with a zeroed
// guard past the last one.
template <bool kPacked>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_tc1_kernel(const __grid_constant__ BwdTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t panel = kPacked ? kPdsPanel : a.panel_bytes, alloc = 2u * panel;
  uint8_t* const sq = base;
  uint8_t* const sk = base + alloc;
  uint8_t* const sv = base + 2 * alloc;
  uint8_t* const sdo = base + 3 * alloc;
  uint8_t* const sp = base + 4 * alloc + (kPacked ? 0u : a.guard_bytes);   // P [query][key], two 64-key panels
  uint8_t* const sds = sp + 2 * kPdsPanel;                                   // dS, the same layout
  BwdBars* const bars = reinterpret_cast<BwdBars*>(sds + 2 * kPdsPanel);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const int s = p.seq_len;
  const int seg = a.seg_rows;                                   // band of one sequence (s rounded to 8)
  const int total = g.B * g.h * p.n_seq;                        // sequences of all (b, head)
  const int n_items = (total + a.pack - 1) / a.pack;

  if constexpr (!kPacked) {
    // Rows past the sequence in each tile, and the guard past the last one, are read by the MMAs:
    // zero them once (the TMA boxes write exactly s rows per panel, item after item).
    const uint32_t tail = panel - static_cast<uint32_t>(s) * 128u;   // bytes per panel
    const uint32_t tail16 = tail / 16u;
    for (uint32_t i = threadIdx.x; i < 8u * tail16; i += kBwdThreads) {
      const uint32_t pnl = i / tail16, j = i - pnl * tail16;
      reinterpret_cast<uint4*>(base + pnl * panel + static_cast<uint32_t>(s) * 128u)[j] = make_uint4(0, 0, 0, 0);
    }
    for (uint32_t i = threadIdx.x; i < a.guard_bytes / 16u; i += kBwdThreads)
      reinterpret_cast<uint4*>(base + 4 * alloc)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();   // zeroed rows -> visible to the MMAs (async proxy)
  }
  if (threadIdx.x == 256) {
    mbar_init(&bars->load_qk, 1);
    mbar_init(&bars->load_vd, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, 128);     // dK read out: S of the next item may overwrite it
    mbar_init(&bars->epi_free, 128);   // dQ and dV read out: the next item's products may overwrite them
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};
  const bool tmem_ok = tmem == 0u;   // all 512 columns requested: anything else is an error
  if (!tmem_ok && threadIdx.x == 0 && a.status != nullptr) atomicCAS(a.status, 0u, kStatusTimeout);

  // The loads of one item: each sequence's boxes into its band (a multiple of 8 rows, so the 128-byte
  // swizzle phase is kept); Q and K on one barrier, V and dO on the other.
  auto issue_loads = [&](int item) {
    const int first = item * a.pack, nseq = min(a.pack, total - first);
    const uint32_t tx_half = static_cast<uint32_t>(nseq) * 4u * static_cast<uint32_t>(s) * 128u;
    mbar_arrive_expect_tx(&bars->load_qk, tx_half);
    mbar_arrive_expect_tx(&bars->load_vd, tx_half);
    const CUtensorMap* maps[4] = {&a.tm_q, &a.tm_k, &a.tm_v, &a.tm_do};
    uint8_t* dsts[4] = {sq, sk, sv, sdo};
    for (int j = 0; j < nseq; ++j) {
      const int gs = first + j;
      const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(gs), p.f_per_bh));
      int c[5];
      chunk_coords(g, p, a.variant, bh, gs - bh * p.n_seq, 0, 0, c);
      const uint32_t row_off = static_cast<uint32_t>(j * seg) * 128u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint64_t* bar = i < 2 ? &bars->load_qk : &bars->load_vd;
        tma_load_5d(dsts[i] + row_off, maps[i], bar, c[0], c[1], c[2], c[3], c[4]);
        tma_load_5d(dsts[i] + panel + row_off, maps[i], bar, c[0] + 64, c[1], c[2], c[3], c[4]);
      }
    }
  };
  uint32_t issued = 0;   // items whose loads this CTA has issued (thread 256)
  if (tmem_ok && threadIdx.x == 256 && static_cast<int>(blockIdx.x) < n_items) {
    issued = 1;
    prefetch_tmap(&a.tm_q);
    prefetch_tmap(&a.tm_k);
    prefetch_tmap(&a.tm_v);
    prefetch_tmap(&a.tm_do);
    issue_loads(static_cast<int>(blockIdx.x));
  }
  if constexpr (kPacked) {
    // Meanwhile, the rows of each tile that no box writes (the gap after each sequence in its band,
    // and the rows past the last band) are zeroed once: the MMAs read them. On an item with fewer
    // sequences than bands, the unused bands hold an earlier item's (finite) rows, which only meet
    // zero P and dS.
    const int nseq0 = min(a.pack, total - static_cast<int>(blockIdx.x) * a.pack);   // this CTA's first item
    for (uint32_t i = threadIdx.x; i < 8u * 128u; i += kBwdThreads) {   // (panel, row) pairs
      const int row = static_cast<int>(i & 127u);
      const int band = row / seg, pos = row - band * seg;
      if (band < nseq0 && pos < s) continue;
      uint4* dst = reinterpret_cast<uint4*>(base + (i >> 7) * panel + static_cast<uint32_t>(row) * 128u);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();   // zeroed rows -> visible to the MMAs (async proxy)
    __syncthreads();
  }

  // Tensor memory: S [0, N) then dK [0, 128); dP [128, 128 + N); dQ [256, 384); dV [384, 512).
  if (!tmem_ok) {
    // nothing issued: fall through to the release below
  } else if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads and MMA issue
      const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv), ado = smem_u32(sdo);
      const uint32_t ap = smem_u32(sp), ads = smem_u32(sds);
      const uint32_t idesc_q = idesc_bf16(128, 128, true);   // A K-major (dS), B MN-major (K)
      const uint32_t idesc_t = idesc_bf16_a_mn(128, 128);    // A = P^T / dS^T, B = dO / Q
      bool ok = true;
      uint32_t it = 0;
      for (int item = static_cast<int>(blockIdx.x); ok && item < n_items; item += static_cast<int>(gridDim.x), ++it) {
        const uint32_t ph = it & 1u;
        const int nseq = min(a.pack, total - item * a.pack);
        const int N = round16b(nseq * seg);   // key (and query) rows in use
        const uint32_t idesc_s = idesc_bf16(128, N, false);
        if (it > 0) {
          // the previous item's products have read all of its operand tiles: load this item's
          ok = mbar_wait(&bars->o_full, ph ^ 1u, ctl);
          if (!ok) break;
          issue_loads(item);
          ++issued;
        }
        ok = mbar_wait(&bars->load_qk, ph, ctl);
        if (ok && it > 0) ok = mbar_wait(&bars->o_free, ph ^ 1u, ctl);   // dK of the previous item read
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk)   // S = Q K^T -> [0, N)
          umma_bf16_ss(tmem, kdesc(aq, kk, panel), kdesc(ak, kk, panel), idesc_s, kk > 0);
        ok = mbar_wait(&bars->load_vd, ph, ctl);
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk)   // dP = dO V^T -> [128, 128 + N)
          umma_bf16_ss(tmem + 128, kdesc(ado, kk, panel), kdesc(av, kk, panel), idesc_s, kk > 0);
        umma_commit(&bars->s_full);
        ok = mbar_wait(&bars->p_full, ph, ctl);
        if (ok && it > 0) ok = mbar_wait(&bars->epi_free, ph ^ 1u, ctl);   // dQ, dV of the previous item read
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < N / 16; ++kk)   // dQ = dS K -> [256, 384)
          umma_bf16_ss(tmem + 256, kdesc(ads, kk, kPdsPanel), sw128_desc(ak + kk * 2048, panel, 1024), idesc_q,
                       kk > 0);
        for (int kk = 0; kk < N / 16; ++kk)   // dV = P^T dO -> [384, 512)
          umma_bf16_ss(tmem + 384, sw128_desc(ap + kk * 2048, kPdsPanel, 1024), sw128_desc(ado + kk * 2048, panel, 1024),
                       idesc_t, kk > 0);
        for (int kk = 0; kk < N / 16; ++kk)   // dK = dS^T Q -> [0, 128)
          umma_bf16_ss(tmem, sw128_desc(ads + kk * 2048, kPdsPanel, 1024), sw128_desc(aq + kk * 2048, panel, 1024),
                       idesc_t, kk > 0);
        umma_commit(&bars->o_full);
      }
      // every MMA issued has completed before the CTA frees tensor memory, and every load issued has
      // landed before it exits
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
      if (issued > 0) {
        mbar_wait_drain(&bars->load_qk, (issued - 1) & 1u, 20000000ull);
        mbar_wait_drain(&bars->load_vd, (issued - 1) & 1u, 20000000ull);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ row-owner warps
    const int r = warp * 32 + lane;   // TMEM lane = query row = key row of this thread
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    const int band = r / seg, pos = r - band * seg;   // this row's sequence within the item, and position
    const int k0 = band * seg;                        // the row's own keys: columns [k0, k0 + s)
    const uint32_t row_p = smem_u32(sp) + static_cast<uint32_t>(r) * 128u;
    const uint32_t row_ds = smem_u32(sds) + static_cast<uint32_t>(r) * 128u;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    bool ok = true;
    uint32_t it = 0;
    for (int item = static_cast<int>(blockIdx.x); ok && item < n_items; item += static_cast<int>(gridDim.x), ++it) {
      const uint32_t ph = it & 1u;
      const int first = item * a.pack;
      const int nseq = min(a.pack, total - first);
      const int N = round16b(nseq * seg);
      int tok = -1, bh = 0;
      if (band < nseq && pos < s) {
        const int gs = first + band;
        bh = static_cast<int>(fdiv(static_cast<uint32_t>(gs), p.f_per_bh));
        tok = token_of(g, p, gs - bh * p.n_seq, 0, pos);
      }
      const size_t gi = static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok);
      const float lse2 = tok >= 0 ? a.lse[gi] * kLog2e : 0.f;
      uint4 orow[16];
      {
        const uint4* src = reinterpret_cast<const uint4*>(a.o + gi * 128);
#pragma unroll
        for (int i = 0; i < 16; ++i) orow[i] = tok >= 0 ? src[i] : make_uint4(0, 0, 0, 0);
      }
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->load_vd, ph, ctl));
      const float D = (ok && tok >= 0) ? row_dot_out(sdo, panel, r, orow) : 0.f;   // D_i = dO_i . O_i
      if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full, ph, ctl));
      if (!ok) break;
      tc_fence_after();
      // P and dS = P o (dP - D) of this row, bf16, into shared memory (zero outside the row's own
      // sequence, and on rows of no sequence: those rows are K rows of dV and dK)
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t pp[16], pd[16];
        if (32 * c < N) {
          uint32_t sr[32], dr[32];
          tmem_ld32(t_row + 32 * c, sr);
          tmem_ld32(t_row + 128 + 32 * c, dr);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j = 32 * c + 2 * i - k0;   // key position within the row's own sequence
            const bool v0 = tok >= 0 && j >= 0 && j < s, v1 = tok >= 0 && j + 1 >= 0 && j + 1 < s;
            float e0, e1, d0, d1, s0, s1;
            ffma2(e0, e1, __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]), sl2, sl2, -lse2, -lse2);
            ffma2(d0, d1, __uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]), 1.f, 1.f, -D, -D);
            const float p0 = v0 ? ex2_approx(e0) : 0.f, p1 = v1 ? ex2_approx(e1) : 0.f;
            fmul2(s0, s1, p0, p1, d0, d1);
            pp[i] = pack2_rn(p0, p1);
            pd[i] = pack2_rn(v0 ? s0 : 0.f, v1 ? s1 : 0.f);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pp[i] = pd[i] = 0u;
        }
        // keys [32 c, 32 c + 32): panel c / 2, 16-byte chunks 4 (c % 2) .. + 3 of the 128-byte row
        const uint32_t pnl = static_cast<uint32_t>(c >> 1) * kPdsPanel;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t off = pnl + (((static_cast<uint32_t>(4 * (c & 1) + q)) ^ sw) << 4);
          st_shared_v4(row_p + off, pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
          st_shared_v4(row_ds + off, pd[4 * q], pd[4 * q + 1], pd[4 * q + 2], pd[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();   // P and dS -> visible to the MMAs (async proxy)
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int r = (warp - 4) * 32 + lane;   // the row of owner warp (warp - 4), lane `lane`
    const uint32_t t_row = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    const int band = r / seg, pos = r - band * seg;
    bool ok = true;
    uint32_t it = 0;
    for (int item = static_cast<int>(blockIdx.x); ok && item < n_items; item += static_cast<int>(gridDim.x), ++it) {
      const int first = item * a.pack;
      const int nseq = min(a.pack, total - first);
      int tok = -1, bh = 0;
      if (band < nseq && pos < s) {
        const int gs = first + band;
        bh = static_cast<int>(fdiv(static_cast<uint32_t>(gs), p.f_per_bh));
        tok = token_of(g, p, gs - bh * p.n_seq, 0, pos);
      }
      const size_t ro = (static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok)) * 128;
      if (a.accumulate && tok >= 0) {   // the earlier passes' fp32 shares of this row: into L2 now
        prefetch_l2(a.dq_acc + ro, 512u);
        prefetch_l2(a.dk_acc + ro, 512u);
      }
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_full, it & 1u, ctl));
      if (!ok) break;
      tc_fence_after();
      // dK first: its columns are where the next item's S goes
      if (a.final_out)
        write_row(t_row, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, a.dk_out + ro, nullptr);
      else
        write_row(t_row, tok >= 0, a.scale, a.accumulate ? a.dk_acc + ro : nullptr, nullptr, a.dk_acc + ro);
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      if (a.final_out)
        write_row(t_row + 256, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, a.dq_out + ro, nullptr);
      else
        write_row(t_row + 256, tok >= 0, a.scale, a.accumulate ? a.dq_acc + ro : nullptr, nullptr, a.dq_acc + ro);
      write_row(t_row + 384, tok >= 0, 1.f, nullptr, a.dv_out + ro, nullptr);
      tc_fence_before();
      mbar_arrive(&bars->epi_free);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_bwd_tc(const BwdTcArgs& a, cudaStream_t stream) {
  static std::atomic<unsigned long long> set{0}, set1{0}, set1p{0};
  cudaError_t e = max_dyn_smem_once(bwd_tc_kernel, kBwdSmemLimit, set);
  if (e != cudaSuccess) return e;
  e = max_dyn_smem_once(bwd_tc1_kernel<false>, kBwdSmemLimit, set1);
  if (e != cudaSuccess) return e;
  e = max_dyn_smem_once(bwd_tc1_kernel<true>, kBwdSmemLimit, set1p);
  if (e != cudaSuccess) return e;
  const int seqs = a.g.B * a.g.h * a.p.n_seq;
  if (seqs == 0) return cudaSuccess;
  if (a.single) {
    // persistent: one CTA per SM (each takes more than half of an SM's shared memory)
    const int items = (seqs + a.pack - 1) / a.pack, sms = num_sms_current();
    const unsigned grid = static_cast<unsigned>(sms > 0 && sms < items ? sms : items);
    if (a.pack > 1)
      bwd_tc1_kernel<true><<<grid, kBwdThreads, a.smem_bytes, stream>>>(a);
    else
      bwd_tc1_kernel<false><<<grid, kBwdThreads, a.smem_bytes, stream>>>(a);
  } else {
    if (a.pds == nullptr) return cudaErrorInvalidValue;
    int grid = num_sms_current();
    if (grid <= 0 || grid > kBwdPdsSlots) grid = kBwdPdsSlots;   // one scratch slot per CTA
    if (grid > seqs) grid = seqs;
    bwd_tc_kernel<<<static_cast<unsigned>(grid), kBwdThreads, a.smem_bytes, stream>>>(a);
  }
  return cudaGetLastError();
}

bool bwd_tc_plan(BwdTcArgs& a) {
  if (a.g.d != 128 || a.p.n_chunks != 1) return false;
  const int s = a.p.seq_len;
  if (s < 1 || s > 256) return false;
  const uint32_t rows8 = static_cast<uint32_t>((s + 7) & ~7);
  const uint32_t rows16 = static_cast<uint32_t>((s + 15) & ~15);
  // Two tiles: operand tiles of the sequence rounded to 16 rows (the column products contract over
  // it in steps of 16), and the P/dS scratch slot in the same panels.
  if (s > 128 && 8u * rows16 * 128u > kBwdPdsSlotMaxBytes) return false;
  a.panel_bytes = (s > 128 ? rows16 : rows8) * 128u;
  a.pds_slot_bytes = s > 128 ? 8u * a.panel_bytes : 0u;
  // Past the last allocation's second panel the MMAs read up to the last 128-row tile's end (A
  // operands) and the sequence rounded to 16 rows (B operands).
  const uint32_t tiles = static_cast<uint32_t>((s + 127) / 128);
  const uint32_t span = tiles * 128u * 128u;
  const uint32_t over = span > a.panel_bytes ? span - a.panel_bytes : 0u;
  a.guard_bytes = (over + 1023u) & ~1023u;
  a.smem_bytes = 1024u + 8u * a.panel_bytes + a.guard_bytes + kBwdVecBytes + kBwdBarBytes;
  if (a.smem_bytes > kBwdSmemLimit) return false;
  // One tile: six 128-row tiles (Q, K, V, dO, P, dS), as many sequences per CTA as fit in 128 rows
  a.single = tiles == 1 ? 1 : 0;
  a.seg_rows = static_cast<int>(rows8);
  a.pack = a.single ? 128 / a.seg_rows : 1;
  if (a.single)
    a.smem_bytes = a.pack > 1 ? 1024u + 12u * kPdsPanel + kBwdBarBytes
                              : 1024u + 8u * a.panel_bytes + a.guard_bytes + 4u * kPdsPanel + kBwdBarBytes;
  if (a.smem_bytes < kBwdSmemMin) a.smem_bytes = kBwdSmemMin;
  return true;
}

}  // namespace squad
