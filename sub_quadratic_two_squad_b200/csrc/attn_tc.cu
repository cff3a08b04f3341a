// Tensor-core (tcgen05 / TMEM / TMA) softmax attention over a batch of short sequences, sm_100a.
//
// One launch runs one attention pass of SQuad (local windows or global slots, paper §3.2) or plain
// full attention (paper eq. 5) over every (b, head). Each sequence is read straight out of the
// caller's [B, h, n, d] tensors through TMA boxes (geometry.cuh): no permuted copy is made.
//
// CTA organisation (persistent, one CTA per SM, 384 threads):
//   warp 0      TMA producer: double-buffered Q tiles per warpgroup and a 3-stage ring of K/V blocks
//               (128 keys x 128 dims, bf16, 128-byte swizzle).
//   warp 1      TMEM allocator and MMA issuer (one thread).
//   warps 4-7   softmax warpgroup 0 (TMEM lanes 0-127 of S0 / O0)
//   warps 8-11  softmax warpgroup 1 (S1 / O1).
// A work unit is a pair of 128-row query tiles, one per softmax warpgroup; when both belong to the
// same sequence they share every K/V block. Per warpgroup, tensor memory holds the scores S (128 fp32
// columns) and the output accumulator O (128 columns). The softmax writes P as bf16 over the first
// half of S, and the PV product reads it from there (tcgen05.mma with A in tensor memory), so the
// MMA issue order per warpgroup is ... S(b), [softmax], PV(b), S(b+1) ... and the in-order tensor
// pipe finishes reading P(b) before S(b+1) overwrites it. Softmax is online across K/V blocks; the
// rescale of O is skipped unless the row maximum grew by more than 2^8. The epilogue stages O through
// the tile's own Q buffer (free once its last S is done) and writes it with coalesced stores.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "geometry.cuh"
#include "tc_pass.h"

namespace squad {

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 3;
constexpr uint32_t kPanel = 16384;   // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kTile = 2 * kPanel;
constexpr uint32_t kOffQ = 0;                      // Q[wg][slot]: 4 tiles
constexpr uint32_t kOffKV = 4 * kTile;             // K/V ring
constexpr uint32_t kOffBar = kOffKV + kStages * kTile;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // + barriers + alignment slack

static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Bars {
  uint64_t q_full[2][2], q_empty[2][2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct TileRef {
  int bh, sigma, q;
};

__device__ __forceinline__ TileRef decode_tile(const PassGeom& p, int tile) {
  TileRef t;
  const int per_bh = p.n_seq * p.n_chunks;
  t.bh = tile / per_bh;
  const int rem = tile - t.bh * per_bh;
  t.sigma = rem / p.n_chunks;
  t.q = rem - t.sigma * p.n_chunks;
  return t;
}

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// Physical byte offset of the 16-byte chunk `ch` (0..15 over 128 columns) of row `row` in a 2-panel
// 128-byte-swizzled tile: the layout TMA writes with SWIZZLE_128B and the MMA reads.
__device__ __forceinline__ uint32_t sw_off(int row, int ch) {
  return (ch >> 3) * kPanel + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
}

// Order of the K/V block loads of one unit (the producer issues them in this order, the MMA issuer
// finds each one's ring position from it): K0, K1, V0, K2, V1, ..., K(nb-1), V(nb-2), V(nb-1).
__device__ __forceinline__ int pos_k(int b) { return b == 0 ? 0 : 2 * b - 1; }
__device__ __forceinline__ int pos_v(int b, int nb) { return b == nb - 1 ? 2 * nb - 1 : 2 * b + 2; }

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) tc_pass_kernel(const __grid_constant__ TcPassArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PassGeom& p = a.p;
  const Grid& g = a.g;

  // Zero the K/V ring once: rows of a block past its box are read by the MMA (masked to P = 0), so
  // they must hold finite values.
  for (uint32_t i = threadIdx.x; i < kStages * kTile / 16; i += kThreads)
    reinterpret_cast<uint4*>(sKV)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int w = 0; w < 2; ++w) {
      for (int sl = 0; sl < 2; ++sl) {
        mbar_init(&bars->q_full[w][sl], 1);
        mbar_init(&bars->q_empty[w][sl], 4);   // one arrival per warp of the warpgroup
      }
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->o_full[w], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&a.tm_q);
    prefetch_tmap(&a.tm_k);
    prefetch_tmap(&a.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};

  const int total_tiles = g.B * g.h * p.n_seq * p.n_chunks;
  const int n_units = (total_tiles + 1) / 2;
  const int nb = p.n_chunks;
  const uint32_t box_bytes = 2u * static_cast<uint32_t>(p.chunk_rows) * 128u;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t q_loads[2][2] = {{0, 0}, {0, 0}};
      uint32_t kv_loads = 0;
      bool ok = true;
      int u_local = 0;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++u_local) {
        const int slot = u_local & 1;
        TileRef t[2];
        t[0] = decode_tile(p, 2 * unit);
        const bool two = 2 * unit + 1 < total_tiles;
        if (two) t[1] = decode_tile(p, 2 * unit + 1);
        const bool shared = two && t[0].bh == t[1].bh && t[0].sigma == t[1].sigma;
        const int nw = two ? 2 : 1;
        const int nsrc = (two && !shared) ? 2 : 1;
        for (int w = 0; w < nw && ok; ++w) {
          uint32_t& n_ld = q_loads[w][slot];
          if (n_ld > 0 && !mbar_wait(&bars->q_empty[w][slot], (n_ld - 1) & 1, ctl)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->q_full[w][slot], box_bytes);
          for (int panel = 0; panel < 2; ++panel) {
            int c[5];
            chunk_coords(g, p, a.global_variant, t[w].bh, t[w].sigma, t[w].q, panel, c);
            tma_load_5d(sQ + (2 * w + slot) * kTile + panel * kPanel, &a.tm_q, &bars->q_full[w][slot], c[0], c[1],
                        c[2], c[3], c[4]);
          }
          ++n_ld;
        }
        for (int j = 0; j < 2 * nb && ok; ++j) {
          // position j of the load order: K(b) or V(b)
          const bool is_k = (j == 0) || (j < 2 * nb - 1 && (j & 1));
          const int blk = is_k ? (j + 1) / 2 : (j == 2 * nb - 1 ? nb - 1 : j / 2 - 1);
          for (int src = 0; src < nsrc && ok; ++src) {
            const uint32_t s = kv_loads % kStages;
            if (kv_loads >= kStages && !mbar_wait(&bars->kv_empty[s], ((kv_loads / kStages) + 1) & 1, ctl)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars->kv_full[s], box_bytes);
            for (int panel = 0; panel < 2; ++panel) {
              int c[5];
              chunk_coords(g, p, a.global_variant, t[src].bh, t[src].sigma, blk, panel, c);
              tma_load_5d(sKV + s * kTile + panel * kPanel, is_k ? &a.tm_k : &a.tm_v, &bars->kv_full[s], c[0], c[1],
                          c[2], c[3], c[4]);
            }
            ++kv_loads;
          }
        }
      }
      // Let every load this thread issued land before the CTA can exit (bounded).
      const uint32_t first = kv_loads > kStages ? kv_loads - kStages : 0;
      for (uint32_t i = first; i < kv_loads; ++i)
        mbar_wait_drain(&bars->kv_full[i % kStages], (i / kStages) & 1, 20000000ull);
      for (int w = 0; w < 2; ++w)
        for (int sl = 0; sl < 2; ++sl)
          if (q_loads[w][sl] > 0) mbar_wait_drain(&bars->q_full[w][sl], (q_loads[w][sl] - 1) & 1, 20000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16(128, 128, true);
      uint32_t kv_base = 0, q_cnt[2][2] = {{0, 0}, {0, 0}}, p_cnt[2] = {0, 0};
      bool ok = true;
      int u_local = 0;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++u_local) {
        const int slot = u_local & 1;
        TileRef t[2];
        t[0] = decode_tile(p, 2 * unit);
        const bool two = 2 * unit + 1 < total_tiles;
        if (two) t[1] = decode_tile(p, 2 * unit + 1);
        const bool shared = two && t[0].bh == t[1].bh && t[0].sigma == t[1].sigma;
        const int nw = two ? 2 : 1;
        const int nsrc = (two && !shared) ? 2 : 1;
        for (int b = 0; b <= nb && ok; ++b) {
          for (int w = 0; w < nw && ok; ++w) {
            const int src = shared ? 0 : w;
            const bool last_user = !shared || w == nw - 1;
            if (b >= 1) {
              // O_w += P_w(b-1) V(b-1), P read from the first columns of S_w
              ok = mbar_wait(&bars->p_full[w], p_cnt[w] & 1, ctl);
              ++p_cnt[w];
              const uint32_t iv = kv_base + static_cast<uint32_t>(pos_v(b - 1, nb) * nsrc + src);
              if (ok && (w == 0 || !shared)) ok = mbar_wait(&bars->kv_full[iv % kStages], (iv / kStages) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              const int nk = round16(chunk_valid_rows(p, b - 1));
              const uint32_t va = smem_u32(sKV + (iv % kStages) * kTile);
              for (int kk = 0; kk < nk / 16; ++kk)
                umma_bf16_ts(tmem + 256 * w + 128, tmem + 256 * w + kk * 8, sw128_desc(va + kk * 2048, kPanel, 1024),
                             idesc_pv, (b - 1 > 0 || kk > 0) ? 1u : 0u);
              if (b == nb) umma_commit(&bars->o_full[w]);
              if (last_user) umma_commit(&bars->kv_empty[iv % kStages]);
            }
            if (b < nb) {
              // S_w = Q_w K(b)^T
              if (b == 0) {
                ok = mbar_wait(&bars->q_full[w][slot], q_cnt[w][slot] & 1, ctl);
                ++q_cnt[w][slot];
              }
              const uint32_t ik = kv_base + static_cast<uint32_t>(pos_k(b) * nsrc + src);
              if (ok && (w == 0 || !shared)) ok = mbar_wait(&bars->kv_full[ik % kStages], (ik / kStages) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              const uint32_t idesc_s = idesc_bf16(128, round16(chunk_valid_rows(p, b)), false);
              const uint32_t qa = smem_u32(sQ + (2 * w + slot) * kTile);
              const uint32_t ka = smem_u32(sKV + (ik % kStages) * kTile);
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
                umma_bf16_ss(tmem + 256 * w, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), idesc_s,
                             kk > 0);
              }
              umma_commit(&bars->s_full[w]);
              if (last_user) umma_commit(&bars->kv_empty[ik % kStages]);
            }
          }
        }
        kv_base += static_cast<uint32_t>(2 * nb * nsrc);
      }
      // Wait (bounded) until every MMA issued above has completed before TMEM can be released.
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_s = tmem + 256 * wg + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t t_o = t_s + 128;
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    int u_local = 0;
    for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++u_local) {
      const int slot = u_local & 1;
      const int tile = 2 * unit + wg;
      if (tile >= total_tiles) break;
      const TileRef t = decode_tile(p, tile);
      // A warp whose 32 query rows are all padding skips the arithmetic but keeps every barrier.
      const bool active = wq * 32 < chunk_valid_rows(p, t.q);
      const int my_tok = token_of(g, p, t.sigma, t.q, row);
      float m_used = -INFINITY;
      float l = 0.f;    // sum of the bf16-rounded weights: normalises O
      float le = 0.f;   // sum of the unrounded weights: the log-sum-exp
      for (int b = 0; b < nb && ok; ++b) {
        ok = mbar_wait(&bars->s_full[wg], s_cnt & 1, ctl);
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();   // S(b) is ready, and so is every earlier PV (in-order tensor pipe)
        const int valid = chunk_valid_rows(p, b);
        const int nk = round16(valid);
        uint32_t r[32];
        float m_new = m_used;
        if (active) {
          // pass 1: row maximum (4 independent partial maxima; the scale is positive, so it is applied
          // to the maximum instead of to every score)
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c * 32 < nk) {
              tmem_ld32(t_s + c * 32, r);
              if (c * 32 + 32 <= valid) {
#pragma unroll
                for (int i = 0; i < 32; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (c * 32 + i < valid) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
              }
            }
          }
          m_new = fmaxf(m_used, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2);
        }
        if (b > 0) {
          // Rescale O only when the running maximum grew by more than 2^8 (until then the unscaled
          // exponentials stay below 256). PV(b-1) has completed: S(b) was issued after it.
          const bool need = active && m_new > m_used + 8.f;
          if (__any_sync(0xffffffffu, need)) {
            const float f = need ? ex2_approx(m_used - m_new) : 1.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              tmem_ld32(t_o + c * 32, r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
              tmem_st32(t_o + c * 32, r);
            }
            if (need) {
              l *= f;
              le *= f;
              m_used = m_new;
            }
          }
        } else {
          m_used = m_new;
        }
        if (active) {
          // pass 2: P = 2^(x - m) rounded to bf16 on the integer pipe (add half an ulp, drop the low
          // half) and packed two per TMEM column over the first half of S.
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
          float lx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c * 32 < nk) {
              tmem_ld32(t_s + c * 32, r);
              const bool full = c * 32 + 32 <= valid;
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                uint32_t bits[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  float x = ex2_approx(fmaf(__uint_as_float(r[i + e]), sl2, -m_used));
                  if (!full && c * 32 + i + e >= valid) x = 0.f;
                  lx[(i + e) & 3] += x;
                  bits[e] = (__float_as_uint(x) + 0x8000u) & 0xFFFF0000u;
                  ls[(i + e) & 3] += __uint_as_float(bits[e]);
                }
                pk[i >> 1] = __byte_perm(bits[0], bits[1], 0x7632);
              }
              tmem_st16(t_s + c * 16, pk);
            }
          }
          l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          le += (lx[0] + lx[1]) + (lx[2] + lx[3]);
        }
        tc_fence_before();
        mbar_arrive(&bars->p_full[wg]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 staged in this tile's Q buffer (its S products are done) -> coalesced
      // global stores; then the Q buffer goes back to the producer.
      ok = mbar_wait(&bars->o_full[wg], o_cnt & 1, ctl);
      ++o_cnt;
      if (!ok) break;
      tc_fence_after();
      uint8_t* buf = sQ + (2 * wg + slot) * kTile;
      if (active) {
        const float inv_l = 1.f / l;
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(t_o + c * 32, r);
#pragma unroll
          for (int h8 = 0; h8 < 4; ++h8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[h8 * 8 + 0]) * inv_l, __uint_as_float(r[h8 * 8 + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(r[h8 * 8 + 2]) * inv_l, __uint_as_float(r[h8 * 8 + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(r[h8 * 8 + 4]) * inv_l, __uint_as_float(r[h8 * 8 + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(r[h8 * 8 + 6]) * inv_l, __uint_as_float(r[h8 * 8 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(buf + sw_off(row, c * 4 + h8)) = v;
          }
        }
        __syncwarp();
        const size_t head_base = static_cast<size_t>(t.bh) * g.n;
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
          const int rr = 2 * it + (lane >> 4);   // row within this warp's 32
          const int ch = lane & 15;
          const int tok = __shfl_sync(0xffffffffu, my_tok, rr);
          if (tok >= 0) {
            const uint4 v = *reinterpret_cast<const uint4*>(buf + sw_off(wq * 32 + rr, ch));
            *reinterpret_cast<uint4*>(a.out + (head_base + tok) * 128 + ch * 8) = v;
          }
        }
        if (a.lse != nullptr && my_tok >= 0) a.lse[head_base + my_tok] = (m_used + __log2f(le)) * 0.69314718055994531f;
      }
      // The generic-proxy writes and reads of the staging area must be ordered before the next TMA
      // load into this Q buffer.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_empty[wg][slot]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

cudaError_t launch_tc_pass(const TcPassArgs& args, int num_sms, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(tc_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int total_tiles = args.g.B * args.g.h * args.p.n_seq * args.p.n_chunks;
  const int n_units = (total_tiles + 1) / 2;
  int grid = n_units < num_sms ? n_units : num_sms;
  if (grid < 1) return cudaSuccess;
  tc_pass_kernel<<<grid, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace squad
