// Tensor-core (tcgen05 / TMEM / TMA) softmax attention over a batch of short sequences, sm_100a.
//
// One launch runs one attention pass of SQuad (local windows or global slots, paper §3.2) or plain
// full attention (paper eq. 5) over every (b, head). Each sequence is read straight out of the
// caller's [B, h, n, d] tensors through TMA boxes (geometry.cuh): no permuted copy is made.
//
// CTA organisation (persistent, one CTA per SM, 352 threads):
//   warps 0-3   softmax warpgroup 0 (TMEM lanes 0-127 of S0 / O0)
//   warps 4-7   softmax warpgroup 1 (S1 / O1)
//   warp 8      TMA producer: double-buffered Q tiles per warpgroup and a 3-stage ring of K/V blocks
//               (128 keys x 128 dims, bf16, 128-byte swizzle)
//   warp 9      TMEM allocator and MMA issuer (one thread)
//   warp 10     TMA store issuer for the outputs.
// A work unit is a pair of 128-row query tiles, one per softmax warpgroup; when both belong to the
// same sequence they share every K/V block. Per warpgroup, tensor memory holds the scores S (128 fp32
// columns) and the output accumulator O (128 columns). A softmax thread owns one query row: it reads
// the row's 128 scores in two 64-column loads, writes P as bf16 over the first half of S, and the PV
// product reads it from there (tcgen05.mma with A in tensor memory); the MMA issue order per
// warpgroup is ... S(b), [softmax], PV(b), S(b+1) ..., so the in-order tensor pipe finishes reading
// P(b) before S(b+1) overwrites it. Softmax is online across K/V blocks in one pass over each block's
// scores: the reference maximum, and with it O, changes only when a score exceeds it by more than
// 2^64 (in practice within the first block). The epilogue stages O through the tile's own Q buffer
// (free once its last S is done); the store warp writes it back with a TMA store of the same chunk
// box, which scatters the rows to their tokens and drops the padding rows.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "host_util.h"
#include "ptx.cuh"
#include "geometry.cuh"
#include "tc_pass.h"

namespace squad {

namespace {

constexpr int kThreads = 352;
constexpr int kWarpProducer = 8, kWarpMma = 9, kWarpStore = 10;
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
  uint64_t s_full[2], p_full[2], o_full[2], staged[2];
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
  t.bh = static_cast<int>(fdiv(static_cast<uint32_t>(tile), p.f_per_bh));
  const int rem = tile - t.bh * per_bh;
  t.sigma = static_cast<int>(fdiv(static_cast<uint32_t>(rem), p.f_chunks));
  t.q = rem - t.sigma * p.n_chunks;
  return t;
}

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

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
        mbar_init(&bars->q_empty[w][sl], 1);   // the store warp, once the tile's store has read it
      }
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->o_full[w], 1);
      mbar_init(&bars->staged[w], 4);   // one arrival per warp of the warpgroup
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&a.tm_q);
    prefetch_tmap(&a.tm_k);
    prefetch_tmap(&a.tm_v);
    prefetch_tmap(&a.tm_o);
  }
  if (warp == kWarpMma) {
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

  if (warp == kWarpProducer) {
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
  } else if (warp == kWarpMma) {
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
  } else if (warp == kWarpStore) {
    // ------------------------------------------------------------------ TMA store issuer
    if (lane == 0) {
      uint32_t st_cnt[2] = {0, 0};
      bool ok = true;
      int u_local = 0;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++u_local) {
        const int slot = u_local & 1;
        for (int w = 0; w < 2 && ok; ++w) {
          const int tile = 2 * unit + w;
          if (tile >= total_tiles) break;
          ok = mbar_wait(&bars->staged[w], st_cnt[w] & 1, ctl);
          ++st_cnt[w];
          if (!ok) break;
          const TileRef t = decode_tile(p, tile);
          const uint8_t* buf = sQ + (2 * w + slot) * kTile;
          int c[5];
          chunk_coords(g, p, a.global_variant, t.bh, t.sigma, t.q, 0, c);
          tma_store_5d(&a.tm_o, buf, c[0], c[1], c[2], c[3], c[4]);
          tma_store_5d(&a.tm_o, buf + kPanel, c[0] + 64, c[1], c[2], c[3], c[4]);
          bulk_commit_group();
          bulk_wait_read_all();   // the Q buffer may be refilled once the store has read it
          mbar_arrive(&bars->q_empty[w][slot]);
        }
      }
      bulk_wait_all();   // outputs written before the CTA exits
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;
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
      float m_used = -INFINITY;
      float l = 0.f;
      for (int b = 0; b < nb && ok; ++b) {
        ok = mbar_wait(&bars->s_full[wg], s_cnt & 1, ctl);
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();   // S(b) is ready, and so is every earlier PV (in-order tensor pipe)
        const int valid = chunk_valid_rows(p, b);
        if (active) {
          // One pass over the block's scores, 64 columns at a time, against a reference maximum m_used
          // (log2 units) that is raised only when a chunk's maximum exceeds it by more than 2^kHeadroom:
          // until then P = 2^(x - m_used) <= 2^kHeadroom is exact in fp32 and bf16 (the normalisation by
          // the row sum cancels m_used), and |O| <= n 2^kHeadroom max|V| stays far inside fp32 for any
          // n < 2^31. Raising m_used scales the P words already written in this block, the partial sums
          // and O by 2^(m_old - m_new), each row by its own factor (1 for rows that keep theirs); the
          // warp takes that path together (tensor-memory accesses are warp-wide). The first chunk of the
          // first block sets m_used (it holds at least one valid column, so its maximum is finite).
          constexpr float kHeadroom = 64.f;
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t r[64];
            tmem_ld64(t_s + 64 * c, r);
            if (64 * c + 64 > valid) {
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (64 * c + i >= valid) r[i] = __float_as_uint(-INFINITY);
            }
            // the scale is positive, so it is applied to the maximum instead of to every score
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 32; ++i)
              mx[i & 3] = fmax3(mx[i & 3], __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            const float cm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
            if (__any_sync(0xFFFFFFFFu, cm > m_used + kHeadroom)) {
              const float m_new = cm > m_used + kHeadroom ? cm : m_used;
              const float f = m_new > m_used ? ex2_approx(m_used - m_new) : 1.f;   // 0 while m_used is -inf
              tmem_wait_st();   // this block's P words written so far have landed
              if (c > 0) {
                uint32_t pw[16];
#pragma unroll 1
                for (int cc = 0; cc < 2; ++cc) {
                  tmem_ld16(t_s + 16 * cc, pw);
#pragma unroll
                  for (int j = 0; j < 16; ++j) {
                    const float x0 = __uint_as_float(pw[j] << 16) * f;
                    const float x1 = __uint_as_float(pw[j] & 0xFFFF0000u) * f;
                    pw[j] = pack_bf16x2(x0, x1);
                  }
                  tmem_st16(t_s + 16 * cc, pw);
                }
              }
              if (b > 0) {
                // O of the earlier blocks: PV(b-1) has completed (S(b) was issued after it)
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                  uint32_t o[64];
                  tmem_ld64(t_o + 64 * h, o);
#pragma unroll
                  for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                  tmem_st64v(t_o + 64 * h, o);
                }
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) ls[i] *= f;
              l *= f;
              m_used = m_new;
            }
            // P = 2^(x - m_used) (masked columns give 0), rounded to bf16 pairs (one conversion per two
            // values), packed two per 32-bit word over columns already read
            const float nm = -m_used;
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float e0, e1;
              ffma2(e0, e1, __uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]), sl2, sl2, nm, nm);
              const float x0 = ex2_approx(e0), x1 = ex2_approx(e1);
              fadd2(ls[2 * (j & 1)], ls[2 * (j & 1) + 1], x0, x1);
              pk[j] = pack_bf16x2(x0, x1);
            }
            tmem_st32_nowait(t_s + 32 * c, pk);   // waited for before p_full
          }
          l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        }
        tmem_wait_st();   // every P word in tensor memory before PV reads it
        tc_fence_before();
        mbar_arrive(&bars->p_full[wg]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 staged in this tile's Q buffer (its S products are done); the store
      // warp writes it back.
      ok = mbar_wait(&bars->o_full[wg], o_cnt & 1, ctl);
      ++o_cnt;
      if (!ok) break;
      tc_fence_after();
      if (active) {
        const uint32_t row_addr = smem_u32(sQ) + (2 * wg + slot) * kTile + row * 128;
        const float inv_l = 1.f / l;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[64];
          tmem_ld64(t_o + h * 64, o);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            // 16-byte chunk c of this panel's 128-byte row, at its 128-byte-swizzled position
            st_shared_v4(row_addr + h * kPanel + ((c ^ (row & 7)) << 4),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv_l, __uint_as_float(o[c * 8 + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv_l, __uint_as_float(o[c * 8 + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv_l, __uint_as_float(o[c * 8 + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv_l, __uint_as_float(o[c * 8 + 7]) * inv_l));
          }
        }
        if (a.lse != nullptr) {
          const int tok = token_of(g, p, t.sigma, t.q, row);
          if (tok >= 0) a.lse[static_cast<size_t>(t.bh) * g.n + tok] = (m_used + __log2f(l)) * 0.69314718055994531f;
        }
      }
      fence_proxy_async_smem();   // staging writes -> visible to the TMA store (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->staged[wg]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

cudaError_t launch_tc_pass(const TcPassArgs& args, int num_sms, cudaStream_t stream) {
  static std::atomic<unsigned long long> set{0};
  const cudaError_t e = max_dyn_smem_once(tc_pass_kernel, kSmemBytes, set);
  if (e != cudaSuccess) return e;
  const int total_tiles = args.g.B * args.g.h * args.p.n_seq * args.p.n_chunks;
  const int n_units = (total_tiles + 1) / 2;
  int grid = n_units < num_sms ? n_units : num_sms;
  if (grid < 1) return cudaSuccess;
  tc_pass_kernel<<<grid, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace squad
