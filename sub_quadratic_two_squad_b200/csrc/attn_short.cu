// Tensor-core attention over sequences of at most 256 tokens, sm_100a: one SQuad pass, or both passes
// fused, in one persistent launch (paper §3.2: the local pass inside windows, then the global pass
// across windows with the local output as values).
//
// Each of Q, K, V of a sequence arrives as one TMA box (the whole window, or the whole slot across all
// windows) in a shared-memory ring; S = Q K^T is one tcgen05.mma per 16-deep K step with N = the
// sequence length rounded up to 16 (<= 256), so the whole row of scores is in tensor memory at once.
// The softmax reads it once: exponentials are taken against the maximum of the first 64 columns, a
// reference raised (and the P already written rescaled) only if a later column exceeds it by more than
// 2^100; the normalisation by the row sum cancels the reference.
//
// CTA organisation (one CTA per SM, 352 threads):
//   warps 0-3   softmax warpgroup 0 (TMEM lanes 0-127 of its S / O)
//   warps 4-7   softmax warpgroup 1
//   warp 8      scheduler + TMA producer   warp 9  TMEM allocator + MMA issuer   warp 10  TMA stores
// Work units are claimed dynamically (an atomic counter) and handed to the other warps through a small
// queue in shared memory. A unit is either one sequence of 129-256 tokens (its two 128-row query tiles
// go to the two warpgroups and share K and V) or two sequences of at most 128 tokens (one per
// warpgroup).
//
// Fused passes: the unit order is L(0) L(1) .. L(lag-1), then L(k) G(k-lag) for each head k, then the
// remaining G: a head's second-pass units trail its first-pass units by `lag` heads, so the second
// pass re-reads that head's Q, K and first-pass output from L2. Before loading the values of a
// second-pass unit (the first pass's output), the producer waits, bounded, until every first-pass unit
// of that head has been stored (a per-head counter the store warp increments with release semantics
// after its TMA stores complete).
//
// Ring: allocations (one per Q, K or V box) get consecutive offsets in a byte ring; every warp derives
// the same offsets from the same unit sequence. Q and K allocations are released when the S products
// that read them complete, a V allocation when the output staged in it has been stored: the softmax
// warps write O (normalised, bf16) into the V allocation after PV has read it, and the store warp
// writes it back with a TMA store of the sequence's box. So the next units' loads overlap this unit's
// softmax and epilogue.
// Tensor memory per warpgroup (256 columns): S in [0, N), P (bf16 pairs) over [0, N/2), and O in
// [128, 256) when N <= 128, else in [N/2, N/2 + 128) over consumed scores; a unit's S then waits until
// the warpgroup has read the previous unit's O.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "host_util.h"
#include "ptx.cuh"
#include "geometry.cuh"
#include "short_pass.h"
#include "unit_sched.cuh"

namespace squad {

namespace {

using namespace units;

constexpr int kThreads = 352;
constexpr int kWarpProducer = 8, kWarpMma = 9, kWarpStore = 10;
constexpr int kND = 16;   // ring allocations in flight (full/empty barrier pairs)
constexpr int kQ = 4;     // unit queue entries
constexpr uint32_t kSmemLimit = 232448;

struct Bars {
  uint64_t full[kND], empty[kND];
  uint64_t qf[kQ], qe[kQ];
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2], staged[2];
  uint64_t drain;
  int unit_q[kQ];
  uint32_t tmem_base;
  uint32_t abort;
};
constexpr uint32_t kBarBytes = 512;
static_assert(sizeof(Bars) <= kBarBytes, "barrier block");

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) short_kernel(const __grid_constant__ ShortArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t RB = a.ring_bytes;
  Bars* bars = reinterpret_cast<Bars*>(ring + RB + a.guard_bytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const int n_total = total_units(a);

  // Zero the ring and guard once: rows past a sequence inside an allocation (and past the ring) are
  // read by the MMAs and must hold finite values.
  for (uint32_t i = threadIdx.x; i < (RB + a.guard_bytes) / 16; i += kThreads)
    reinterpret_cast<uint4*>(ring)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kND; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < kQ; ++i) {
      mbar_init(&bars->qf[i], 1);
      mbar_init(&bars->qe[i], 10);   // MMA issuer, store warp and the 8 softmax warps
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->o_full[w], 1);
      mbar_init(&bars->o_free[w], 4);
      mbar_init(&bars->staged[w], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    for (int ps = 0; ps < a.n_passes; ++ps) {
      prefetch_tmap(&a.pass[ps].tm_q);
      prefetch_tmap(&a.pass[ps].tm_k);
      prefetch_tmap(&a.pass[ps].tm_v);
      prefetch_tmap(&a.pass[ps].tm_o);
    }
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

  // Next unit from the queue (consumers); returns false at the end of the work.
  // (A failed wait counts as the end of the work.)
  auto next_unit = [&](uint32_t& qi, int& U, bool arrive) -> bool {
    const uint32_t e = qi % kQ;
    U = mbar_wait(&bars->qf[e], (qi / kQ) & 1, ctl) ? *reinterpret_cast<volatile int*>(&bars->unit_q[e]) : n_total;
    if (arrive) mbar_arrive(&bars->qe[e]);
    ++qi;
    return U < n_total;
  };

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ scheduler + TMA producer
    if (lane == 0) {
      Cursor cur;
      uint32_t tail = 0, vstart[kND] = {};
      uint32_t qi = 0;
      bool ok = true;
      // Wait until allocation `idx`, virtual range [vs, vs + sz), may be filled. Its bytes were last used
      // by virtual [vs - RB, vs + sz - RB): every live allocation starting before vs + sz - RB overlaps
      // them, and live allocations start in increasing order, so release the oldest ones until the
      // oldest starts at or after that point (or none is left). The allocation whose barriers it reuses
      // (idx - kND) must be released too.
      auto make_room = [&](uint32_t idx, uint32_t vs, uint32_t sz) -> bool {
        while (tail < idx &&
               (idx - tail >= static_cast<uint32_t>(kND) || (vs + sz > RB && vstart[tail % kND] < vs + sz - RB))) {
          if (!mbar_wait(&bars->empty[tail % kND], (tail / kND) & 1, ctl)) return false;
          ++tail;
        }
        vstart[idx % kND] = vs;
        return true;
      };
      // Q, K and V of one sequence are the same box of three tensors: its coordinates c are computed
      // once per sequence.
      auto load = [&](const PassView& ps, const CUtensorMap* m, const int (&c)[5], uint32_t idx, uint32_t off,
                      uint32_t vs) -> bool {
        if (!make_room(idx, vs, ps.alloc)) return false;
        uint64_t* fb = &bars->full[idx % kND];
        mbar_arrive_expect_tx(fb, 2u * static_cast<uint32_t>(ps.p.seq_len) * 128u);
        tma_load_5d(ring + off, m, fb, c[0], c[1], c[2], c[3], c[4]);
        tma_load_5d(ring + off + ps.panel, m, fb, c[0] + 64, c[1], c[2], c[3], c[4]);
        return true;
      };
      while (ok) {
        // claim the next unit and publish it to the other warps
        const uint32_t e = qi % kQ;
        if (qi >= kQ && !mbar_wait(&bars->qe[e], ((qi / kQ) + 1) & 1, ctl)) break;
        const int U = static_cast<int>(atomicAdd(a.work, 1u));
        bars->unit_q[e] = U;
        mbar_arrive(&bars->qf[e]);   // release: the entry is visible to the waiting warps
        ++qi;
        if (U >= n_total) break;
        const Unit u = plan_unit(a, U, cur, RB);
        const PassView ps = view_of(a, u.pass);
        const int nsrc = u.shared ? 1 : u.nw;
        int cs[2][5];
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if (w < nsrc) chunk_coords(g, ps.p, ps.variant, u.bh, u.sigma[w], 0, 0, cs[w]);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w < nsrc && ok) {
            ok = load(ps, ps.q, cs[w], u.q[w], u.qo[w], u.qvs[w]);
            if (ok) ok = load(ps, ps.k, cs[w], u.k[w], u.ko[w], u.kvs[w]);
          }
        }
        if (ok && u.pass == 1) {
          // values = the first pass's output for this head: wait until all of it is in memory
          const uint32_t need = static_cast<uint32_t>(a.pass[0].units_per_head);
          const uint32_t* cnt = &a.done[u.bh];
          if (ld_acquire_gpu(cnt) < need) {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(cnt) < need) {
              if (*ctl.abort || globaltimer_ns() - t0 > a.timeout_ns) {
                record_timeout(ctl);
                ok = false;
                break;
              }
              __nanosleep(256);
            }
          }
          fence_proxy_async_global();   // the TMA loads below must observe those stores
        }
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if (w < nsrc && ok) ok = load(ps, ps.v, cs[w], u.v[w], u.vo[w], u.vvs[w]);
      }
      if (!ok) {   // make sure the other warps see the end of the work
        for (int i = 0; i < kQ; ++i) {
          const uint32_t e = qi % kQ;
          if (qi >= kQ) mbar_wait_drain(&bars->qe[e], ((qi / kQ) + 1) & 1, 20000000ull);
          bars->unit_q[e] = n_total;
          mbar_arrive(&bars->qf[e]);
          ++qi;
        }
      }
      // Let every load this thread issued land before the CTA can exit (bounded).
      const uint32_t first = cur.ai > static_cast<uint32_t>(kND) ? cur.ai - kND : 0;
      for (uint32_t i = first; i < cur.ai; ++i) mbar_wait_drain(&bars->full[i % kND], (i / kND) & 1, 20000000ull);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16(128, 128, true);
      Cursor cur;
      uint32_t qi = 0, p_cnt[2] = {0, 0}, wu[2] = {0, 0}, prev_ooff[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      int U;
      bool ok = true;
      while (ok && next_unit(qi, U, true)) {
        const Unit u = plan_unit(a, U, cur, RB);
        const uint32_t panel = u.pass ? a.pass[1].panel_bytes : a.pass[0].panel_bytes;
        const int N = round16(u.pass ? a.pass[1].p.seq_len : a.pass[0].p.seq_len);
        const uint32_t o_off = N > 128 ? static_cast<uint32_t>(N / 2) : 128u;
        const uint32_t idesc_s = idesc_bf16(128, N, false);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w >= u.nw || !ok) break;
          if (w == 0 || !u.shared) {
            ok = mbar_wait(&bars->full[u.q[w] % kND], (u.q[w] / kND) & 1, ctl);
            if (ok) ok = mbar_wait(&bars->full[u.k[w] % kND], (u.k[w] / kND) & 1, ctl);
          }
          if (ok && prev_ooff[w] != 0xFFFFFFFFu && static_cast<uint32_t>(N) > prev_ooff[w])
            ok = mbar_wait(&bars->o_free[w], (wu[w] - 1) & 1, ctl);   // previous O read before S overwrites it
          if (!ok) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(ring + u.qo[w]) + (u.shared ? static_cast<uint32_t>(w) * 16384u : 0u);
          const uint32_t ka = smem_u32(ring + u.ko[w]);
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * panel + (kk & 3) * 32;
            umma_bf16_ss(tmem + 256 * w, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), idesc_s,
                         kk > 0);
          }
          umma_commit(&bars->s_full[w]);
          if (!u.shared || w == u.nw - 1) {
            umma_commit(&bars->empty[u.q[w] % kND]);
            umma_commit(&bars->empty[u.k[w] % kND]);
          }
        }
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w >= u.nw || !ok) break;
          ok = mbar_wait(&bars->p_full[w], p_cnt[w] & 1, ctl);
          ++p_cnt[w];
          if (ok && (w == 0 || !u.shared)) ok = mbar_wait(&bars->full[u.v[w] % kND], (u.v[w] / kND) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t va = smem_u32(ring + u.vo[w]);
          for (int kk = 0; kk < N / 16; ++kk)
            umma_bf16_ts(tmem + 256 * w + o_off, tmem + 256 * w + kk * 8,
                         sw128_desc(va + kk * 2048, panel, 1024), idesc_pv, kk > 0);
          if (!u.shared) umma_commit(&bars->o_full[w]);
        }
        if (ok && u.shared) {   // both tiles read the one V allocation: neither overwrites it before both PVs
          umma_commit(&bars->o_full[0]);
          umma_commit(&bars->o_full[1]);
        }
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w < u.nw) {
            ++wu[w];
            prev_ooff[w] = o_off;
          }
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
    }
  } else if (warp == kWarpStore) {
    // ------------------------------------------------------------------ TMA store issuer
    if (lane == 0) {
      Cursor cur;
      uint32_t qi = 0, st_cnt[2] = {0, 0};
      int U;
      bool ok = true;
      while (ok && next_unit(qi, U, true)) {
        const Unit u = plan_unit(a, U, cur, RB);
        const PassView ps = view_of(a, u.pass);
        const int nseq = u.shared ? 1 : u.nw;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w < u.nw && ok) {
            ok = mbar_wait(&bars->staged[w], st_cnt[w] & 1, ctl);
            ++st_cnt[w];
          }
        }
        if (!ok) break;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (w < nseq) {
            int c[5];
            chunk_coords(g, ps.p, ps.variant, u.bh, u.sigma[w], 0, 0, c);
            const uint8_t* src = ring + u.vo[w];
            tma_store_5d(ps.o, src, c[0], c[1], c[2], c[3], c[4]);
            tma_store_5d(ps.o, src + ps.panel, c[0] + 64, c[1], c[2], c[3], c[4]);
          }
        }
        bulk_commit_group();
        bulk_wait_read_all();   // the V allocations may be refilled once their stores have read them
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if (w < nseq) mbar_arrive(&bars->empty[u.v[w] % kND]);
        if (a.n_passes == 2 && u.pass == 0) {
          // publish this head's progress once the output is in global memory
          bulk_wait_all();
          fence_proxy_async_global();
          red_release_gpu_add(&a.done[u.bh], 1u);
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
    const float sl2 = a.scale_log2;
    Cursor cur;
    uint32_t qi = 0, s_cnt = 0, o_cnt = 0;
    int U;
    bool ok = true;
    while (ok) {
      const bool more = next_unit(qi, U, false);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qe[(qi - 1) % kQ]);
      if (!more) break;
      const Unit u = plan_unit(a, U, cur, RB);
      if (wg >= u.nw) continue;
      const int s_len = u.pass ? a.pass[1].p.seq_len : a.pass[0].p.seq_len;
      const uint32_t panel = u.pass ? a.pass[1].panel_bytes : a.pass[0].panel_bytes;
      const int N = round16(s_len);
      const uint32_t t_o = t_s + (N > 128 ? static_cast<uint32_t>(N / 2) : 128u);
      const int nchunk = (N + 63) / 64;
      const int row0 = u.shared ? 128 * wg : 0;   // first sequence row of this tile
      const int src = u.shared ? 0 : wg;
      const uint32_t v_off = src ? u.vo[1] : u.vo[0];
      const int sigma = src ? u.sigma[1] : u.sigma[0];
      int valid = s_len - row0;
      if (valid > 128) valid = 128;
      const bool active = wq * 32 < valid;        // warps of padding rows only keep the barriers
      ok = mbar_wait(&bars->s_full[wg], s_cnt & 1, ctl);
      ++s_cnt;
      if (!ok) break;
      tc_fence_after();
      float m = -INFINITY, l = 0.f;
      if (active) {
        uint32_t r[64];
        // One pass over the scores. The exponentials are taken against m, the scaled maximum of the
        // columns read so far, which is raised only when a later column exceeds it by more than 100 (in
        // log2 units): until then every exponential is below 2^100 and the row sum below 2^109, finite
        // in fp32 and bf16, and the normalisation by the row sum cancels m. Raising m lowers the packed P
        // already written and the partial sums by 2^(m_old - m_new); the warp does it together (the
        // TMEM accesses are warp-wide), each row with its own factor (1 for rows that keep their m).
        const float kHeadroom = 100.f;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int c = 0; c < nchunk; ++c) {
          tmem_ld64(t_s + 64 * c, r);
          if (64 * c + 64 > s_len) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (64 * c + i >= s_len) r[i] = __float_as_uint(-INFINITY);
          }
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 32; ++i)
            mx[i & 3] = fmax3(mx[i & 3], __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          const float cm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
          if (c == 0) {
            m = cm;   // chunk 0 holds at least one column of the sequence: finite
          } else if (__any_sync(0xFFFFFFFFu, cm > m + kHeadroom)) {
            const float m_new = cm > m + kHeadroom ? cm : m;
            const float f = m_new > m ? ex2_approx(m - m_new) : 1.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) ls[i] *= f;
            uint32_t pw[16];   // 16 columns at a time: the current chunk's 64 scores stay live
            tmem_wait_st();    // the P words written so far have landed
#pragma unroll 1
            for (int cc = 0; cc < 2 * c; ++cc) {
              tmem_ld16(t_s + 16 * cc, pw);
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float x0 = __uint_as_float(pw[j] << 16) * f;
                const float x1 = __uint_as_float(pw[j] & 0xFFFF0000u) * f;
                pw[j] = pack_bf16x2(x0, x1);
              }
              tmem_st16(t_s + 16 * cc, pw);
            }
            m = m_new;
          }
          const float nm = -m;
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float e0, e1;
            ffma2(e0, e1, __uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]), sl2, sl2, nm, nm);
            const float x0 = ex2_approx(e0), x1 = ex2_approx(e1);
            fadd2(ls[2 * (j & 1)], ls[2 * (j & 1) + 1], x0, x1);
            pk[j] = pack_bf16x2(x0, x1);
          }
          tmem_st32_nowait(t_s + 32 * c, pk);   // over scores already read; waited for below
        }
        tmem_wait_st();
        l = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      }
      tc_fence_before();
      mbar_arrive(&bars->p_full[wg]);

      // epilogue: O / l -> bf16 into this tile's rows of the V allocation (PV has finished reading it);
      // the store warp writes the allocation back with the sequence's box.
      ok = mbar_wait(&bars->o_full[wg], o_cnt & 1, ctl);
      ++o_cnt;
      if (!ok) break;
      tc_fence_after();
      const int vrow = row0 + row;   // row within the V allocation's panels
      const uint32_t row_addr = smem_u32(ring + v_off) + static_cast<uint32_t>(vrow) * 128u;
      const bool store_row = row < valid;
      const float inv_l = active ? 1.f / l : 0.f;
      {
        // both halves of O into registers (the first packed to bf16 at once), then release O
        uint32_t pk0[32], o[64];
        if (active) tmem_ld64(t_o, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) pk0[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (active) tmem_ld64(t_o + 64, o);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->o_free[wg]);
        if (store_row) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + ((c ^ (vrow & 7)) << 4), pk0[4 * c], pk0[4 * c + 1], pk0[4 * c + 2], pk0[4 * c + 3]);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + panel + ((c ^ (vrow & 7)) << 4),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv_l, __uint_as_float(o[c * 8 + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv_l, __uint_as_float(o[c * 8 + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv_l, __uint_as_float(o[c * 8 + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv_l, __uint_as_float(o[c * 8 + 7]) * inv_l));
        }
      }
      float* lse = u.pass ? a.pass[1].lse : a.pass[0].lse;
      if (lse != nullptr && store_row) {
        const PassGeom pg = u.pass ? a.pass[1].p : a.pass[0].p;
        const int tok = token_of(g, pg, sigma, 0, vrow);
        if (tok >= 0) lse[static_cast<size_t>(u.bh) * g.n + tok] = (m + __log2f(l)) * 0.69314718055994531f;
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

bool short_plan(ShortArgs& a) {
  if (a.n_passes < 1 || a.n_passes > 2 || a.g.d != 128) return false;
  uint32_t guard = 2048u, max_alloc = 0u;
  for (int i = 0; i < a.n_passes; ++i) {
    ShortPass& ps = a.pass[i];
    const int s = ps.p.seq_len;
    if (s < 1 || s > 256 || ps.p.n_chunks != 1) return false;
    const uint32_t rows8 = static_cast<uint32_t>((s + 7) & ~7);
    ps.panel_bytes = rows8 * 128u;
    ps.alloc_bytes = 2u * ps.panel_bytes;
    ps.units_per_head = s > 128 ? ps.p.n_seq : (ps.p.n_seq + 1) / 2;
    // Past an allocation's end the MMAs read at most the second 128-row query tile of a 256-row pair
    // (or the only 128-row tile), and K/V rows up to the sequence length rounded to 16.
    const uint32_t tile_span = s > 128 ? 32768u : 16384u;
    const uint32_t over = tile_span > ps.panel_bytes ? tile_span - ps.panel_bytes : 0u;
    if (over > guard) guard = over;
    if (ps.alloc_bytes > max_alloc) max_alloc = ps.alloc_bytes;
  }
  a.guard_bytes = (guard + 1023u) & ~1023u;
  const uint32_t fixed = 1024u + a.guard_bytes + kBarBytes;
  a.ring_bytes = ((kSmemLimit - fixed) / 1024u) * 1024u;
  // One unit holds up to 6 allocations (or 3 for a shared pair) at once.
  for (int i = 0; i < a.n_passes; ++i) {
    const uint32_t need = (a.pass[i].p.seq_len > 128 ? 3u : 6u) * a.pass[i].alloc_bytes;
    if (need + max_alloc <= a.ring_bytes) continue;   // + max_alloc: room lost to a wrap
    // One pass has one allocation size: a ring of whole allocations loses nothing at the wrap.
    if (a.n_passes != 1 || need > a.ring_bytes) return false;
    a.ring_bytes = a.ring_bytes / a.pass[i].alloc_bytes * a.pass[i].alloc_bytes;
  }
  a.smem_bytes = fixed + a.ring_bytes;
  const int H = a.g.B * a.g.h;
  a.lag = a.n_passes == 2 ? (H < 2 ? H : 2) : 0;
  a.f_u0 = make_fastdiv(static_cast<uint32_t>(a.pass[0].units_per_head));
  if (a.n_passes == 2) {
    a.f_u1 = make_fastdiv(static_cast<uint32_t>(a.pass[1].units_per_head));
    a.f_u01 = make_fastdiv(static_cast<uint32_t>(a.pass[0].units_per_head + a.pass[1].units_per_head));
  }
  return true;
}

cudaError_t launch_short(const ShortArgs& args, int num_sms, cudaStream_t stream) {
  static std::atomic<unsigned long long> set{0};
  const cudaError_t e = max_dyn_smem_once(short_kernel, kSmemLimit, set);
  if (e != cudaSuccess) return e;
  const int H = args.g.B * args.g.h;
  const int n_units = H * (args.pass[0].units_per_head + (args.n_passes == 2 ? args.pass[1].units_per_head : 0));
  const int grid = n_units < num_sms ? n_units : num_sms;
  if (grid < 1) return cudaSuccess;
  short_kernel<<<grid, kThreads, args.smem_bytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace squad
