// Tensor-core attention over sequences of at most 256 tokens, sm_100a: one SQuad pass (local windows
// or global slots, paper §3.2) per launch, every sequence handled in one block.
//
// Each of Q, K, V of a sequence arrives as one TMA box (the whole window, or the whole slot across
// all windows) in a slot of a shared-memory ring; S = Q K^T is one tcgen05.mma per 16-deep K step
// with N = the sequence length rounded up to 16 (<= 256), so the softmax needs no running maximum.
//
// CTA organisation (persistent, one CTA per SM, 352 threads):
//   warps 0-3   softmax warpgroup 0 (TMEM lanes 0-127 of its S / O)
//   warps 4-7   softmax warpgroup 1
//   warp 8      TMA producer       warp 9  TMEM allocator and MMA issuer     warp 10  TMA store issuer
// A work unit is either one sequence of 129-256 tokens (its two 128-row query tiles go to the two
// warpgroups and share K and V) or two sequences of at most 128 tokens (one per warpgroup).
// Per unit the producer fills ring slots in the order Q, K (per tile) then V (per tile); Q and K slots
// are released as soon as the S products that read them complete, the V slot when the output stored
// through it has left: the softmax warps stage O (normalised, bf16) in the V slot after PV has read
// it, and the store warp writes it back with a TMA store of the same box. So the next unit's loads
// overlap this unit's softmax and epilogue.
// Tensor memory per warpgroup (256 columns): S in [0, N), P (bf16 pairs) over [0, N/2), and O in
// [128, 256) when N <= 128, else in [N/2, N/2 + 128) over the consumed scores; in the second case the
// next unit's S waits until the epilogue has read O.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "geometry.cuh"
#include "short_pass.h"

namespace squad {

namespace {

constexpr int kThreads = 352;
constexpr int kWarpProducer = 8, kWarpMma = 9, kWarpStore = 10;
constexpr int kMaxSlots = 8;
constexpr uint32_t kSmemLimit = 232448;

struct Bars {
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2], staged[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
};
constexpr uint32_t kBarBytes = 256;
static_assert(sizeof(Bars) <= kBarBytes, "barrier block");

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// The sequences and ring allocations of one work unit. Allocation indices count every slot fill of
// the launch in order; slot = index % n_slots.
struct Unit {
  int nw;            // query tiles in the unit (1 or 2)
  bool shared;       // both tiles belong to one sequence (shared K and V)
  int bh[2], sigma[2];
  uint32_t q[2], k[2], v[2];
  uint32_t n_alloc;  // allocations this unit makes
};

__device__ __forceinline__ Unit plan_unit(const Grid& g, const PassGeom& p, int unit, uint32_t base) {
  Unit u;
  const int total = g.B * g.h * p.n_seq;
  const bool two_tiles = p.seq_len > 128;
  int seq[2];
  if (two_tiles) {
    u.nw = 2;
    u.shared = true;
    seq[0] = seq[1] = unit;
    u.q[0] = u.q[1] = base;
    u.k[0] = u.k[1] = base + 1;
    u.v[0] = u.v[1] = base + 2;
    u.n_alloc = 3;
  } else {
    u.shared = false;
    seq[0] = 2 * unit;
    seq[1] = 2 * unit + 1;
    u.nw = seq[1] < total ? 2 : 1;
    u.q[0] = base;
    u.k[0] = base + 1;
    if (u.nw == 2) {
      u.q[1] = base + 2;
      u.k[1] = base + 3;
      u.v[0] = base + 4;
      u.v[1] = base + 5;
      u.n_alloc = 6;
    } else {
      u.q[1] = u.k[1] = u.v[1] = 0;
      u.v[0] = base + 2;
      u.n_alloc = 3;
    }
  }
  for (int w = 0; w < 2; ++w) {
    const int sq = seq[w] < total ? seq[w] : seq[0];
    u.bh[w] = static_cast<int>(fdiv(static_cast<uint32_t>(sq), p.f_per_bh));
    u.sigma[w] = sq - u.bh[w] * p.n_seq;
  }
  return u;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) short_pass_kernel(const __grid_constant__ ShortPassArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring_bytes = static_cast<uint32_t>(a.n_slots) * a.slot_bytes;
  Bars* bars = reinterpret_cast<Bars*>(ring + ring_bytes + a.guard_bytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PassGeom& p = a.p;
  const Grid& g = a.g;
  const int NS = a.n_slots;
  const int s_len = p.seq_len;
  const int N = round16(s_len);
  const bool o_overlap = N > 128;
  const uint32_t o_off = o_overlap ? static_cast<uint32_t>(N / 2) : 128u;

  // Zero the ring and guard once: rows past a sequence inside a slot (and past the ring) are read by
  // the MMAs and must hold finite values.
  for (uint32_t i = threadIdx.x; i < (ring_bytes + a.guard_bytes) / 16; i += kThreads)
    reinterpret_cast<uint4*>(ring)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxSlots; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
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
  const int total_seq = g.B * g.h * p.n_seq;
  const int n_units = s_len > 128 ? total_seq : (total_seq + 1) / 2;
  const uint32_t box_bytes = 2u * static_cast<uint32_t>(s_len) * 128u;
  auto slot_ptr = [&](uint32_t alloc) { return ring + (alloc % static_cast<uint32_t>(NS)) * a.slot_bytes; };

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t base = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* m, int bh, int sigma, uint32_t alloc) -> bool {
        const uint32_t sl = alloc % static_cast<uint32_t>(NS);
        if (alloc >= static_cast<uint32_t>(NS) &&
            !mbar_wait(&bars->empty[sl], ((alloc / NS) + 1) & 1, ctl))
          return false;
        mbar_arrive_expect_tx(&bars->full[sl], box_bytes);
        int c[5];
        chunk_coords(g, p, a.global_variant, bh, sigma, 0, 0, c);
        uint8_t* dst = slot_ptr(alloc);
        tma_load_5d(dst, m, &bars->full[sl], c[0], c[1], c[2], c[3], c[4]);
        tma_load_5d(dst + a.panel_bytes, m, &bars->full[sl], c[0] + 64, c[1], c[2], c[3], c[4]);
        return true;
      };
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        const Unit u = plan_unit(g, p, unit, base);
        const int nsrc = u.shared ? 1 : u.nw;
        for (int w = 0; w < nsrc && ok; ++w) {
          ok = load(&a.tm_q, u.bh[w], u.sigma[w], u.q[w]);
          if (ok) ok = load(&a.tm_k, u.bh[w], u.sigma[w], u.k[w]);
        }
        for (int w = 0; w < nsrc && ok; ++w) ok = load(&a.tm_v, u.bh[w], u.sigma[w], u.v[w]);
        base += u.n_alloc;
      }
      // Let every load this thread issued land before the CTA can exit (bounded).
      const uint32_t first = base > static_cast<uint32_t>(NS) ? base - NS : 0;
      for (uint32_t i = first; i < base; ++i)
        mbar_wait_drain(&bars->full[i % NS], (i / NS) & 1, 20000000ull);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(128, N, false);
      const uint32_t idesc_pv = idesc_bf16(128, 128, true);
      uint32_t base = 0, p_cnt[2] = {0, 0}, of_cnt[2] = {0, 0};
      bool ok = true;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        const Unit u = plan_unit(g, p, unit, base);
        for (int w = 0; w < u.nw && ok; ++w) {
          const bool first_user = w == 0 || !u.shared;
          if (first_user) {
            ok = mbar_wait(&bars->full[u.q[w] % NS], (u.q[w] / NS) & 1, ctl);
            if (ok) ok = mbar_wait(&bars->full[u.k[w] % NS], (u.k[w] / NS) & 1, ctl);
          }
          if (ok && o_overlap && unit != static_cast<int>(blockIdx.x)) {
            // the previous unit's epilogue must have read O, which overlaps this S
            ok = mbar_wait(&bars->o_free[w], of_cnt[w] & 1, ctl);
            ++of_cnt[w];
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(slot_ptr(u.q[w])) + (u.shared ? static_cast<uint32_t>(w) * 16384u : 0u);
          const uint32_t ka = smem_u32(slot_ptr(u.k[w]));
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * a.panel_bytes + (kk & 3) * 32;
            umma_bf16_ss(tmem + 256 * w, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), idesc_s,
                         kk > 0);
          }
          umma_commit(&bars->s_full[w]);
          if (!u.shared || w == u.nw - 1) {
            umma_commit(&bars->empty[u.q[w] % NS]);
            umma_commit(&bars->empty[u.k[w] % NS]);
          }
        }
        for (int w = 0; w < u.nw && ok; ++w) {
          ok = mbar_wait(&bars->p_full[w], p_cnt[w] & 1, ctl);
          ++p_cnt[w];
          if (ok && (w == 0 || !u.shared)) ok = mbar_wait(&bars->full[u.v[w] % NS], (u.v[w] / NS) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t va = smem_u32(slot_ptr(u.v[w]));
          for (int kk = 0; kk < N / 16; ++kk)
            umma_bf16_ts(tmem + 256 * w + o_off, tmem + 256 * w + kk * 8, sw128_desc(va + kk * 2048, a.panel_bytes, 1024),
                         idesc_pv, kk > 0);
          if (!u.shared) umma_commit(&bars->o_full[w]);
        }
        if (ok && u.shared) {   // both tiles read the one V slot: neither may overwrite it before both PVs end
          umma_commit(&bars->o_full[0]);
          umma_commit(&bars->o_full[1]);
        }
        base += u.n_alloc;
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
    }
  } else if (warp == kWarpStore) {
    // ------------------------------------------------------------------ TMA store issuer
    if (lane == 0) {
      uint32_t base = 0, st_cnt[2] = {0, 0};
      bool ok = true;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        const Unit u = plan_unit(g, p, unit, base);
        const int nseq = u.shared ? 1 : u.nw;
        for (int w = 0; w < u.nw && ok; ++w) {
          ok = mbar_wait(&bars->staged[w], st_cnt[w] & 1, ctl);
          ++st_cnt[w];
        }
        for (int w = 0; w < nseq && ok; ++w) {
          int c[5];
          chunk_coords(g, p, a.global_variant, u.bh[w], u.sigma[w], 0, 0, c);
          const uint8_t* src = slot_ptr(u.v[w]);
          tma_store_5d(&a.tm_o, src, c[0], c[1], c[2], c[3], c[4]);
          tma_store_5d(&a.tm_o, src + a.panel_bytes, c[0] + 64, c[1], c[2], c[3], c[4]);
          bulk_commit_group();
        }
        bulk_wait_read_all();   // the V slots may be refilled once their stores have read them
        for (int w = 0; w < nseq; ++w) mbar_arrive(&bars->empty[u.v[w] % NS]);
        base += u.n_alloc;
      }
      bulk_wait_all();   // outputs written before the CTA exits
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_s = tmem + 256 * wg + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t t_o = t_s + o_off;
    const float sl2 = a.scale_log2;
    const int nchunk = (N + 63) / 64;
    uint32_t s_cnt = 0, o_cnt = 0, base = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
      const Unit u = plan_unit(g, p, unit, base);
      base += u.n_alloc;
      if (wg >= u.nw) break;
      const int row0 = u.shared ? 128 * wg : 0;           // first sequence row of this tile
      const int src = u.shared ? 0 : wg;
      int valid = s_len - row0;
      if (valid > 128) valid = 128;
      const bool active = wq * 32 < valid;                 // warps of padding rows only keep the barriers
      ok = mbar_wait(&bars->s_full[wg], s_cnt & 1, ctl);
      ++s_cnt;
      if (!ok) break;
      tc_fence_after();
      float m = -INFINITY, l = 0.f;
      if (active) {
        uint32_t r[64];
        // pass 1: row maximum of the scores (the scale is positive: applied to the maximum)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int c = 0; c < nchunk; ++c) {
          tmem_ld64(t_s + 64 * c, r);
          if (64 * c + 64 <= s_len) {
#pragma unroll
            for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (64 * c + i < s_len) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
          }
        }
        m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
        // pass 2: P = 2^(x - m), rounded to bf16 on the integer pipe (add half an ulp, keep the high
        // half), packed two per 32-bit word over the first half of the scores; masked columns give 0.
        const float nm = -m;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int c = 0; c < nchunk; ++c) {
          tmem_ld64(t_s + 64 * c, r);
          if (64 * c + 64 > s_len) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (64 * c + i >= s_len) r[i] = __float_as_uint(-INFINITY);
          }
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x0 = ex2_approx(fmaf(__uint_as_float(r[2 * j]), sl2, nm));
            const float x1 = ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), sl2, nm));
            ls[(2 * j) & 3] += x0;
            ls[(2 * j + 1) & 3] += x1;
            pk[j] = __byte_perm(__float_as_uint(x0) + 0x8000u, __float_as_uint(x1) + 0x8000u, 0x7632);
          }
          tmem_st32(t_s + 32 * c, pk);
        }
        l = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      }
      tc_fence_before();
      mbar_arrive(&bars->p_full[wg]);

      // epilogue: O / l -> bf16 into this tile's rows of the V slot (PV has finished reading it); the
      // store warp writes the slot back with the sequence's box.
      ok = mbar_wait(&bars->o_full[wg], o_cnt & 1, ctl);
      ++o_cnt;
      if (!ok) break;
      tc_fence_after();
      const int vrow = row0 + row;   // row within the V slot's panels
      const uint32_t row_addr = smem_u32(slot_ptr(u.v[src])) + static_cast<uint32_t>(vrow) * 128u;
      const bool store_row = row < valid;
      const float inv_l = active ? 1.f / l : 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[64];
        if (active) tmem_ld64(t_o + 64 * h, o);
        if (h == 1) {
          // O has been read into registers: the next unit's S may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->o_free[wg]);
        }
        if (store_row) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row_addr + h * a.panel_bytes + ((c ^ (vrow & 7)) << 4),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 0]) * inv_l, __uint_as_float(o[c * 8 + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 2]) * inv_l, __uint_as_float(o[c * 8 + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 4]) * inv_l, __uint_as_float(o[c * 8 + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[c * 8 + 6]) * inv_l, __uint_as_float(o[c * 8 + 7]) * inv_l));
        }
      }
      if (a.lse != nullptr && store_row) {
        const int tok = token_of(g, p, u.sigma[src], 0, vrow);
        if (tok >= 0) a.lse[static_cast<size_t>(u.bh[src]) * g.n + tok] = (m + __log2f(l)) * 0.69314718055994531f;
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

bool short_pass_plan(ShortPassArgs& a) {
  const int s = a.p.seq_len;
  if (s < 1 || s > 256 || a.p.n_chunks != 1 || a.g.d != 128) return false;
  const uint32_t rows8 = static_cast<uint32_t>((s + 7) & ~7);
  a.panel_bytes = rows8 * 128u;
  a.slot_bytes = 2u * a.panel_bytes;
  // Past a slot's end the MMAs read at most: the second 128-row query tile of a 256-row tile pair
  // (or the only 128-row tile), and the K/V rows up to the sequence length rounded to 16.
  const uint32_t tile_span = s > 128 ? 32768u : 16384u;
  uint32_t guard = tile_span > a.panel_bytes ? tile_span - a.panel_bytes : 0u;
  if (guard < 2048u) guard = 2048u;
  a.guard_bytes = (guard + 1023u) & ~1023u;
  const uint32_t fixed = 1024u + a.guard_bytes + kBarBytes;
  int n = static_cast<int>((kSmemLimit - fixed) / a.slot_bytes);
  if (n > kMaxSlots) n = kMaxSlots;
  const int need = s > 128 ? 3 : 6;   // slots one unit holds at once
  if (n < need) return false;
  a.n_slots = n;
  a.smem_bytes = fixed + static_cast<uint32_t>(n) * a.slot_bytes;
  return true;
}

cudaError_t launch_short_pass(const ShortPassArgs& args, int num_sms, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(short_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int total_seq = args.g.B * args.g.h * args.p.n_seq;
  const int n_units = args.p.seq_len > 128 ? total_seq : (total_seq + 1) / 2;
  const int grid = n_units < num_sms ? n_units : num_sms;
  if (grid < 1) return cudaSuccess;
  short_pass_kernel<<<grid, kThreads, args.smem_bytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace squad
