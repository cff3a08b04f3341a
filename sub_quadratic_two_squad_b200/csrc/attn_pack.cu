// Tensor-core softmax attention over sequences of at most 64 tokens, several per CTA, sm_100a.
//
// One pass of SQuad (a window or a slot sequence, SQuad paper §3.2; in a k-pass chain, one level) is
// ordinary softmax attention inside each sequence. Short sequences would leave most of a 128-row tile
// idle, so a CTA takes `pack` consecutive sequences (of all B h n_seq), each in its own band of
// `seg` rows (the length rounded up to 8) of the Q, K and V tiles. S = Q K^T is computed once over
// the whole tile; a score counts only where query and key lie in the same band, so P is
// block-diagonal and O = P V gives every sequence its own output.
//
// 160 threads: warps 0-3 own one TMEM lane (one query row) per thread, thread 128 issues the TMA
// loads and the tcgen05 MMAs. Tensor memory: S in columns [0, 128), P packed as bf16 pairs over its
// first half, O in [128, 256); 256 columns and 99 KB of shared memory per CTA, so two CTAs share an
// SM and one's loads and MMAs overlap the other's softmax.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "host_util.h"
#include "ptx.cuh"
#include "geometry.cuh"
#include "pack_pass.h"

namespace squad {

namespace {

constexpr int kThreads = 160;
constexpr uint32_t kPanel = 16384;       // 128 rows x 128 bytes (64 bf16)
constexpr uint32_t kTile = 2 * kPanel;   // one tensor's 128-row tile, both 64-column panels
constexpr uint32_t kOffQ = 0, kOffK = kTile, kOffV = 2 * kTile, kOffBar = 3 * kTile;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr float kLn2 = 0.69314718055994531f;

struct Bars {
  uint64_t load_qk, load_v, s_full, p_full, o_full, drain;
  uint32_t tmem_base;
  uint32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

__device__ __forceinline__ int round16p(int x) { return (x + 15) & ~15; }

__global__ void __launch_bounds__(kThreads, 2) pack_fwd_kernel(const __grid_constant__ PackFwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const sq = base + kOffQ;
  uint8_t* const sk = base + kOffK;
  uint8_t* const sv = base + kOffV;
  Bars* const bars = reinterpret_cast<Bars*>(base + kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Grid& g = a.g;
  const PassGeom& p = a.p;
  const int s = p.seq_len;
  const int seg = a.seg_rows;
  const int total = g.B * g.h * p.n_seq;
  const int first = static_cast<int>(blockIdx.x) * a.pack;
  const int nseq = min(a.pack, total - first);
  const int N = round16p(nseq * seg);   // key rows in use

  if (threadIdx.x == 128) {
    mbar_init(&bars->load_qk, 1);
    mbar_init(&bars->load_v, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  WaitCtl ctl{&bars->abort, a.status, a.timeout_ns};
  if (threadIdx.x == 128) {
    // each sequence's boxes into its band (a multiple of 8 rows: the 128-byte swizzle phase is kept)
    prefetch_tmap(&a.tm_q);
    prefetch_tmap(&a.tm_k);
    prefetch_tmap(&a.tm_v);
    const uint32_t box = static_cast<uint32_t>(s) * 128u;   // one panel of one sequence
    mbar_arrive_expect_tx(&bars->load_qk, static_cast<uint32_t>(nseq) * 4u * box);
    mbar_arrive_expect_tx(&bars->load_v, static_cast<uint32_t>(nseq) * 2u * box);
    for (int j = 0; j < nseq; ++j) {
      const int gs = first + j;
      const int bh = static_cast<int>(fdiv(static_cast<uint32_t>(gs), p.f_per_bh));
      int c[5];
      chunk_coords(g, p, a.variant, bh, gs - bh * p.n_seq, 0, 0, c);
      const uint32_t off = static_cast<uint32_t>(j * seg) * 128u;
      tma_load_5d(sq + off, &a.tm_q, &bars->load_qk, c[0], c[1], c[2], c[3], c[4]);
      tma_load_5d(sq + kPanel + off, &a.tm_q, &bars->load_qk, c[0] + 64, c[1], c[2], c[3], c[4]);
      tma_load_5d(sk + off, &a.tm_k, &bars->load_qk, c[0], c[1], c[2], c[3], c[4]);
      tma_load_5d(sk + kPanel + off, &a.tm_k, &bars->load_qk, c[0] + 64, c[1], c[2], c[3], c[4]);
      tma_load_5d(sv + off, &a.tm_v, &bars->load_v, c[0], c[1], c[2], c[3], c[4]);
      tma_load_5d(sv + kPanel + off, &a.tm_v, &bars->load_v, c[0] + 64, c[1], c[2], c[3], c[4]);
    }
  }
  // Meanwhile, the rows no box writes (the gap after each sequence in its band, the rows past the last
  // band) are zeroed: the MMAs read them.
  for (uint32_t i = threadIdx.x; i < 6u * 128u; i += kThreads) {   // (panel, row) pairs
    const int row = static_cast<int>(i & 127u);
    const int band = row / seg, pos = row - band * seg;
    if (band < nseq && pos < s) continue;
    uint4* dst = reinterpret_cast<uint4*>(base + (i >> 7) * kPanel + static_cast<uint32_t>(row) * 128u);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();   // zeroed rows -> visible to the MMAs (async proxy)
  __syncthreads();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issue
      const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv);
      bool ok = mbar_wait(&bars->load_qk, 0, ctl);
      if (ok) {
        tc_fence_after();
        const uint32_t idesc_s = idesc_bf16(128, N, false);
        for (int kk = 0; kk < 8; ++kk) {   // S = Q K^T -> [0, N)
          const uint32_t off = static_cast<uint32_t>(kk >> 2) * kPanel + static_cast<uint32_t>(kk & 3) * 32u;
          umma_bf16_ss(tmem, sw128_desc(aq + off, 16, 1024), sw128_desc(ak + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&bars->s_full);
        ok = mbar_wait(&bars->p_full, 0, ctl) && mbar_wait(&bars->load_v, 0, ctl);
      }
      if (ok) {
        tc_fence_after();
        const uint32_t idesc_o = idesc_bf16(128, 128, true);   // A = P (TMEM), B = V (MN-major, d wide)
        for (int kk = 0; kk < N / 16; ++kk)   // O = P V -> [128, 256)
          umma_bf16_ts(tmem + 128, tmem + kk * 8, sw128_desc(av + kk * 2048, kPanel, 1024), idesc_o, kk > 0);
        umma_commit(&bars->o_full);
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, 20000000ull);
      // every load issued has landed before the CTA exits (bounded)
      mbar_wait_drain(&bars->load_qk, 0, 20000000ull);
      mbar_wait_drain(&bars->load_v, 0, 20000000ull);
    }
  } else {
    // ------------------------------------------------------------------ row owners
    const int r = warp * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    const int band = r / seg, pos = r - band * seg;
    int tok = -1, bh = 0;
    if (band < nseq && pos < s) {
      const int gs = first + band;
      bh = static_cast<int>(fdiv(static_cast<uint32_t>(gs), p.f_per_bh));
      tok = token_of(g, p, gs - bh * p.n_seq, 0, pos);
    }
    const int k0 = band * seg;   // the row's own keys: columns [k0, k0 + s)
    const size_t gi = static_cast<size_t>(bh) * g.n + (tok < 0 ? 0 : tok);
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full, 0, ctl));
    float m2 = 0.f, l = 0.f;   // row maximum (log2 units) and row sum
    if (ok) {
      tc_fence_after();
      // the whole row of scores (at most 128 columns) in registers; the maximum over the row's band
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t t[32];
        if (32 * c < N) tmem_ld32(t_row + 32 * c, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) sr[32 * c + i] = 32 * c < N ? t[i] : __float_as_uint(-INFINITY);
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        const bool own = tok >= 0 && i >= k0 && i < k0 + s;
        if (!own) sr[i] = __float_as_uint(-INFINITY);
        mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(sr[i]));
      }
      // the scale is positive, so it is applied to the maximum instead of to every score; rows of no
      // sequence keep m2 = 0 and P = 0
      m2 = tok >= 0 ? fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2 : 0.f;
      // P = 2^(x - m2) (0 outside the band), bf16 pairs over the first columns of S (all read)
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (32 * c >= N) break;
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float x0 = ex2_approx(fmaf(__uint_as_float(sr[32 * c + 2 * j]), sl2, -m2));
          const float x1 = ex2_approx(fmaf(__uint_as_float(sr[32 * c + 2 * j + 1]), sl2, -m2));
          ls[(2 * j) & 3] += x0;
          ls[(2 * j + 1) & 3] += x1;
          pk[j] = pack_bf16x2(x0, x1);
        }
        tmem_st16_nowait(t_row + 16 * c, pk);
      }
      l = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->o_full, 0, ctl));
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = tok >= 0 ? 1.f / l : 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[64];
        tmem_ld64(t_row + 128 + 64 * h, o);
        if (tok >= 0) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + gi * 128 + 64 * h);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * i]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l));
        }
      }
      if (tok >= 0 && a.lse != nullptr) a.lse[gi] = (m2 + __log2f(l)) * kLn2;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) {
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool pack_eligible(const Grid& g, const PassGeom& p) {
  return g.d == 128 && p.kind != kFull && p.n_chunks == 1 && p.seq_len >= 1 && p.seq_len <= 64;
}

void pack_plan(PackFwdArgs& a) {
  a.seg_rows = (a.p.seq_len + 7) & ~7;
  a.pack = 128 / a.seg_rows;
}

cudaError_t launch_pack_fwd(const PackFwdArgs& a, cudaStream_t stream) {
  static std::atomic<unsigned long long> set{0};
  const cudaError_t e = max_dyn_smem_once(pack_fwd_kernel, kSmemBytes, set);
  if (e != cudaSuccess) return e;
  const int seqs = a.g.B * a.g.h * a.p.n_seq;
  if (seqs == 0) return cudaSuccess;
  pack_fwd_kernel<<<static_cast<unsigned>((seqs + a.pack - 1) / a.pack), kThreads, kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace squad
