// Work units of the persistent short-sequence attention kernels (attn_short.cu, attn_pipe.cu): the
// global unit order of one pass or of both SQuad passes fused (a head's second-pass units trailing its
// first-pass units by `lag` heads), the split of a unit into one or two query tiles, and the byte-ring
// allocation cursor that every warp of a CTA replays identically.
#pragma once

#include <cstdint>

#include "geometry.cuh"
#include "short_pass.h"

namespace squad {
namespace units {

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One work unit: its pass, head, sequences and ring allocations.
struct Unit {
  int pass, bh, nw;
  bool shared;       // both query tiles belong to one sequence (shared K and V)
  int sigma[2];
  uint32_t q[2], k[2], v[2];        // allocation indices
  uint32_t qo[2], ko[2], vo[2];     // their byte offsets in the ring
  uint32_t qvs[2], kvs[2], vvs[2];  // their virtual starts (producer bookkeeping)
};

// Allocation cursor over the byte ring, identical in every warp.
struct Cursor {
  uint32_t ai = 0, vpos = 0, phys = 0;
  __device__ __forceinline__ void take(uint32_t sz, uint32_t ring, uint32_t& idx, uint32_t& off, uint32_t& vstart) {
    if (phys + sz > ring) {
      vpos += ring - phys;
      phys = 0;
    }
    idx = ai++;
    off = phys;
    vstart = vpos;
    phys += sz;
    vpos += sz;
  }
};

// Global unit index -> (pass, head, unit within head).
__device__ __forceinline__ void decode_unit(const ShortArgs& a, int U, int& pass, int& bh, int& j) {
  const int H = a.g.B * a.g.h;
  const int n0 = a.pass[0].units_per_head;
  if (a.n_passes == 1) {
    bh = static_cast<int>(fdiv(static_cast<uint32_t>(U), a.f_u0));
    pass = 0;
    j = U - bh * n0;
    return;
  }
  const int n1 = a.pass[1].units_per_head;
  const int lag = a.lag;
  const int lead = lag * n0;                 // blocks 0..lag-1: first-pass units only
  const int mid = lead + (H - lag) * (n0 + n1);
  if (U < lead) {
    bh = static_cast<int>(fdiv(static_cast<uint32_t>(U), a.f_u0));
    pass = 0;
    j = U - bh * n0;
  } else if (U < mid) {
    const int r = U - lead;
    const int k = static_cast<int>(fdiv(static_cast<uint32_t>(r), a.f_u01));
    const int o = r - k * (n0 + n1);
    if (o < n0) {
      pass = 0;
      bh = lag + k;
      j = o;
    } else {
      pass = 1;
      bh = k;
      j = o - n0;
    }
  } else {
    const int r = U - mid;
    const int k = static_cast<int>(fdiv(static_cast<uint32_t>(r), a.f_u1));
    pass = 1;
    bh = H - lag + k;
    j = r - k * n1;
  }
}

__device__ __forceinline__ Unit plan_unit(const ShortArgs& a, int U, Cursor& cur, uint32_t ring) {
  Unit u;
  int j;
  decode_unit(a, U, u.pass, u.bh, j);
  const int seq_len = u.pass ? a.pass[1].p.seq_len : a.pass[0].p.seq_len;
  const int n_seq = u.pass ? a.pass[1].p.n_seq : a.pass[0].p.n_seq;
  const uint32_t sz = u.pass ? a.pass[1].alloc_bytes : a.pass[0].alloc_bytes;
  u.shared = seq_len > 128;
  if (u.shared) {
    u.nw = 2;
    u.sigma[0] = u.sigma[1] = j;
    cur.take(sz, ring, u.q[0], u.qo[0], u.qvs[0]);
    cur.take(sz, ring, u.k[0], u.ko[0], u.kvs[0]);
    cur.take(sz, ring, u.v[0], u.vo[0], u.vvs[0]);
    u.q[1] = u.q[0]; u.qo[1] = u.qo[0]; u.qvs[1] = u.qvs[0];
    u.k[1] = u.k[0]; u.ko[1] = u.ko[0]; u.kvs[1] = u.kvs[0];
    u.v[1] = u.v[0]; u.vo[1] = u.vo[0]; u.vvs[1] = u.vvs[0];
  } else {
    u.sigma[0] = 2 * j;
    u.sigma[1] = 2 * j + 1;
    u.nw = u.sigma[1] < n_seq ? 2 : 1;
    cur.take(sz, ring, u.q[0], u.qo[0], u.qvs[0]);
    cur.take(sz, ring, u.k[0], u.ko[0], u.kvs[0]);
    if (u.nw == 2) {
      cur.take(sz, ring, u.q[1], u.qo[1], u.qvs[1]);
      cur.take(sz, ring, u.k[1], u.ko[1], u.kvs[1]);
    }
    cur.take(sz, ring, u.v[0], u.vo[0], u.vvs[0]);
    if (u.nw == 2) cur.take(sz, ring, u.v[1], u.vo[1], u.vvs[1]);
    if (u.nw == 1) {
      u.sigma[1] = u.sigma[0];
      u.q[1] = u.q[0]; u.qo[1] = u.qo[0]; u.qvs[1] = u.qvs[0];
      u.k[1] = u.k[0]; u.ko[1] = u.ko[0]; u.kvs[1] = u.kvs[0];
      u.v[1] = u.v[0]; u.vo[1] = u.vo[0]; u.vvs[1] = u.vvs[0];
    }
  }
  return u;
}

// The fields of one pass, selected with static offsets into the kernel parameters (indexing the
// parameter array with a run-time pass number would go through local memory).
struct PassView {
  const CUtensorMap *q, *k, *v, *o;
  PassGeom p;
  int variant;
  float* lse;
  uint32_t panel, alloc;
};

__device__ __forceinline__ PassView view_of(const ShortArgs& a, int pass) {
  PassView v;
  if (pass == 0) {
    v.q = &a.pass[0].tm_q; v.k = &a.pass[0].tm_k; v.v = &a.pass[0].tm_v; v.o = &a.pass[0].tm_o;
    v.p = a.pass[0].p; v.variant = a.pass[0].variant; v.lse = a.pass[0].lse;
    v.panel = a.pass[0].panel_bytes; v.alloc = a.pass[0].alloc_bytes;
  } else {
    v.q = &a.pass[1].tm_q; v.k = &a.pass[1].tm_k; v.v = &a.pass[1].tm_v; v.o = &a.pass[1].tm_o;
    v.p = a.pass[1].p; v.variant = a.pass[1].variant; v.lse = a.pass[1].lse;
    v.panel = a.pass[1].panel_bytes; v.alloc = a.pass[1].alloc_bytes;
  }
  return v;
}

__device__ __forceinline__ int total_units(const ShortArgs& a) {
  const int H = a.g.B * a.g.h;
  return H * (a.pass[0].units_per_head + (a.n_passes == 2 ? a.pass[1].units_per_head : 0));
}

}  // namespace units
}  // namespace squad
