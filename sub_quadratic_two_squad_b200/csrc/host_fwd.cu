// squad_attn_fwd_host: the SQuad forward from pinned host buffers, with the host<->device copies of one
// group of heads overlapping the forward of another (include/squad_attn.h). Every (batch, head) pair
// is independent in both passes, so a group of consecutive pairs of the [B, h, n, d] layout is a
// forward of its own (B = 1, h = the group's size) on contiguous slices of the tensors.
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "squad_attn.h"

namespace {

constexpr int kMaxGroups = 64;
constexpr int kMaxDevices = 64;

// Events linking the three streams: for each group, "inputs copied" and "forward done", plus the two
// joins at the start of a call. Created once per device on first use (cudaEventDisableTiming) and kept
// until the process exits; calls on one device are serialised by the pool's mutex while they enqueue.
struct EventPool {
  std::mutex mu;
  std::vector<cudaEvent_t> ev;   // 2 * kMaxGroups + 2 events, empty until created
};
EventPool g_pools[kMaxDevices];

bool ensure_events(EventPool& pool) {
  if (!pool.ev.empty()) return true;
  std::vector<cudaEvent_t> ev(2 * kMaxGroups + 2, nullptr);
  for (auto& e : ev) {
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (auto& x : ev)
        if (x != nullptr) cudaEventDestroy(x);
      return false;
    }
  }
  pool.ev.swap(ev);
  return true;
}

size_t tensor_bytes(const squad_params_t* p) {
  const size_t eb = p->dtype == SQUAD_BF16 ? 2u : 4u;
  return static_cast<size_t>(p->B) * p->h * p->T * p->H * p->W * p->d * eb;
}

// The problem of heads [h0, h1) of the flattened B*h: one batch of h1 - h0 heads.
squad_params_t group_params(const squad_params_t* p, int h0, int h1) {
  squad_params_t s = *p;
  s.B = 1;
  s.h = h1 - h0;
  return s;
}

bool aligned16(const void* x) { return x != nullptr && reinterpret_cast<uintptr_t>(x) % 16u == 0u; }

}  // namespace

extern "C" size_t squad_attn_fwd_host_workspace_bytes(const squad_params_t* p, int groups) {
  if (p == nullptr || groups < 1 || groups > kMaxGroups) return 0;
  if (squad_attn_fwd_workspace_bytes(p) == 0) return 0;   // validates p
  const int bh = p->B * p->h;
  if (groups > bh) return 0;
  const int widest = (bh + groups - 1) / groups;
  const squad_params_t s = group_params(p, 0, widest);
  return squad_attn_fwd_workspace_bytes(&s);
}

extern "C" squad_status_t squad_attn_fwd_host(const squad_params_t* p, const void* q_host, const void* k_host,
                                              const void* v_host, void* o_host, void* q_dev, void* k_dev,
                                              void* v_dev, void* o_dev, void* workspace, int groups,
                                              squad_stream_t copy_in_, squad_stream_t compute_,
                                              squad_stream_t copy_out_) {
  if (squad_attn_fwd_host_workspace_bytes(p, groups) == 0) return SQUAD_ERR_INVALID_ARG;
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(o_dev)) return SQUAD_ERR_INVALID_ARG;
  if (workspace == nullptr || reinterpret_cast<uintptr_t>(workspace) % 256u != 0u) return SQUAD_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SQUAD_ERR_CUDA;
  cudaStream_t s_in = reinterpret_cast<cudaStream_t>(copy_in_);
  cudaStream_t s_comp = reinterpret_cast<cudaStream_t>(compute_);
  cudaStream_t s_out = reinterpret_cast<cudaStream_t>(copy_out_);

  EventPool& pool = g_pools[dev];
  std::lock_guard<std::mutex> lock(pool.mu);
  if (!ensure_events(pool)) return SQUAD_ERR_CUDA;
  cudaEvent_t* in_done = pool.ev.data();
  cudaEvent_t* comp_done = pool.ev.data() + kMaxGroups;
  cudaEvent_t join_comp = pool.ev[2 * kMaxGroups], join_out = pool.ev[2 * kMaxGroups + 1];

  // Work already queued on the compute stream may still read q_dev, k_dev, v_dev (an earlier call), and
  // work on the copy-out stream may still read o_dev: this call's copies and forwards start after both.
  if (cudaEventRecord(join_comp, s_comp) != cudaSuccess || cudaStreamWaitEvent(s_in, join_comp, 0) != cudaSuccess)
    return SQUAD_ERR_CUDA;
  if (cudaEventRecord(join_out, s_out) != cudaSuccess || cudaStreamWaitEvent(s_comp, join_out, 0) != cudaSuccess)
    return SQUAD_ERR_CUDA;

  const int bh = p->B * p->h;
  const size_t head_bytes = tensor_bytes(p) / static_cast<size_t>(bh);
  for (int gi = 0; gi < groups; ++gi) {
    const int h0 = static_cast<int>(static_cast<long long>(bh) * gi / groups);
    const int h1 = static_cast<int>(static_cast<long long>(bh) * (gi + 1) / groups);
    const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(h1 - h0) * head_bytes;
    auto dptr = [&](void* base) { return static_cast<uint8_t*>(base) + off; };
    auto hptr = [&](const void* base) { return static_cast<const uint8_t*>(base) + off; };
    // inputs of this group: one copy per tensor
    if (cudaMemcpyAsync(dptr(q_dev), hptr(q_host), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(dptr(k_dev), hptr(k_host), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(dptr(v_dev), hptr(v_host), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(in_done[gi], s_in) != cudaSuccess)
      return SQUAD_ERR_CUDA;
    // its forward, once its inputs are on the device (the workspace is reused group after group)
    if (cudaStreamWaitEvent(s_comp, in_done[gi], 0) != cudaSuccess) return SQUAD_ERR_CUDA;
    const squad_params_t sp = group_params(p, h0, h1);
    const squad_status_t st =
        squad_attn_fwd(&sp, dptr(q_dev), dptr(k_dev), dptr(v_dev), dptr(o_dev), workspace, compute_);
    if (st != SQUAD_OK) return st;
    if (cudaEventRecord(comp_done[gi], s_comp) != cudaSuccess) return SQUAD_ERR_CUDA;
    // its output back to the host
    if (cudaStreamWaitEvent(s_out, comp_done[gi], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + off, dptr(o_dev), bytes, cudaMemcpyDeviceToHost, s_out) !=
            cudaSuccess)
      return SQUAD_ERR_CUDA;
  }
  return SQUAD_OK;
}
