// squad_attn_fwd_noalloc: the SQuad forward with its scratch in a fixed device array, for callers that
// cannot allocate device memory (see include/squad_attn.h).
#include <cstddef>
#include <mutex>

#include <cuda_runtime.h>

#include "squad_attn.h"

namespace {

// Scratch for one forward call: the control block, the pass-1 output and both LSE buffers. Every GPU
// that loads this library reserves it until the process exits.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(SQUAD_NOALLOC_MAX_WORKSPACE_BYTES);
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device. In host code the symbol itself is only a
// host-side stand-in, so the address is looked up once per device, with that device current.
void* scratch_on_current_device() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = ptr;
  }
  return addr[dev];
}

}  // namespace

extern "C" squad_status_t squad_attn_fwd_noalloc(const squad_params_t* p, const void* q, const void* k,
                                                 const void* v, void* o, squad_stream_t stream) {
  const size_t need = squad_attn_fwd_workspace_bytes(p);
  if (need == 0) return SQUAD_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return SQUAD_ERR_UNSUPPORTED;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return SQUAD_ERR_CUDA;
  // The forward zeroes the control block at the start of every call; the rest of the scratch is
  // written before it is read.
  return squad_attn_fwd(p, q, k, v, o, scratch, stream);
}
