// squad_attn_fwd_noalloc: the SQuad forward with its scratch in a fixed device array, for callers that
// cannot allocate device memory (see include/squad_attn.h).
#include <cstddef>

#include <cuda_runtime.h>

#include "squad_attn.h"

namespace {

// Scratch for one forward call: the control block, the pass-1 output and both LSE buffers. Every GPU
// that loads this library reserves it until the process exits.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(SQUAD_NOALLOC_MAX_WORKSPACE_BYTES);
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device. In host code the symbol itself is only a
// host-side stand-in, so the address is looked up with the device current. The lookup is a host-side
// query with no stream work and is repeated on every call, so a context that was torn down and created
// again (cudaDeviceReset) never sees a stale address.
void* scratch_on_current_device() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
  return ptr;
}

// True when `p` is device memory of the current device (the kernels run there, with its scratch).
bool on_current_device(const void* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();   // an unknown pointer's error is not sticky: clear it for later callers
    return false;
  }
  return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
}

}  // namespace

extern "C" squad_status_t squad_attn_fwd_noalloc(const squad_params_t* p, const void* q, const void* k,
                                                 const void* v, void* o, squad_stream_t stream) {
  const size_t need = squad_attn_fwd_workspace_bytes(p);
  if (need == 0) return SQUAD_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return SQUAD_ERR_UNSUPPORTED;
  // Every tensor must live on the current device: the scratch used below is that device's copy.
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (!on_current_device(q) || !on_current_device(k) || !on_current_device(v) || !on_current_device(o))
    return SQUAD_ERR_INVALID_ARG;
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return SQUAD_ERR_CUDA;
  // The forward zeroes the control block at the start of every call; the rest of the scratch is
  // written before it is read.
  return squad_attn_fwd(p, q, k, v, o, scratch, stream);
}
