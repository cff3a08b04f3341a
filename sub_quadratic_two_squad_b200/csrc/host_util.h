// Host-side launch helpers shared by the kernel launchers.
#pragma once

#include <atomic>

#include <cuda_runtime.h>

namespace squad {

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device. The attribute is
// per device, so it is set once for every device a process launches on; `done` is the launcher's
// bit mask of devices already set (devices 64 and up are set on every call). Setting it twice from
// racing threads is harmless.
template <typename Kernel>
cudaError_t max_dyn_smem_once(Kernel kernel, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Number of SMs of the current device (0 if it cannot be read), looked up once per device.
inline int num_sms_current() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::atomic<int> cache[64];   // per device; 0 = not looked up yet (calls may come from many threads)
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

}  // namespace squad
