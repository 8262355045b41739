// host_setup.cu -- per-device host-side setup of the kernels. Kernel attributes
// (cudaFuncSetAttribute) and device properties belong to one device, so every cache here is
// keyed by the calling thread's current device and guarded by one lock: a process may drive
// several GPUs, from several host threads.
#include <map>
#include <mutex>
#include <utility>

#include "kernels.cuh"

namespace moe {

namespace {
std::mutex g_setup_mu;
}

std::mutex& setup_mutex() { return g_setup_mu; }

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

int device_sm_count() {
  static int n[kMaxDevices] = {0};
  const int dev = current_device();
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      (void)cudaGetLastError();
      return 148;
    }
    n[dev] = v;
  }
  return n[dev];
}

cudaError_t ensure_smem_attr(const void* kernel, int bytes) {
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  static std::map<std::pair<const void*, int>, int> done;
  int& have = done[{kernel, dev}];
  if (bytes <= have) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

}  // namespace moe
