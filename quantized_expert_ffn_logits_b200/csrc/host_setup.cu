// host_setup.cu -- per-device host-side setup of the kernels. Kernel attributes
// (cudaFuncSetAttribute) and device properties belong to one device, so every cache here is
// keyed by the calling thread's current device and guarded by one lock: a process may drive
// several GPUs, from several host threads.
#include <map>
#include <mutex>
#include <tuple>
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

int max_active_clusters(const void* kernel, int dev, int cluster, int smem, int threads) {
  if (ensure_smem_attr(kernel, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lk(g_setup_mu);
  static std::map<std::tuple<const void*, int, int, int>, int> done;
  const auto key = std::make_tuple(kernel, dev, cluster, smem);
  const auto it = done.find(key);
  if (it != done.end()) return it->second;
  if (cluster > 8) (void)cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaLaunchConfig_t q = {};
  cudaLaunchAttribute qa[1];
  qa[0].id = cudaLaunchAttributeClusterDimension;
  qa[0].val.clusterDim.x = cluster;
  qa[0].val.clusterDim.y = 1;
  qa[0].val.clusterDim.z = 1;
  q.gridDim = dim3(cluster * 8);
  q.blockDim = dim3(threads);
  q.dynamicSmemBytes = (size_t)smem;
  q.attrs = qa;
  q.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &q) != cudaSuccess) n = 0;
  (void)cudaGetLastError();
  done[key] = n;
  return n;
}

}  // namespace moe
