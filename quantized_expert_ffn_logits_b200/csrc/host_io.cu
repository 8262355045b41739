// host_io.cu -- the layer's input and output moved between page-locked host memory and the
// device by the SMs, through the buffers' device-mapped addresses, as two small kernels on
// the layer's stream. Both are chained by programmatic dependent launch, so unlike
// copy-engine copies they keep the launches of consecutive calls overlapped.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

namespace {

constexpr int kIoThreads = 256;

// x_host -> x_dev, then the wait for the preceding kernel. Writing x_dev before that wait is
// safe: the preceding kernel is the previous call's output copy, which reads no x and was
// itself launched only when the previous layer's last kernel let it -- which every kernel of
// the layer does only after waiting for its predecessor (the single-token kernel after its grid
// barrier), so every kernel that read x_dev in the previous call had finished or was past its
// reads of x. The PCIe round trip and the copy then overlap the previous call's tail.
__global__ void __launch_bounds__(kIoThreads) k_copy_in(const float4* __restrict__ src, float4* __restrict__ dst,
                                                         int64_t n4) {
  pdl_trigger();                         // the layer's first kernel may become resident now; it
                                         // waits for this kernel's completion before reading x
  const int64_t i0 = (int64_t)blockIdx.x * kIoThreads + threadIdx.x, stride = (int64_t)gridDim.x * kIoThreads;
  float4 v[4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (i0 + u * stride < n4) v[u] = src[i0 + u * stride];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (i0 + u * stride < n4) dst[i0 + u * stride] = v[u];
  for (int64_t i = i0 + 4 * stride; i < n4; i += stride) dst[i] = src[i];
  pdl_wait();                            // complete only after the previous call's last kernel:
                                         // the layer's first kernel waits for this one
}

// y_dev -> y_host, after the layer. The next call's input copy may launch at once (it writes
// only x_dev, and completes only after this kernel).
__global__ void __launch_bounds__(kIoThreads) k_copy_out(const float4* __restrict__ src, float4* __restrict__ dst,
                                                          int64_t n4) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * kIoThreads + threadIdx.x; i < n4; i += (int64_t)gridDim.x * kIoThreads)
    dst[i] = src[i];
}

int io_grid(int64_t n4) {
  const int64_t per_round = (int64_t)kIoThreads * 4;   // four float4 per thread in flight
  const int64_t g = (n4 + per_round - 1) / per_round;
  return (int)(g < 1 ? 1 : (g > 4 * 148 ? 4 * 148 : g));
}

}  // namespace

cudaError_t launch_copy_in(const float* x_host_mapped, float* x_dev, int64_t n, cudaStream_t st) {
  const int64_t n4 = n / 4;
  return launch_pdl(k_copy_in, dim3(io_grid(n4)), dim3(kIoThreads), 0, st,
                    reinterpret_cast<const float4*>(x_host_mapped), reinterpret_cast<float4*>(x_dev), n4);
}

cudaError_t launch_copy_out(const float* y_dev, float* y_host_mapped, int64_t n, cudaStream_t st) {
  const int64_t n4 = n / 4;
  return launch_pdl(k_copy_out, dim3(io_grid(n4)), dim3(kIoThreads), 0, st, reinterpret_cast<const float4*>(y_dev),
                    reinterpret_cast<float4*>(y_host_mapped), n4);
}

}  // namespace moe
