// synth_gpu.cu -- seeded synthetic inputs, device side.
//
// Independent device implementation of the generator described in
// synth_cpu.c (SplitMix64 counter hash + Irwin-Hall sum of twelve 24-bit
// uniforms). It produces bit-identical floats for the same (seed, index), so
// large expert tensors can be generated directly in HBM while the oracle
// regenerates only the slices it needs on the host. Holds none of the MoE
// layer's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__global__ void normal_kernel(float* __restrict__ out, uint64_t n, uint64_t seed,
                              uint64_t offset, float c) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t base = 6ULL * (offset + i);
    int64_t s = 0;
#pragma unroll
    for (int m = 0; m < 6; ++m) {
      const uint64_t h = mix64(seed + (base + (uint64_t)m + 1ULL) * 0x9E3779B97F4A7C15ULL);
      s += (int64_t)(h >> 40) + (int64_t)((h >> 16) & 0xFFFFFFULL);
    }
    const int32_t z = (int32_t)(s - 6LL * 16777216LL);
    out[i] = __fmul_rn(__int2float_rn(z), c);
  }
}

}  // namespace

extern "C" int synth_normal_f32_device(float* out, uint64_t n, uint64_t seed, uint64_t offset,
                                       float sigma, void* stream) {
  if (n == 0) return 0;
  if (out == nullptr) return 1;
  const float c = sigma * 0x1p-24f;
  const int threads = 256;
  uint64_t blocks = (n + threads - 1) / threads;
  if (blocks > 148ULL * 64ULL) blocks = 148ULL * 64ULL;
  normal_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(out, n, seed, offset, c);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
