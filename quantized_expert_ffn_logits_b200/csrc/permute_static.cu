// permute_static.cu -- batch-union grouping without any caller-supplied or
// library-allocated workspace.
//
// Some callers cannot hand this library a scratch buffer and cannot let it
// allocate one either: code that runs while a CUDA graph is being captured
// (cudaMalloc is not a stream operation and breaks or invalidates the capture),
// serving loops with a fixed memory plan where a framework's caching allocator
// owns the whole device budget, and plugin hosts that pass only the tensors of an
// operator. moe_permute_no_alloc serves them: its scratch is a fixed-size array
// compiled into this library as a device global, so every GPU that loads the
// library reserves kPermuteScratchBytes for it until the process exits.
#include <cstdint>
#include <mutex>

#include "../../include/moe_b200.h"
#include "kernels.cuh"

namespace {

// Largest grouping this entry point accepts: two [ceil(T/32)][E] uint32 tables plus
// the distinct-expert lists must fit (e.g. T = 4096 tokens with E = 512 experts).
constexpr size_t kPermuteScratchBytes = size_t(1) << 20;   // 1 MiB

static __device__ __align__(256) unsigned char g_permute_scratch[kPermuteScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

inline int64_t al256(int64_t v) { return (v + 255) & ~int64_t(255); }

// Device address of g_permute_scratch on the current device. In host code the
// symbol names a host-side shadow, not device memory, so the address must come
// from cudaGetSymbolAddress (once per device, with that device current).
moe_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_no_alloc(const int32_t* idx, int32_t T, int32_t k, int32_t E,
                                           int32_t* offsets, int32_t* perm, void* stream) {
  if (T < 0 || k < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!idx || !offsets || !perm) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_permute_workspace_bytes(T, k, E);
  if (need == 0 || need > kPermuteScratchBytes) return MOE_ERR_WORKSPACE;
  void* base_addr = nullptr;
  const moe_status s = scratch_address(&base_addr);
  if (s != MOE_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(base_addr);
  const int64_t C = (T + 31) / 32;
  int64_t o = 256;                       // bytes [0, 256): status word
  uint32_t* masks = reinterpret_cast<uint32_t*>(ws + o);
  o += al256(C * E * 4);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + o);
  o += al256(C * E * 4);
  moe::Grouping g{};
  g.offsets = offsets;
  g.perm = perm;
  g.n_active = reinterpret_cast<int32_t*>(ws + o);
  o += 256;
  g.act_expert = reinterpret_cast<int32_t*>(ws + o);
  o += al256((int64_t)(E + 1) * 4);
  g.act_begin = reinterpret_cast<int32_t*>(ws + o);
  // The kernel zeroes its mask rows before use and resets the status word, so
  // nothing left in the array by an earlier call leaks into this one.
  moe::launch_permute(idx, T, k, E, 0, E, g, masks, prefix, reinterpret_cast<int*>(ws), 1,
                      static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
