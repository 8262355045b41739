// expert_gemv.cu -- per-group integer dots of sampled expert rows (debug entry point).
//
// The integer-dot step of the GLM-5.2 colibri page ("Integer-dot kernels",
// "Quantization kernels: ... dequant-on-use"), evaluated through the blob layout
// with the same dot helpers (common.cuh) as the expert kernels.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// Per-group int32 dots of sampled rows, through the same blob addressing and dot
// helpers as the kernels above. One thread per (sample, group).
__global__ void k_group_dots(BlobView b, int which, int n, const int32_t* __restrict__ expert,
                             const int32_t* __restrict__ row, const int8_t* __restrict__ act,
                             int32_t* __restrict__ dots) {
  const int K = which == 0 ? b.H : b.I;
  const int G = K / 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (int64_t)n * G) return;
  const int smp = (int)(id / G), g = (int)(id % G);
  const int e = expert[smp], r = row[smp];
  const int KB = kbytes(K, b.wbits);
  const int gbytes = 4 * b.wbits;                // code bytes of one group: 32, 16 or 8
  const uint8_t* p0;                             // the group's first code byte
  if (which == 0) {
    const int half = r >= b.I;
    const int i = r - half * b.I;
    const int64_t blk = (int64_t)e * 2 * b.I + (int64_t)(i >> 6) * 128;
    const int byte = g * gbytes;
    p0 = b.gu_w + blk * KB + ((int64_t)(byte >> 4) * 128 + half * 64 + (i & 63)) * 16 + (byte & 15);
  } else {
    // slab of the group's 64 columns; the group starts at byte (g % 2) * gbytes of it
    const int U = b.I / 64, HB = b.H / 128, sbytes = 2 * gbytes;
    const int64_t slab = ((int64_t)e * U + g / 2) * HB + (r >> 7);
    const int byte = (g & 1) * gbytes;
    p0 = b.dn_w + ((slab * (sbytes / 16) + (byte >> 4)) * 128 + (r & 127)) * 16 + (byte & 15);
  }
  const uint8_t* xg = reinterpret_cast<const uint8_t*>(act) + (int64_t)smp * K + 32 * g;
  const uint4 x0 = *reinterpret_cast<const uint4*>(xg);
  const uint4 x1 = *reinterpret_cast<const uint4*>(xg + 16);
  int d;
  if (b.wbits == 8) {
    const uint4 w0 = *reinterpret_cast<const uint4*>(p0);
    const uint4 w1 = *reinterpret_cast<const uint4*>(p0 + 128 * 16);
    d = group_dot_i8(w0, w1, x0, x1);
  } else if (b.wbits == 2) {
    const uint2 w = *reinterpret_cast<const uint2*>(p0);
    d = group_dot_i2(w, deinterleave16(x0), deinterleave16(x1), code_sum32(x0, x1));
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(p0);
    uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
    deinterleave8(x0.x, x0.y, e0, o0);
    deinterleave8(x0.z, x0.w, e1, o1);
    deinterleave8(x1.x, x1.y, e2, o2);
    deinterleave8(x1.z, x1.w, e3, o3);
    int xsum = __dp4a((int)x0.x, 0x01010101, 0);
    xsum = __dp4a((int)x0.y, 0x01010101, xsum);
    xsum = __dp4a((int)x0.z, 0x01010101, xsum);
    xsum = __dp4a((int)x0.w, 0x01010101, xsum);
    xsum = __dp4a((int)x1.x, 0x01010101, xsum);
    xsum = __dp4a((int)x1.y, 0x01010101, xsum);
    xsum = __dp4a((int)x1.z, 0x01010101, xsum);
    xsum = __dp4a((int)x1.w, 0x01010101, xsum);
    d = group_dot_i4(w, make_uint4(e0, e1, e2, e3), make_uint4(o0, o1, o2, o3), xsum);
  }
  dots[(int64_t)smp * G + g] = d;
}

void launch_group_dots(const BlobView& b, int which, int n, const int32_t* expert,
                       const int32_t* row, const int8_t* act, int32_t* dots, cudaStream_t st) {
  const int K = which == 0 ? b.H : b.I;
  const int64_t total = (int64_t)n * (K / 32);
  if (total <= 0) return;
  k_group_dots<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(b, which, n, expert, row, act, dots);
}

}  // namespace moe
