// common.cuh -- device helpers shared by the kernels of the B200 MoE FFN layer.
//
// Every helper that takes part in a decision that yields an integer (a
// quantized code, a top-k selection) is written with explicit round-to-nearest
// intrinsics (__fmaf_rn, __fmul_rn, __fadd_rn, __fdiv_rn) so that nvcc cannot
// contract or reorder it: these sequences are the numerical contract stated
// in include/moe_b200.h.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kStatusDeviceCheck = 5;
constexpr int kStatusTimeout = 6;

// ------------------------------------------------------------------ exp & co.
// exp(a) in fp32: Cody-Waite reduction a = n ln2 + r with ln 2 split into a
// 24-bit head and its fp32-rounded tail, degree-7 Taylor polynomial (1/k!
// rounded to fp32) in Horner form, then scaling by 2^n built in the exponent
// field. The argument is clamped to [-87, 88] so 2^n stays a normal number.
__device__ __forceinline__ float cexp(float a) {
  a = fminf(fmaxf(a, -87.0f), 88.0f);
  const float kf = rintf(__fmul_rn(a, 0x1.715476p+0f));   // log2(e)
  float r = __fmaf_rn(-kf, 0x1.62e43p-1f, a);              // ln2 head
  r = __fmaf_rn(-kf, -0x1.05c61p-29f, r);                  // ln2 tail
  float p = 0x1.a01a02p-13f;                               // 1/7!
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);                    // 1/6!
  p = __fmaf_rn(p, r, 0x1.111112p-7f);                     // 1/5!
  p = __fmaf_rn(p, r, 0x1.555556p-5f);                     // 1/4!
  p = __fmaf_rn(p, r, 0x1.555556p-3f);                     // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int n = (int)kf;
  return __fmul_rn(p, __int_as_float((n + 127) << 23));
}

__device__ __forceinline__ float csigmoid(float L) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, cexp(-L)));
}

// SwiGLU: h = (g / (1 + exp(-g))) * u.
__device__ __forceinline__ float cswiglu(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, cexp(-g))), u);
}

// Exact int -> float for |v| < 2^22 with two full-rate operations: the bits of 1.5 * 2^23
// plus v are the float 1.5 * 2^23 + v (the exponent stays 2^23, so the ulp is 1); subtracting
// 1.5 * 2^23 leaves v exactly. Group dots stay below 32 * 127 * 127 < 2^19.
__device__ __forceinline__ float exact_i2f(int v) {
  return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
}

// ---------------------------------------------------------------- quantization
__device__ __forceinline__ float f16_round(float d) { return __half2float(__float2half_rn(d)); }

// Code of v under stored scale s: round half away from zero, clamp to [-qmax, qmax].
__device__ __forceinline__ int quant_code(float v, float s, float qmax) {
  if (s == 0.0f) return 0;
  float r = roundf(__fdiv_rn(v, s));
  r = fminf(fmaxf(r, -qmax), qmax);
  return (int)r;
}

// quant_code(v, s, qmax) with one multiplication by rs = fl(1 / s) instead of the division:
// fl(v * rs) and fl(v / s) both lie within 2 ulp of v / s (|v / s| <= qmax + 1 < 2^7), so they
// round to different integers only when v / s is that close to a half-integer; such values
// (fractional part within 2^-16 * max(|q|, 1) of 0.5) take the exact division, and so does
// any product that is not a plausible code (1 / s overflowed for a tiny s). Bit-identical to
// quant_code.
__device__ __forceinline__ int quant_code_rcp(float v, float s, float rs, float qmax) {
  if (s == 0.0f) return 0;
  const float r = __fmul_rn(v, rs);
  const float a = fabsf(r);
  const float f = a - truncf(a);
  float q;
  if (!(a < 256.0f) || fabsf(f - 0.5f) <= 0x1p-16f * fmaxf(a, 1.0f)) q = roundf(__fdiv_rn(v, s));
  else q = roundf(r);
  q = fminf(fmaxf(q, -qmax), qmax);
  return (int)q;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Record the first bounded wait that gave up: status word = timeout, word 2 = kernel | wait
// << 4 | stage << 8, word 3 = the CTA.
__device__ __forceinline__ void wait_failed(int* status, int kernel, int role, int stage) {
  if (!status) return;
  if (atomicCAS(status, 0, kStatusTimeout) == 0) {
    status[2] = kernel | (role << 4) | (stage << 8);
    status[3] = (int)blockIdx.x;
  }
}

// y[0..3] += (a, b, c, d): one 16-byte reduction (sm_90+), p 16-byte aligned.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// --------------------------------------------------------------- integer dots
// Signed x signed 4-way byte dot.
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  return __dp4a((int)a, (int)b, c);
}

// Unsigned (a) x signed (b) 4-way byte dot.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// One group of 32 int8 weights (two 16-byte pieces) against 32 int8 activations.
__device__ __forceinline__ int group_dot_i8(const uint4& w0, const uint4& w1, const uint4& x0,
                                            const uint4& x1) {
  int d = dp4a_ss(w0.x, x0.x, 0);
  d = dp4a_ss(w0.y, x0.y, d);
  d = dp4a_ss(w0.z, x0.z, d);
  d = dp4a_ss(w0.w, x0.w, d);
  d = dp4a_ss(w1.x, x1.x, d);
  d = dp4a_ss(w1.y, x1.y, d);
  d = dp4a_ss(w1.z, x1.z, d);
  d = dp4a_ss(w1.w, x1.w, d);
  return d;
}

// One group of 32 packed int4 weights (one 16-byte piece, element 2j in the low
// nibble of byte j) against activations stored de-interleaved per 8 elements:
// xe.* hold elements {0,2,4,6} and xo.* elements {1,3,5,7} of each 8-element
// word. Nibbles are read as unsigned n ^ 8 = q + 8, so the dot is corrected by
// 8 * (sum of the group's activations), xsum.
__device__ __forceinline__ int group_dot_i4(const uint4& w, const uint4& xe, const uint4& xo,
                                            int xsum) {
  const uint32_t m = 0x0F0F0F0Fu;
  uint32_t v0 = w.x ^ 0x88888888u, v1 = w.y ^ 0x88888888u;
  uint32_t v2 = w.z ^ 0x88888888u, v3 = w.w ^ 0x88888888u;
  int d = dp4a_us(v0 & m, xe.x, 0);
  d = dp4a_us((v0 >> 4) & m, xo.x, d);
  d = dp4a_us(v1 & m, xe.y, d);
  d = dp4a_us((v1 >> 4) & m, xo.y, d);
  d = dp4a_us(v2 & m, xe.z, d);
  d = dp4a_us((v2 >> 4) & m, xo.z, d);
  d = dp4a_us(v3 & m, xe.w, d);
  d = dp4a_us((v3 >> 4) & m, xo.w, d);
  return d - 8 * xsum;
}

// One group of 32 packed int2 weights (8 bytes: w.x holds elements 0..15, w.y 16..31; element
// 4j + i in bits 2i .. 2i + 1 of byte j) against activations stored de-interleaved per 16
// elements: xa.{x,y,z,w} hold elements {0,4,8,12}, {1,5,9,13}, {2,6,10,14}, {3,7,11,15} of the
// group's first 16, xb the same of its last 16. Each 2-bit field is read as unsigned
// f ^ 2 = q + 2 (two's complement q in -2..1), so the dot is corrected by 2 * xsum.
__device__ __forceinline__ int group_dot_i2(const uint2& w, const uint4& xa, const uint4& xb, int xsum) {
  const uint32_t m = 0x03030303u;
  const uint32_t v0 = w.x ^ 0xAAAAAAAAu, v1 = w.y ^ 0xAAAAAAAAu;
  int d = dp4a_us(v0 & m, xa.x, 0);
  d = dp4a_us((v0 >> 2) & m, xa.y, d);
  d = dp4a_us((v0 >> 4) & m, xa.z, d);
  d = dp4a_us((v0 >> 6) & m, xa.w, d);
  d = dp4a_us(v1 & m, xb.x, d);
  d = dp4a_us((v1 >> 2) & m, xb.y, d);
  d = dp4a_us((v1 >> 4) & m, xb.z, d);
  d = dp4a_us((v1 >> 6) & m, xb.w, d);
  return d - 2 * xsum;
}

// 16 activation bytes (words a = x0..x3, x4..x7, x8..x11, x12..x15) -> (x0 x4 x8 x12),
// (x1 x5 x9 x13), (x2 x6 x10 x14), (x3 x7 x11 x15): the order of a packed int2 word's fields.
__device__ __forceinline__ uint4 deinterleave16(const uint4& a) {
  const uint32_t t0 = __byte_perm(a.x, a.y, 0x5140), t1 = __byte_perm(a.z, a.w, 0x5140);
  const uint32_t t2 = __byte_perm(a.x, a.y, 0x7362), t3 = __byte_perm(a.z, a.w, 0x7362);
  return make_uint4(__byte_perm(t0, t1, 0x5410), __byte_perm(t0, t1, 0x7632), __byte_perm(t2, t3, 0x5410),
                    __byte_perm(t2, t3, 0x7632));
}

// Sum of the 32 signed codes of a group (two 16-byte words).
__device__ __forceinline__ int code_sum32(const uint4& a0, const uint4& a1) {
  int s = __dp4a((int)a0.x, 0x01010101, 0);
  s = __dp4a((int)a0.y, 0x01010101, s);
  s = __dp4a((int)a0.z, 0x01010101, s);
  s = __dp4a((int)a0.w, 0x01010101, s);
  s = __dp4a((int)a1.x, 0x01010101, s);
  s = __dp4a((int)a1.y, 0x01010101, s);
  s = __dp4a((int)a1.z, 0x01010101, s);
  return __dp4a((int)a1.w, 0x01010101, s);
}

// 8 activation bytes x0..x7 -> (x0 x2 x4 x6), (x1 x3 x5 x7).
__device__ __forceinline__ void deinterleave8(uint32_t lo, uint32_t hi, uint32_t& even,
                                              uint32_t& odd) {
  even = __byte_perm(lo, hi, 0x6420);
  odd = __byte_perm(lo, hi, 0x7531);
}

// ------------------------------------------------------------------ layouts
// Views of one expert blob (layout documented in include/moe_b200.h).
struct BlobView {
  const uint8_t* gu_w;  // R0 gate/up codes
  const uint8_t* dn_w;  // R1 down codes
  const uint8_t* gu_s;  // R2 gate/up scales
  const uint8_t* dn_s;  // R3 down scales
  int E, H, I;
  int wbits;            // 8, 4 or 2
  int wg32;             // 1: fp16 group-32 scales, 0: fp32 per row
};

__host__ __device__ __forceinline__ int kbytes(int K, int wbits) { return K * wbits / 8; }

}  // namespace moe
