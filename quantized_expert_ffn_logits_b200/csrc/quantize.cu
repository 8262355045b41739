// quantize.cu -- expert weight and activation quantization kernels.
//
// Symmetric quantization with stored-scale codes (GLM-5.2 colibri page, "What's
// implemented": "Quantization kernels: int8 / packed int4 / packed int2,
// per-row scales, dequant-on-use"; Q8_0-style int8 activations from the same
// section; group size 32 from the mtlm-7m-base card, "Files").
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

// A float8 E4M3 code ("fn": no infinities) as fp32, from the format's bit layout: sign bit 7,
// exponent bits 6-3 (bias 7), mantissa bits 2-0; exponent 0 is subnormal (m * 2^-9);
// exponent 15 with mantissa 7 is NaN. Exact.
__device__ __forceinline__ float fp8_e4m3(uint32_t v) {
  const uint32_t e = (v >> 3) & 15u, m = v & 7u;
  float mag = e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) mag = __uint_as_float(0x7fc00000u);
  return (v & 0x80u) ? -mag : mag;
}

// Weight values to quantize: fp32 rows, or FP8 checkpoint rows (the GLM page's FP8 -> int4
// converter): E4M3 codes with one fp32 inverse scale per 128 x 128 block of each expert's
// matrix, value = code * scale (one fp32 rounding).
struct WSource {
  const float* gu;          // fp32 [E][2I][H]
  const float* dn;          // fp32 [E][H][I]
  const uint8_t* gu8;       // E4M3 [E][2I][H]
  const float* gu_s;        //   [E][ceil(2I/128)][ceil(H/128)]
  const uint8_t* dn8;       // E4M3 [E][H][I]
  const float* dn_s;        //   [E][ceil(H/128)][ceil(I/128)]
};

// One warp per weight row. Rows [0, E*2I) are gate/up rows (logical [E][2I][H]),
// rows [E*2I, E*2I + E*H) are down rows (logical [E][H][I]). Codes and scales are
// written straight into the blob's tiled layout (include/moe_b200.h).
template <bool FP8>
__global__ void __launch_bounds__(256) k_quantize_experts(const WSource w, BlobView b, uint8_t* gu_w,
                                                          uint8_t* dn_w, uint8_t* gu_s, uint8_t* dn_s) {
  const int lane = threadIdx.x & 31;
  const int64_t n_gu = (int64_t)b.E * 2 * b.I;
  const int64_t n_rows = n_gu + (int64_t)b.E * b.H;
  const float qmax = b.wbits == 8 ? 127.0f : b.wbits == 4 ? 7.0f : 1.0f;   // 2^(bits-1) - 1
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t R = warp0; R < n_rows; R += nwarps) {
    const float* src = nullptr;             // fp32 source row
    const uint8_t* src8 = nullptr;          // FP8 source row and its blocks' scales
    const float* srow = nullptr;
    int K;
    bool down;
    int64_t blk = 0;     // gate/up: first row of the row's 128-row block
    int r = 0;           // row inside its block
    int e = 0, hb = 0;   // down: expert, 128-row block of H
    if (R < n_gu) {
      e = (int)(R / (2 * b.I));
      const int lr = (int)(R % (2 * b.I));
      const int half = lr >= b.I;
      const int i = lr - half * b.I;
      K = b.H;
      down = false;
      r = half * 64 + (i & 63);
      blk = (int64_t)e * 2 * b.I + (int64_t)(i >> 6) * 128;
      if constexpr (FP8) {
        src8 = w.gu8 + R * (int64_t)K;
        srow = w.gu_s + ((int64_t)e * ((2 * b.I + 127) / 128) + lr / 128) * ((K + 127) / 128);
      } else {
        src = w.gu + R * (int64_t)K;
      }
    } else {
      const int64_t R2 = R - n_gu;
      e = (int)(R2 / b.H);
      const int n = (int)(R2 % b.H);
      K = b.I;
      down = true;
      hb = n >> 7;
      r = n & 127;
      if constexpr (FP8) {
        src8 = w.dn8 + R2 * (int64_t)K;
        srow = w.dn_s + ((int64_t)e * ((b.H + 127) / 128) + n / 128) * ((K + 127) / 128);
      } else {
        src = w.dn + R2 * (int64_t)K;
      }
    }
    auto value = [&](int k) -> float {
      if constexpr (FP8) return __fmul_rn(fp8_e4m3(src8[k]), srow[k >> 7]);
      else return src[k];
    };
    const int G = K / 32;
    const int kb = kbytes(K, b.wbits);
    const int U = b.I / 64, HB = b.H / 128;
    const int sb = 8 * b.wbits;                       // bytes of 64 elements
    // byte `byte` of this row's codes -> its place in the tiled region
    auto code_at = [&](int byte) -> uint8_t* {
      if (!down) return gu_w + blk * kb + (int64_t)(byte >> 4) * (128 * 16) + r * 16 + (byte & 15);
      const int u = byte / sb, bb = byte - u * sb;
      const int64_t slab = ((int64_t)e * U + u) * HB + hb;
      return dn_w + ((slab * (sb / 16) + (bb >> 4)) * 128 + r) * 16 + (bb & 15);
    };
    // scale slot of group g (fp16) or of the row (fp32)
    auto scale_at = [&](int g) -> uint8_t* {
      if (!down) return b.wg32 ? gu_s + ((blk * G) + (int64_t)g * 128 + r) * 2 : gu_s + (blk + r) * 4;
      if (!b.wg32) return dn_s + ((int64_t)e * b.H + hb * 128 + r) * 4;
      const int64_t slab = ((int64_t)e * U + (g >> 1)) * HB + hb;
      return dn_s + ((slab * 2 + (g & 1)) * 128 + r) * 2;
    };
    float s_row = 0.0f;
    if (!b.wg32) {
      float amax = 0.0f;
      for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(value(k)));
      amax = warp_max(amax);
      s_row = __fdiv_rn(amax, qmax);
      if (lane == 0) *reinterpret_cast<float*>(scale_at(0)) = s_row;
    }
    for (int g = 0; g < G; ++g) {
      const float v = value(32 * g + lane);
      float s = s_row;
      if (b.wg32) {
        const float amax = warp_max(fabsf(v));
        s = f16_round(__fdiv_rn(amax, qmax));
        if (lane == 0) *reinterpret_cast<__half*>(scale_at(g)) = __float2half_rn(s);
      }
      const int q = quant_code(v, s, qmax);
      if (b.wbits == 8) {
        *code_at(32 * g + lane) = (uint8_t)(int8_t)q;
      } else if (b.wbits == 4) {
        const int hi = __shfl_down_sync(0xffffffffu, q, 1);
        if ((lane & 1) == 0) *code_at(16 * g + (lane >> 1)) = (uint8_t)((q & 15) | ((hi & 15) << 4));
      } else {
        // four 2-bit fields per byte: element 4j + i in bits 2i .. 2i + 1
        const int q1 = __shfl_down_sync(0xffffffffu, q, 1);
        const int q2 = __shfl_down_sync(0xffffffffu, q, 2);
        const int q3 = __shfl_down_sync(0xffffffffu, q, 3);
        if ((lane & 3) == 0)
          *code_at(8 * g + (lane >> 2)) = (uint8_t)((q & 3) | ((q1 & 3) << 2) | ((q2 & 3) << 4) | ((q3 & 3) << 6));
      }
    }
  }
}

// One CTA per token. g32: a warp per group of 32; token mode: one fp32 scale over
// the row. Optionally zeroes the token's output row (the layer accumulates y).
__global__ void __launch_bounds__(256) k_quantize_act(const float* __restrict__ x, int T, int H,
                                                      int g32, int8_t* __restrict__ q,
                                                      void* scales, float* y_zero, int* status) {
  pdl_wait();
  const int t = blockIdx.x;
  if (t >= T) return;
  if (status && t == 0 && threadIdx.x == 0) {
    status[0] = 0;
    status[2] = 0;
    status[3] = 0;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* xr = x + (int64_t)t * H;
  int8_t* qr = q + (int64_t)t * H;
  if (y_zero) {
    float4* yr = reinterpret_cast<float4*>(y_zero + (int64_t)t * H);
    for (int k = threadIdx.x; k < H / 4; k += blockDim.x) yr[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (g32) {
    __half* sr = reinterpret_cast<__half*>(scales) + (int64_t)t * (H / 32);
    for (int g = warp; g < H / 32; g += nw) {
      const float v = xr[32 * g + lane];
      const float s = f16_round(__fdiv_rn(warp_max(fabsf(v)), 127.0f));
      qr[32 * g + lane] = (int8_t)quant_code_rcp(v, s, __frcp_rn(s), 127.0f);
      if (lane == 0) sr[g] = __float2half_rn(s);
    }
  } else {
    __shared__ float red[32];
    float amax = 0.0f;
    for (int k = threadIdx.x; k < H; k += blockDim.x) amax = fmaxf(amax, fabsf(xr[k]));
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (warp == 0) {
      float v = lane < nw ? red[lane] : 0.0f;
      v = warp_max(v);
      if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const float s = __fdiv_rn(red[0], 127.0f);
    const float rs = __frcp_rn(s);
    for (int k = threadIdx.x; k < H; k += blockDim.x) qr[k] = (int8_t)quant_code_rcp(xr[k], s, rs, 127.0f);
    if (threadIdx.x == 0) reinterpret_cast<float*>(scales)[t] = s;
  }
}

// Token-mode quantization of h (one fp32 scale per (token, expert) over I).
__global__ void __launch_bounds__(256) k_quantize_rows_token(const float* __restrict__ h, int rows,
                                                             int K, int8_t* __restrict__ q,
                                                             float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  if (r >= rows) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* hr = h + (int64_t)r * K;
  __shared__ float red[32];
  float amax = 0.0f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(hr[k]));
  amax = warp_max(amax);
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  if (warp == 0) {
    float v = lane < nw ? red[lane] : 0.0f;
    v = warp_max(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  const float s = __fdiv_rn(red[0], 127.0f);
  for (int k = threadIdx.x; k < K; k += blockDim.x) q[(int64_t)r * K + k] = (int8_t)quant_code(hr[k], s, 127.0f);
  if (threadIdx.x == 0) scales[r] = s;
}

namespace {
int64_t quantize_blocks(const BlobView& b) {
  const int64_t rows = (int64_t)b.E * (2 * b.I + b.H);
  return std::min<int64_t>((rows + 7) / 8, 148 * 64);
}
}  // namespace

void launch_quantize_experts(const float* w_gu, const float* w_dn, const BlobView& b,
                             uint8_t* gu_w, uint8_t* dn_w, uint8_t* gu_s, uint8_t* dn_s,
                             cudaStream_t st) {
  WSource w{};
  w.gu = w_gu;
  w.dn = w_dn;
  k_quantize_experts<false><<<(unsigned)quantize_blocks(b), 256, 0, st>>>(w, b, gu_w, dn_w, gu_s, dn_s);
}

void launch_quantize_experts_fp8(const uint8_t* w_gu, const float* s_gu, const uint8_t* w_dn,
                                 const float* s_dn, const BlobView& b, uint8_t* gu_w, uint8_t* dn_w,
                                 uint8_t* gu_s, uint8_t* dn_s, cudaStream_t st) {
  WSource w{};
  w.gu8 = w_gu;
  w.gu_s = s_gu;
  w.dn8 = w_dn;
  w.dn_s = s_dn;
  k_quantize_experts<true><<<(unsigned)quantize_blocks(b), 256, 0, st>>>(w, b, gu_w, dn_w, gu_s, dn_s);
}

void launch_quantize_act(const float* x, int T, int H, int g32, int8_t* q, void* scales,
                         float* y_zero, int* status, cudaStream_t st) {
  if (T <= 0) return;
  launch_pdl(k_quantize_act, dim3(T), dim3(256), 0, st, x, T, H, g32, q, scales, y_zero, status);
}

void launch_quantize_rows_token(const float* h, int rows, int K, int8_t* q, float* scales,
                                cudaStream_t st) {
  if (rows <= 0) return;
  launch_pdl(k_quantize_rows_token, dim3(rows), dim3(256), 0, st, h, rows, K, q, scales);
}

}  // namespace moe
