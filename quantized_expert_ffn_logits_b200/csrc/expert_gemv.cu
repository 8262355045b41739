// expert_gemv.cu -- weight-streaming grouped expert kernels (decode / small batches).
//
// Dequant-on-use integer dots (GLM-5.2 colibri page, "What's implemented":
// "Integer-dot kernels (Q8_0-style int8 activations ...)", "Quantization kernels:
// int8 / packed int4 ... dequant-on-use") over the batch-union grouping ("Batch-union
// MoE"): one CTA streams one block of one selected expert's rows from HBM exactly
// once and applies it to every token routed to that expert.
//
// Lane-per-row mapping: in the blob every 16-byte piece of 256 (gate/up) or 128
// (down) consecutive rows is contiguous, so the 32 lanes of a warp, each owning one
// row, read 512 contiguous bytes per 128-bit load. A lane accumulates its row's
// exact int32 group dots with dp4a and runs the row's fp32 scale chain in group
// order, so no cross-lane reduction is needed and the chain order is fixed.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int TM = 4;   // token slots per pass over the weights
constexpr int GU = 4;   // groups of 32 per register batch (two batches in flight)

struct ActSmem {
  uint8_t* xs;   // [TM][K] activation codes (int4 weights: each 8-byte word de-interleaved)
  float* sx;     // [TM][G] group scales or [TM] token scales
  int* xsum;     // [TM][G] sums of the activation codes of each group (int4 weights)
};

__host__ __device__ inline size_t act_smem_bytes(int K) {
  const int G = K / 32;
  return (size_t)TM * K + (size_t)TM * G * sizeof(float) * 2;
}

__device__ __forceinline__ ActSmem carve(uint8_t* smem, int K) {
  const int G = K / 32;
  ActSmem s;
  s.xs = smem;
  s.sx = reinterpret_cast<float*>(smem + TM * K);
  s.xsum = reinterpret_cast<int*>(s.sx + TM * G);
  return s;
}

// Stage the activation rows of up to TM slots into shared memory.
template <int WBITS, bool AG32>
__device__ __forceinline__ void stage_acts(const int8_t* __restrict__ qa, const void* sa, int K,
                                           int m, const int* rows, const ActSmem& s) {
  const int G = K / 32;
  const int words = K / 8;
  for (int l = threadIdx.x; l < m * words; l += blockDim.x) {
    const int tt = l / words, wi = l - tt * words;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(qa + (int64_t)rows[tt] * K) + wi);
    uint2 o = v;
    if (WBITS == 4) deinterleave8(v.x, v.y, o.x, o.y);
    reinterpret_cast<uint2*>(s.xs + tt * K)[wi] = o;
  }
  for (int l = threadIdx.x; l < m * G; l += blockDim.x) {
    const int tt = l / G, g = l - tt * G;
    if (AG32) {
      s.sx[tt * G + g] = __half2float(reinterpret_cast<const __half*>(sa)[(int64_t)rows[tt] * G + g]);
    } else if (g == 0) {
      s.sx[tt] = reinterpret_cast<const float*>(sa)[rows[tt]];
    }
    if (WBITS == 4) {
      const uint4* p = reinterpret_cast<const uint4*>(qa + (int64_t)rows[tt] * K + 32 * g);
      const uint4 a = __ldg(p), b = __ldg(p + 1);
      int sum = __dp4a((int)a.x, 0x01010101, 0);
      sum = __dp4a((int)a.y, 0x01010101, sum);
      sum = __dp4a((int)a.z, 0x01010101, sum);
      sum = __dp4a((int)a.w, 0x01010101, sum);
      sum = __dp4a((int)b.x, 0x01010101, sum);
      sum = __dp4a((int)b.y, 0x01010101, sum);
      sum = __dp4a((int)b.z, 0x01010101, sum);
      sum = __dp4a((int)b.w, 0x01010101, sum);
      s.xsum[tt * G + g] = sum;
    }
  }
}

// Per-lane row accumulator over K for up to TM activation rows, in canonical order.
// wrow: this lane's piece 0; piece p is at wrow + p * pstride. Scales: srow (fp16,
// group g at srow[g * sstride]) or sw_row.
template <int WBITS, bool WG32, bool AG32>
__device__ __forceinline__ void row_values(const uint8_t* __restrict__ wrow, int pstride,
                                           const __half* __restrict__ srow, int sstride,
                                           float sw_row, int K, int m, const ActSmem& s,
                                           float (&v)[TM]) {
  constexpr int PPG = WBITS == 8 ? 2 : 1;   // 16-byte pieces per group of 32
  constexpr int PB = GU * PPG;              // pieces per batch
  const int G = K / 32;
  float acc[TM];
  int isum[TM];
#pragma unroll
  for (int tt = 0; tt < TM; ++tt) {
    acc[tt] = 0.0f;
    isum[tt] = 0;
  }
  uint4 bufA[PB], bufB[PB];
  float scA[GU], scB[GU];
  auto load = [&](uint4 (&buf)[PB], float (&sc)[GU], int g0) {
#pragma unroll
    for (int q = 0; q < PB; ++q)
      buf[q] = __ldg(reinterpret_cast<const uint4*>(wrow + (int64_t)(g0 * PPG + q) * pstride));
    if (WG32) {
#pragma unroll
      for (int u = 0; u < GU; ++u) sc[u] = __half2float(srow[(int64_t)(g0 + u) * sstride]);
    }
  };
  auto compute = [&](const uint4 (&buf)[PB], const float (&sc)[GU], int g0) {
#pragma unroll
    for (int u = 0; u < GU; ++u) {
      const int g = g0 + u;
#pragma unroll
      for (int tt = 0; tt < TM; ++tt) {
        if (tt >= m) break;
        const uint8_t* xg = s.xs + tt * K + 32 * g;
        const uint4 x0 = *reinterpret_cast<const uint4*>(xg);
        const uint4 x1 = *reinterpret_cast<const uint4*>(xg + 16);
        int d;
        if (WBITS == 8) {
          d = group_dot_i8(buf[2 * u], buf[2 * u + 1], x0, x1);
        } else {
          const uint4 xe = make_uint4(x0.x, x0.z, x1.x, x1.z);
          const uint4 xo = make_uint4(x0.y, x0.w, x1.y, x1.w);
          d = group_dot_i4(buf[u], xe, xo, s.xsum[tt * G + g]);
        }
        if (WG32 && AG32) {
          acc[tt] = __fmaf_rn(__int2float_rn(d), __fmul_rn(sc[u], s.sx[tt * G + g]), acc[tt]);
        } else if (WG32) {
          acc[tt] = __fmaf_rn(__int2float_rn(d), sc[u], acc[tt]);
        } else if (AG32) {
          acc[tt] = __fmaf_rn(__int2float_rn(d), s.sx[tt * G + g], acc[tt]);
        } else {
          isum[tt] += d;
        }
      }
    }
  };
  load(bufA, scA, 0);
  for (int g0 = 0; g0 < G; g0 += 2 * GU) {
    if (g0 + GU < G) load(bufB, scB, g0 + GU);
    compute(bufA, scA, g0);
    if (g0 + 2 * GU < G) load(bufA, scA, g0 + 2 * GU);
    if (g0 + GU < G) compute(bufB, scB, g0 + GU);
  }
#pragma unroll
  for (int tt = 0; tt < TM; ++tt) {
    if (WG32 && AG32) v[tt] = acc[tt];
    else if (WG32) v[tt] = __fmul_rn(acc[tt], s.sx[tt]);
    else if (AG32) v[tt] = __fmul_rn(acc[tt], sw_row);
    else v[tt] = __fmul_rn(__fmaf_rn(__int2float_rn(isum[tt]), s.sx[tt], 0.0f), sw_row);
  }
}

// Resolve the expert and slot range of grouped unit a_idx; false if the unit is idle.
__device__ __forceinline__ bool unit_range(const ExpertArgs& a, int a_idx, int& e, int& s0,
                                           int& s1) {
  if (a.act_expert) {
    if (a_idx >= *a.n_active) return false;
    e = a.act_expert[a_idx];
    s0 = a.act_begin[a_idx];
    s1 = a.act_begin[a_idx + 1];
    if (e < 0 || e >= a.b.E || s0 < 0 || s0 > s1 || s1 > a.T * a.k) {
      if (threadIdx.x == 0) set_status(a.status, kStatusDeviceCheck);
      return false;
    }
  } else {
    if (a_idx != 0) return false;
    e = 0;
    s0 = 0;
    s1 = a.T;
  }
  return true;
}

// Gate/up + SwiGLU + h quantization. CTA = one selected expert x 32 intermediate
// indices; warp 0 streams the 32 gate rows, warp 1 the 32 up rows.
template <int WBITS, bool WG32, bool AG32>
__global__ void __launch_bounds__(64) k_gateup(ExpertArgs a) {
  const int I = a.b.I, H = a.b.H, K = H, G = K / 32;
  const int IB = I / 32;
  const int a_idx = blockIdx.x / IB, ib = blockIdx.x - a_idx * IB;
  int e, s0, s1;
  if (!unit_range(a, a_idx, e, s0, s1)) return;
  extern __shared__ __align__(16) uint8_t smem[];
  const ActSmem s = carve(smem, K);
  __shared__ float ubuf[TM][32];
  __shared__ int rows[TM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = ib * 32 + lane;
  const int r = warp * 128 + (i & 127);
  const int KB = kbytes(K, WBITS);
  const int64_t blk = (int64_t)e * 2 * I + (int64_t)(i >> 7) * 256;
  const uint8_t* wrow = a.b.gu_w + blk * KB + (int64_t)r * 16;
  const __half* srow = WG32 ? reinterpret_cast<const __half*>(a.b.gu_s) + blk * G + r : nullptr;
  const float sw_row = WG32 ? 0.0f : reinterpret_cast<const float*>(a.b.gu_s)[blk + r];
  for (int c0 = s0; c0 < s1; c0 += TM) {
    const int m = min(TM, s1 - c0);
    if (threadIdx.x < m) {
      const int slot = c0 + threadIdx.x;
      int row = slot;
      if (a.act_expert) {
        const int p = a.perm[slot];
        row = (p >= 0 && p < a.T * a.k) ? p / a.k : 0;
        if (p < 0 || p >= a.T * a.k) set_status(a.status, kStatusDeviceCheck);
      }
      rows[threadIdx.x] = row;
    }
    __syncthreads();
    stage_acts<WBITS, AG32>(a.qa, a.sa, K, m, rows, s);
    __syncthreads();
    float v[TM];
    row_values<WBITS, WG32, AG32>(wrow, 256 * 16, srow, 256, sw_row, K, m, s, v);
    if (a.dbg_a) {
      float* d = warp == 0 ? a.dbg_a : a.dbg_b;
      for (int tt = 0; tt < m; ++tt) d[(int64_t)(c0 + tt) * I + i] = v[tt];
    }
    if (warp == 1)
      for (int tt = 0; tt < m; ++tt) ubuf[tt][lane] = v[tt];
    __syncthreads();
    if (warp == 0) {
      for (int tt = 0; tt < m; ++tt) {
        const int slot = c0 + tt;
        const float h = cswiglu(v[tt], ubuf[tt][lane]);
        if (AG32) {
          const float sc = f16_round(__fdiv_rn(warp_max(fabsf(h)), 127.0f));
          a.qh[(int64_t)slot * I + i] = (int8_t)quant_code(h, sc, 127.0f);
          if (lane == 0) a.sh[(int64_t)slot * IB + ib] = __float2half_rn(sc);
        } else {
          a.hbuf[(int64_t)slot * I + i] = h;
        }
      }
    }
    __syncthreads();
  }
}

// Down projection + weighted combine. CTA = one selected expert x 128 output rows
// (four warps of 32). Each slot's row value is scaled by its routing weight and
// added into y with an fp32 atomic.
template <int WBITS, bool WG32, bool AG32>
__global__ void __launch_bounds__(128) k_down(ExpertArgs a) {
  const int I = a.b.I, H = a.b.H, K = I, G = K / 32;
  const int NB = H / 128;
  const int a_idx = blockIdx.x / NB, sb = blockIdx.x - a_idx * NB;
  int e, s0, s1;
  if (!unit_range(a, a_idx, e, s0, s1)) return;
  extern __shared__ __align__(16) uint8_t smem[];
  const ActSmem s = carve(smem, K);
  __shared__ int rows[TM], toks[TM];
  __shared__ float wts[TM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = warp * 32 + lane;
  const int n = sb * 128 + rl;
  const int KB = kbytes(K, WBITS);
  const int64_t blk = (int64_t)e * H + (int64_t)sb * 128;
  const uint8_t* wrow = a.b.dn_w + blk * KB + (int64_t)rl * 16;
  const __half* srow = WG32 ? reinterpret_cast<const __half*>(a.b.dn_s) + blk * G + rl : nullptr;
  const float sw_row = WG32 ? 0.0f : reinterpret_cast<const float*>(a.b.dn_s)[blk + rl];
  for (int c0 = s0; c0 < s1; c0 += TM) {
    const int m = min(TM, s1 - c0);
    if (threadIdx.x < m) {
      const int slot = c0 + threadIdx.x;
      rows[threadIdx.x] = slot;
      if (a.act_expert) {
        int p = a.perm[slot];
        if (p < 0 || p >= a.T * a.k) {
          set_status(a.status, kStatusDeviceCheck);
          p = 0;
        }
        toks[threadIdx.x] = p / a.k;
        wts[threadIdx.x] = a.wts[p];
      } else {
        toks[threadIdx.x] = slot;
        wts[threadIdx.x] = 1.0f;
      }
    }
    __syncthreads();
    stage_acts<WBITS, AG32>(a.qa, a.sa, K, m, rows, s);
    __syncthreads();
    float v[TM];
    row_values<WBITS, WG32, AG32>(wrow, 128 * 16, srow, 128, sw_row, K, m, s, v);
    for (int tt = 0; tt < m; ++tt) {
      if (a.dbg_a) a.dbg_a[(int64_t)(c0 + tt) * H + n] = v[tt];
      atomicAdd(a.y + (int64_t)toks[tt] * H + n, wts[tt] * v[tt]);
    }
    __syncthreads();
  }
}

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
  const uint8_t* base;
  int pstride;
  if (which == 0) {
    const int half = r >= b.I;
    const int i = r - half * b.I;
    const int64_t blk = (int64_t)e * 2 * b.I + (int64_t)(i >> 7) * 256;
    base = b.gu_w + blk * KB + (int64_t)(half * 128 + (i & 127)) * 16;
    pstride = 256 * 16;
  } else {
    const int64_t blk = (int64_t)e * b.H + (int64_t)(r >> 7) * 128;
    base = b.dn_w + blk * KB + (int64_t)(r & 127) * 16;
    pstride = 128 * 16;
  }
  const uint8_t* xg = reinterpret_cast<const uint8_t*>(act) + (int64_t)smp * K + 32 * g;
  const uint4 x0 = *reinterpret_cast<const uint4*>(xg);
  const uint4 x1 = *reinterpret_cast<const uint4*>(xg + 16);
  int d;
  if (b.wbits == 8) {
    const uint4 w0 = *reinterpret_cast<const uint4*>(base + (int64_t)(2 * g) * pstride);
    const uint4 w1 = *reinterpret_cast<const uint4*>(base + (int64_t)(2 * g + 1) * pstride);
    d = group_dot_i8(w0, w1, x0, x1);
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(base + (int64_t)g * pstride);
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

// ------------------------------------------------------------------ launches
template <int WBITS, bool WG32, bool AG32>
static void launch_gateup_t(const ExpertArgs& a, cudaStream_t st) {
  const size_t smem = act_smem_bytes(a.b.H);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_gateup<WBITS, WG32, AG32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         200 * 1024);
    attr = true;
  }
  const int units = (a.act_expert ? a.max_active : 1) * (a.b.I / 32);
  if (units > 0) k_gateup<WBITS, WG32, AG32><<<units, 64, smem, st>>>(a);
}

template <int WBITS, bool WG32, bool AG32>
static void launch_down_t(const ExpertArgs& a, cudaStream_t st) {
  const size_t smem = act_smem_bytes(a.b.I);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_down<WBITS, WG32, AG32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         200 * 1024);
    attr = true;
  }
  const int units = (a.act_expert ? a.max_active : 1) * (a.b.H / 128);
  if (units > 0) k_down<WBITS, WG32, AG32><<<units, 128, smem, st>>>(a);
}

#define MOE_DISPATCH(FN, a, st)                                          \
  do {                                                                   \
    const int sel = ((a).b.wbits == 8 ? 4 : 0) | ((a).b.wg32 ? 2 : 0) | ((a).ag32 ? 1 : 0); \
    switch (sel) {                                                       \
      case 7: FN<8, true, true>(a, st); break;                           \
      case 6: FN<8, true, false>(a, st); break;                          \
      case 5: FN<8, false, true>(a, st); break;                          \
      case 4: FN<8, false, false>(a, st); break;                         \
      case 3: FN<4, true, true>(a, st); break;                           \
      case 2: FN<4, true, false>(a, st); break;                          \
      case 1: FN<4, false, true>(a, st); break;                          \
      default: FN<4, false, false>(a, st); break;                        \
    }                                                                    \
  } while (0)

void launch_gateup(const ExpertArgs& a, cudaStream_t st) { MOE_DISPATCH(launch_gateup_t, a, st); }
void launch_down(const ExpertArgs& a, cudaStream_t st) { MOE_DISPATCH(launch_down_t, a, st); }

void launch_group_dots(const BlobView& b, int which, int n, const int32_t* expert,
                       const int32_t* row, const int8_t* act, int32_t* dots, cudaStream_t st) {
  const int K = which == 0 ? b.H : b.I;
  const int64_t total = (int64_t)n * (K / 32);
  if (total <= 0) return;
  k_group_dots<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(b, which, n, expert, row, act, dots);
}

}  // namespace moe
