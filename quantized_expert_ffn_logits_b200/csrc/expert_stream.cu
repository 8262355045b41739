// expert_stream.cu -- weight-streaming expert kernels (decode and small batches).
//
// Integer dots per group of 32, the canonical fp32 scale chain per row, SwiGLU and h
// quantization in the gate/up epilogue (GLM-5.2 colibri page, "Integer-dot kernels",
// "Quantization kernels: ... dequant-on-use"; "Batch-union MoE": every selected expert's
// weights are streamed once per call, whatever the number of tokens routed to it).
//
// Memory design. In the blob the rows of one 16-byte piece are contiguous, so a warp whose
// lanes own 32 consecutive rows reads 512 contiguous bytes per 128-bit load. A CTA splits
// its 64 rows' K range over four warps per 32 rows; at start every warp prefetches its whole
// range into L2 (one prefetch per 512-byte run), so HBM streams the unit at full rate while
// the warp consumes it in batches of 16 register loads per lane. The exact int32 group dots
// are parked in shared memory and the ordered fp32 chain of each row runs once all of its
// groups are in. (Measured on this part: plain streaming loads reach 7.2 TB/s; bulk copies
// of 512-byte runs stay below 2 TB/s, and a multistage cp.async ring spent more
// instructions on bookkeeping than it saved.)
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

constexpr int TMT = 4;   // most token slots per pass over the weights
constexpr int NQ = 4;    // warps per 32-row group, each one quarter of the groups along K
constexpr int NT = 32 * 2 * NQ;         // threads per CTA

// Shared-memory layout of one CTA (64 rows; base aligned to 1024 bytes).
struct SmemPlan {
  int xs, sx, xsum, idot, sw, ubuf, rows, total;
};

__host__ __device__ inline SmemPlan smem_plan(int K, int tm, int wg32) {
  SmemPlan p;
  const int G = K / 32;
  int o = 0;
  p.xs = o;
  o += tm * K;
  p.sx = o;
  o += tm * G * 4;
  p.xsum = o;
  o += tm * G * 4;
  p.idot = o;
  o += tm * G * 64 * 4;
  p.sw = o;
  o += wg32 ? G * 64 * 4 : 0;
  p.ubuf = o;
  o += tm * 32 * 4;
  p.rows = o;
  o += 4 * TMT * 4;
  p.total = o + 1024;   // slack for aligning the base to 1024 bytes
  return p;
}

// Token slots per pass: up to TMT, as many as the int32 dot buffer budget allows.
__host__ __device__ inline int pass_tokens(int K, int max_tokens) {
  const int G = K / 32;
  int tm = (32 * 1024) / (G * 64 * 4);
  tm = tm < 1 ? 1 : (tm > TMT ? TMT : tm);
  return max_tokens < tm ? (max_tokens < 1 ? 1 : max_tokens) : tm;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Activation rows of up to tm slots into shared memory (int4 weights: each 8-byte word
// de-interleaved into even / odd elements, plus per-group sums). Threads [0, nthr).
template <int WBITS, bool AG32>
__device__ __forceinline__ void load_acts(const int8_t* __restrict__ qa, const void* sa, int K, int m,
                                          const int* rows, uint8_t* xs, float* sx, int* xsum,
                                          int tid, int nthr) {
  const int G = K / 32;
  const int words = K / 8;
  for (int l = tid; l < m * words; l += nthr) {
    const int tt = l / words, wi = l - tt * words;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(qa + (int64_t)rows[tt] * K) + wi);
    uint2 o = v;
    if (WBITS == 4) deinterleave8(v.x, v.y, o.x, o.y);
    reinterpret_cast<uint2*>(xs + tt * K)[wi] = o;
  }
  for (int l = tid; l < m * G; l += nthr) {
    const int tt = l / G, g = l - tt * G;
    if (AG32) sx[tt * G + g] = __half2float(reinterpret_cast<const __half*>(sa)[(int64_t)rows[tt] * G + g]);
    else if (g == 0) sx[tt] = reinterpret_cast<const float*>(sa)[rows[tt]];
    if (WBITS == 4) {
      const uint4* p = reinterpret_cast<const uint4*>(qa + (int64_t)rows[tt] * K + 32 * g);
      const uint4 a = __ldg(p), b = __ldg(p + 1);
      int s = __dp4a((int)a.x, 0x01010101, 0);
      s = __dp4a((int)a.y, 0x01010101, s);
      s = __dp4a((int)a.z, 0x01010101, s);
      s = __dp4a((int)a.w, 0x01010101, s);
      s = __dp4a((int)b.x, 0x01010101, s);
      s = __dp4a((int)b.y, 0x01010101, s);
      s = __dp4a((int)b.z, 0x01010101, s);
      s = __dp4a((int)b.w, 0x01010101, s);
      xsum[tt * G + g] = s;
    }
  }
}

// The canonical fp32 chain of one row over all groups: acc = fma((float)I_g, c_g, acc) for
// ascending g from +0, then the per-row / per-token scale.
template <bool WG32, bool AG32>
__device__ __forceinline__ float row_chain(const int* idot_t, const float* sw, const float* sx_t, int G,
                                           int row, float sx_tok, float sw_row) {
  if (!WG32 && !AG32) {
    int isum = 0;
    for (int g = 0; g < G; ++g) isum += idot_t[g * 64 + row];
    return __fmul_rn(__fmaf_rn(__int2float_rn(isum), sx_tok, 0.0f), sw_row);
  }
  float acc = 0.0f;
  int g = 0;
  for (; g + 8 <= G; g += 8) {
    int d[8];
    float c[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      d[q] = idot_t[(g + q) * 64 + row];
      if (WG32 && AG32) c[q] = __fmul_rn(sw[(g + q) * 64 + row], sx_t[g + q]);
      else if (WG32) c[q] = sw[(g + q) * 64 + row];
      else c[q] = sx_t[g + q];
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) acc = __fmaf_rn(__int2float_rn(d[q]), c[q], acc);
  }
  for (; g < G; ++g) {
    float c;
    if (WG32 && AG32) c = __fmul_rn(sw[g * 64 + row], sx_t[g]);
    else if (WG32) c = sw[g * 64 + row];
    else c = sx_t[g];
    acc = __fmaf_rn(__int2float_rn(idot_t[g * 64 + row]), c, acc);
  }
  if (WG32 && AG32) return acc;
  if (WG32) return __fmul_rn(acc, sx_tok);
  return __fmul_rn(acc, sw_row);
}

// Resolve grid work unit u (routed units first, then the shared expert's); false if idle.
__device__ __forceinline__ bool unit_of(const ExpertArgs& r, const ExpertArgs& s, int has_shared,
                                        int routed_units, int per_expert_r, int u, bool& shared,
                                        int& e, int& s0, int& s1, int& sub) {
  if (u < routed_units) {
    shared = false;
    const int ai = u / per_expert_r;
    sub = u - ai * per_expert_r;
    const int na = *r.n_active;
    if (ai >= na) return false;
    e = r.act_expert[ai];
    s0 = r.act_begin[ai];
    s1 = r.act_begin[ai + 1];
    if (e < 0 || e >= r.b.E || s0 < 0 || s0 > s1 || s1 > r.T * r.k) {
      if (threadIdx.x == 0) set_status(r.status, kStatusDeviceCheck);
      return false;
    }
    return true;
  }
  if (!has_shared) return false;
  shared = true;
  e = 0;
  s0 = 0;
  s1 = s.T;
  sub = u - routed_units;
  return true;
}

// Up to GB groups of a lane's row from global memory (16-byte pieces; piece p at
// wrow + p * PSTRIDE, group scales at srow[g * SSTRIDE]) -> exact int32 dots against the
// staged token rows, into idot[(tt * G + g) * 64 + row]; scales into sw[g * 64 + row].
// Strides are compile-time so every load uses an immediate offset; full batches with one
// token (the decode case) take a straight-line path.
template <int WBITS, bool WG32, int PSTRIDE, int SSTRIDE>
struct Batch {
  static constexpr int PPG = WBITS == 8 ? 2 : 1;
  static constexpr int GB = WBITS == 8 ? 8 : 16;     // 16 pieces = 16 loads in flight per lane
  uint4 w[PPG * GB];
  float sc[GB];

  __device__ __forceinline__ void load(const uint8_t* __restrict__ wrow, const __half* __restrict__ srow,
                                       int g0, int nb) {
    const uint8_t* wp = wrow + (int64_t)g0 * PPG * PSTRIDE;
    const __half* sp = srow + (int64_t)g0 * SSTRIDE;
    if (nb == GB) {
#pragma unroll
      for (int p = 0; p < PPG * GB; ++p) w[p] = ldg_stream(reinterpret_cast<const uint4*>(wp + p * PSTRIDE));
      if (WG32) {
#pragma unroll
        for (int u = 0; u < GB; ++u) sc[u] = __half2float(sp[u * SSTRIDE]);
      }
    } else {
#pragma unroll
      for (int p = 0; p < PPG * GB; ++p)
        if (p < PPG * nb) w[p] = ldg_stream(reinterpret_cast<const uint4*>(wp + p * PSTRIDE));
      if (WG32) {
#pragma unroll
        for (int u = 0; u < GB; ++u)
          if (u < nb) sc[u] = __half2float(sp[u * SSTRIDE]);
      }
    }
  }

  __device__ __forceinline__ int dot1(int u, const uint8_t* xg, int xs_sum) const {
    const uint4 x0 = *reinterpret_cast<const uint4*>(xg);
    const uint4 x1 = *reinterpret_cast<const uint4*>(xg + 16);
    if (WBITS == 8) return group_dot_i8(w[2 * u], w[2 * u + 1], x0, x1);
    return group_dot_i4(w[u], make_uint4(x0.x, x0.z, x1.x, x1.z), make_uint4(x0.y, x0.w, x1.y, x1.w), xs_sum);
  }

  __device__ __forceinline__ void dots(int g0, int nb, int K, int m, int row, const uint8_t* xs,
                                       const int* xsum, int* idot, float* sw) const {
    const int G = K / 32;
    if (nb == GB && m == 1) {
      const uint8_t* xg = xs + 32 * g0;
      int* id = idot + g0 * 64 + row;
      const int* xsm = xsum + g0;
#pragma unroll
      for (int u = 0; u < GB; ++u) id[u * 64] = dot1(u, xg + 32 * u, WBITS == 4 ? xsm[u] : 0);
      if (WG32) {
#pragma unroll
        for (int u = 0; u < GB; ++u) sw[(g0 + u) * 64 + row] = sc[u];
      }
      return;
    }
    if (WG32) {
#pragma unroll
      for (int u = 0; u < GB; ++u)
        if (u < nb) sw[(g0 + u) * 64 + row] = sc[u];
    }
    for (int tt = 0; tt < m; ++tt) {
      const uint8_t* xg = xs + tt * K + 32 * g0;
      int* id = idot + (tt * G + g0) * 64 + row;
      const int* xsm = xsum + tt * G + g0;
#pragma unroll
      for (int u = 0; u < GB; ++u)
        if (u < nb) id[u * 64] = dot1(u, xg + 32 * u, WBITS == 4 ? xsm[u] : 0);
    }
  }
};

// L2 prefetch of a lane's pieces [p0, p1) (one instruction per piece covers the warp's 512
// contiguous bytes) and, for group-32 scales, groups [g0, g1).
template <int WBITS, bool WG32>
__device__ __forceinline__ void prefetch_rows(const uint8_t* wrow, int pstride, const __half* srow,
                                              int sstride, int g0, int g1) {
  constexpr int PPG = WBITS == 8 ? 2 : 1;
  for (int p = g0 * PPG; p < g1 * PPG; ++p) prefetch_l2(wrow + (int64_t)p * pstride);
  if (WG32)
    for (int g = g0; g < g1; ++g) prefetch_l2(srow + (int64_t)g * sstride);
}

// ------------------------------------------------------------------ gate / up
// CTA = one work unit: one selected expert x 32 intermediate indices = 32 gate rows + the
// matching 32 up rows (routed units first, then the shared expert's). Eight warps: warps
// 0..NQ-1 own the gate rows, NQ..2NQ-1 the up rows (one row per lane), warp quarter q takes
// the q-th quarter of the groups along K. As soon as the unit is known every warp asks L2
// for its whole K range (and for this unit's 1/(I/32) share of the expert's down
// projection, which the next kernel reads), then keeps 16 register loads per lane in flight
// batch by batch; the token rows are staged meanwhile. One warp per (half, token) then runs
// the ordered row chains, and the gate warps apply SwiGLU and quantize h.
template <int WBITS, bool WG32, bool AG32>
__global__ void __launch_bounds__(NT, 2)
    k_gateup_rows(const __grid_constant__ ExpertArgs ra, const __grid_constant__ ExpertArgs sa,
                  int has_shared, int routed_units, int tm) {
  using B = Batch<WBITS, WG32, 256 * 16, 256>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const int K = ra.b.H, G = K / 32, KB = kbytes(K, WBITS);
  const SmemPlan P = smem_plan(K, tm, WG32);
  uint8_t* xs = base + P.xs;
  float* sx = reinterpret_cast<float*>(base + P.sx);
  int* xsum = reinterpret_cast<int*>(base + P.xsum);
  int* idot = reinterpret_cast<int*>(base + P.idot);
  float* swb = reinterpret_cast<float*>(base + P.sw);
  float* ubuf = reinterpret_cast<float*>(base + P.ubuf);
  int* rows = reinterpret_cast<int*>(base + P.rows);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_wait();
  pdl_trigger();
  bool shd;
  int e, s0, s1, ib;
  if (!unit_of(ra, sa, has_shared, routed_units, ra.b.I / 32, blockIdx.x, shd, e, s0, s1, ib)) return;
  const ExpertArgs& a = shd ? sa : ra;
  const int I = a.b.I, IB = I / 32;
  const int64_t blk = (int64_t)e * 2 * I + (int64_t)(ib >> 2) * 256;     // first row of the block
  const int r_gate = (ib & 3) * 32;
  const int half = warp / NQ, q = warp % NQ;
  const int row = half * 32 + lane;
  const int i = ib * 32 + lane;
  const uint8_t* wrow = a.b.gu_w + blk * KB + (int64_t)(half * 128 + r_gate + lane) * 16;
  const __half* srow = reinterpret_cast<const __half*>(a.b.gu_s) + blk * G + half * 128 + r_gate + lane;
  const int GQ = G / NQ, gq0 = q * GQ;

  // ask L2 for everything this warp will read, then for the down slice of this expert
  prefetch_rows<WBITS, WG32>(wrow, 256 * 16, srow, 256, gq0 + B::GB, gq0 + GQ);
  {
    const int64_t dn_bytes = (int64_t)a.b.H * kbytes(I, WBITS);
    const int64_t per = dn_bytes / IB;
    const uint8_t* d0 = a.b.dn_w + (int64_t)e * dn_bytes + (int64_t)ib * per;
    for (int64_t o = (int64_t)threadIdx.x * 128; o < per; o += (int64_t)NT * 128) prefetch_l2(d0 + o);
    if (WG32) {
      const int64_t ds_bytes = (int64_t)a.b.H * (I / 32) * 2;
      const int64_t sper = ds_bytes / IB;
      const uint8_t* s0p = a.b.dn_s + (int64_t)e * ds_bytes + (int64_t)ib * sper;
      for (int64_t o = (int64_t)threadIdx.x * 128; o < sper; o += (int64_t)NT * 128) prefetch_l2(s0p + o);
    }
  }

  for (int c0 = s0; c0 < s1; c0 += tm) {
    const int m = min(tm, s1 - c0);
    B bt;
    bt.load(wrow, srow, gq0, min(B::GB, GQ));      // first batch in flight
    if (threadIdx.x < m) {
      const int slot = c0 + threadIdx.x;
      int r = slot;
      if (!shd) {
        const int p = a.perm[slot];
        const bool okp = p >= 0 && p < a.T * a.k;
        if (!okp) set_status(a.status, kStatusDeviceCheck);
        r = okp ? p / a.k : 0;
      }
      rows[threadIdx.x] = r;
    }
    __syncthreads();
    load_acts<WBITS, AG32>(a.qa, a.sa, K, m, rows, xs, sx, xsum, threadIdx.x, NT);
    __syncthreads();
    for (int g0 = gq0; g0 < gq0 + GQ; g0 += B::GB) {
      const int nb = min(B::GB, gq0 + GQ - g0);
      if (g0 != gq0) bt.load(wrow, srow, g0, nb);
      bt.dots(g0, nb, K, m, row, xs, xsum, idot, swb);
    }
    __syncthreads();
    // row chains: warp w -> (half w / tm, token w % tm)
    float v = 0.0f;
    const int ch_half = warp / tm, ch_tt = warp % tm;
    const bool chain = warp < 2 * tm && ch_tt < m;
    if (chain) {
      const int crow = ch_half * 32 + lane;
      const float swr =
          WG32 ? 0.0f : reinterpret_cast<const float*>(a.b.gu_s)[blk + ch_half * 128 + r_gate + lane];
      v = row_chain<WG32, AG32>(idot + ch_tt * G * 64, swb, sx + ch_tt * G, G, crow, sx[ch_tt], swr);
      if (a.dbg_a) (ch_half == 0 ? a.dbg_a : a.dbg_b)[(int64_t)(c0 + ch_tt) * I + i] = v;
      if (ch_half == 1) ubuf[ch_tt * 32 + lane] = v;
    }
    __syncthreads();
    if (chain && ch_half == 0) {
      const int slot = c0 + ch_tt;
      const float h = cswiglu(v, ubuf[ch_tt * 32 + lane]);
      if (AG32) {
        const float sc = f16_round(__fdiv_rn(warp_max(fabsf(h)), 127.0f));
        a.qh[(int64_t)slot * I + i] = (int8_t)quant_code(h, sc, 127.0f);
        if (lane == 0) a.sh[(int64_t)slot * IB + ib] = __float2half_rn(sc);
      } else {
        a.hbuf[(int64_t)slot * I + i] = h;
      }
    }
    __syncthreads();
  }
}

// -------------------------------------------------------------------- down
// CTA = one selected expert x 64 output rows (two row warps of 32; NQ warps per row warp
// split the groups along K; rows of a piece are contiguous). Same load scheme as gate/up.
// Chains per (row warp, token); the weighted value is added into y with an fp32 atomic.
template <int WBITS, bool WG32, bool AG32>
__global__ void __launch_bounds__(NT, 2)
    k_down_rows(const __grid_constant__ ExpertArgs ra, const __grid_constant__ ExpertArgs sa,
                int has_shared, int routed_units, int tm) {
  using B = Batch<WBITS, WG32, 128 * 16, 128>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const int H = ra.b.H;
  const int Kmax = has_shared && sa.b.I > ra.b.I ? sa.b.I : ra.b.I;
  const SmemPlan P = smem_plan(Kmax, tm, WG32);
  uint8_t* xs = base + P.xs;
  float* sx = reinterpret_cast<float*>(base + P.sx);
  int* xsum = reinterpret_cast<int*>(base + P.xsum);
  int* idot = reinterpret_cast<int*>(base + P.idot);
  float* swb = reinterpret_cast<float*>(base + P.sw);
  int* rows = reinterpret_cast<int*>(base + P.rows);
  int* toks = rows + TMT;
  float* wts = reinterpret_cast<float*>(toks + TMT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_wait();
  pdl_trigger();
  bool shd;
  int e, s0, s1, hb;
  if (!unit_of(ra, sa, has_shared, routed_units, H / 64, blockIdx.x, shd, e, s0, s1, hb)) return;
  const ExpertArgs& a = shd ? sa : ra;
  const int K = a.b.I, G = K / 32, KB = kbytes(K, WBITS);
  const int64_t blk = (int64_t)e * H + (int64_t)(hb >> 1) * 128;
  const int r0 = (hb & 1) * 64;
  const int rw = warp / NQ, q = warp % NQ;
  const int row = rw * 32 + lane;
  const uint8_t* wrow = a.b.dn_w + blk * KB + (int64_t)(r0 + row) * 16;
  const __half* srow = reinterpret_cast<const __half*>(a.b.dn_s) + blk * G + r0 + row;
  const int GQ = G / NQ, gq0 = q * GQ;
  prefetch_rows<WBITS, WG32>(wrow, 128 * 16, srow, 128, gq0 + B::GB, gq0 + GQ);

  for (int c0 = s0; c0 < s1; c0 += tm) {
    const int m = min(tm, s1 - c0);
    B bt;
    bt.load(wrow, srow, gq0, min(B::GB, GQ));
    if (threadIdx.x < m) {
      const int slot = c0 + threadIdx.x;
      rows[threadIdx.x] = slot;
      if (!shd) {
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
    load_acts<WBITS, AG32>(a.qa, a.sa, K, m, rows, xs, sx, xsum, threadIdx.x, NT);
    __syncthreads();
    for (int g0 = gq0; g0 < gq0 + GQ; g0 += B::GB) {
      const int nb = min(B::GB, gq0 + GQ - g0);
      if (g0 != gq0) bt.load(wrow, srow, g0, nb);
      bt.dots(g0, nb, K, m, row, xs, xsum, idot, swb);
    }
    __syncthreads();
    const int ch_rw = warp / tm, ch_tt = warp % tm;
    if (warp < 2 * tm && ch_tt < m) {
      const int crow = ch_rw * 32 + lane;
      const float swr = WG32 ? 0.0f : reinterpret_cast<const float*>(a.b.dn_s)[blk + r0 + crow];
      const float v = row_chain<WG32, AG32>(idot + ch_tt * G * 64, swb, sx + ch_tt * G, G, crow, sx[ch_tt], swr);
      const int n = hb * 64 + crow;
      if (a.dbg_a) a.dbg_a[(int64_t)(c0 + ch_tt) * H + n] = v;
      atomicAdd(a.y + (int64_t)toks[ch_tt] * H + n, wts[ch_tt] * v);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ host side
namespace {

template <int WBITS, bool WG32, bool AG32>
cudaError_t launch_gateup_t(const ExpertArgs& r, const ExpertArgs* s, cudaStream_t st) {
  const int K = r.b.H;
  const int tm = pass_tokens(K, r.T);
  const SmemPlan P = smem_plan(K, tm, WG32);
  static int attr_bytes = 0;
  if (P.total > attr_bytes) {
    const cudaError_t e = cudaFuncSetAttribute(k_gateup_rows<WBITS, WG32, AG32>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, P.total);
    if (e != cudaSuccess) return e;
    attr_bytes = P.total;
  }
  const int routed = r.max_active * (r.b.I / 32);
  const int grid = routed + (s ? s->b.I / 32 : 0);
  return launch_pdl(k_gateup_rows<WBITS, WG32, AG32>, dim3(grid), dim3(NT), (size_t)P.total, st, r,
                    s ? *s : r, s ? 1 : 0, routed, tm);
}

template <int WBITS, bool WG32, bool AG32>
cudaError_t launch_down_t(const ExpertArgs& r, const ExpertArgs* s, cudaStream_t st) {
  const int H = r.b.H;
  const int Kmax = s && s->b.I > r.b.I ? s->b.I : r.b.I;
  const int tm = pass_tokens(Kmax, r.T);
  const SmemPlan P = smem_plan(Kmax, tm, WG32);
  static int attr_bytes = 0;
  if (P.total > attr_bytes) {
    const cudaError_t e = cudaFuncSetAttribute(k_down_rows<WBITS, WG32, AG32>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, P.total);
    if (e != cudaSuccess) return e;
    attr_bytes = P.total;
  }
  const int routed = r.max_active * (H / 64);
  const int grid = routed + (s ? H / 64 : 0);
  return launch_pdl(k_down_rows<WBITS, WG32, AG32>, dim3(grid), dim3(NT), (size_t)P.total, st, r,
                    s ? *s : r, s ? 1 : 0, routed, tm);
}

}  // namespace

#define MOE_DISPATCH_TMA(FN, r, s, st)                                                        \
  ([&]() -> cudaError_t {                                                                     \
    const int sel = ((r).b.wbits == 8 ? 4 : 0) | ((r).b.wg32 ? 2 : 0) | ((r).ag32 ? 1 : 0); \
    switch (sel) {                                                                            \
      case 7: return FN<8, true, true>(r, s, st);                                             \
      case 6: return FN<8, true, false>(r, s, st);                                            \
      case 5: return FN<8, false, true>(r, s, st);                                            \
      case 4: return FN<8, false, false>(r, s, st);                                           \
      case 3: return FN<4, true, true>(r, s, st);                                             \
      case 2: return FN<4, true, false>(r, s, st);                                            \
      case 1: return FN<4, false, true>(r, s, st);                                            \
      default: return FN<4, false, false>(r, s, st);                                          \
    }                                                                                         \
  }())

cudaError_t launch_gateup_tma(const ExpertArgs& r, const ExpertArgs* s, cudaStream_t st) {
  return MOE_DISPATCH_TMA(launch_gateup_t, r, s, st);
}

cudaError_t launch_down_tma(const ExpertArgs& r, const ExpertArgs* s, cudaStream_t st) {
  return MOE_DISPATCH_TMA(launch_down_t, r, s, st);
}

}  // namespace moe
