// route_fused.cu -- everything before the experts, in one launch, for small batches
// (decode, MTP verification: T <= 32 tokens).
//
// Grid = one CTA per expert. Every CTA quantizes a share of the activation groups
// (Q8_0-style, GLM-5.2 colibri page "Integer-dot kernels"), zeroes a share of y and
// computes its expert's router logit for every token in the fixed fp32 chunk order.
// The last CTA to finish (ticket counter) then selects the top-k experts per token
// (warp top-k, topk.cuh) and builds the batch-union grouping ("Batch-union MoE"):
// offsets, the (expert, token)-sorted pair list and the list of distinct experts.
// One launch replaces four dependent ones on the decode critical path.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"
#include "topk.cuh"

namespace moe {

// Largest T*E whose keys the last CTA ranks in shared memory.
constexpr int kRankKeys = 2048;

template <int NE>
__global__ void __launch_bounds__(256, 1) k_route_fused(const __grid_constant__ RouteArgs r) {
  extern __shared__ float part[];                 // [T][C] chunk partials of this expert
  __shared__ uint32_t masks[1024];
  __shared__ int32_t offs[1024];
  __shared__ int32_t aidx[1024];
  __shared__ int32_t sel[32 * 32];
  __shared__ int32_t wsum[8], fsum[8];
  __shared__ float red[8];
  __shared__ float rank_keys[2 * kRankKeys];
  __shared__ int is_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x;
  const int T = r.T, E = r.E, H = r.H, k = r.k;
  const int C = H / 32, G = H / 32;

  pdl_wait();
  pdl_trigger();
  if (e == 0 && tid == 0) {
    r.status[0] = 0;
    r.status[2] = 0;
    r.status[3] = 0;
  }

  // 1. activation quantization
  if (r.ag32) {
    __half* sxh = reinterpret_cast<__half*>(r.sx);
    for (int gi = e * 8 + warp; gi < T * G; gi += E * 8) {
      const int t = gi / G, g = gi - t * G;
      const float v = r.x[(int64_t)t * H + 32 * g + lane];
      const float s = f16_round(__fdiv_rn(warp_max(fabsf(v)), 127.0f));
      r.qx[(int64_t)t * H + 32 * g + lane] = (int8_t)quant_code(v, s, 127.0f);
      if (lane == 0) sxh[(int64_t)t * G + g] = __float2half_rn(s);
    }
  } else {
    for (int t = e; t < T; t += E) {
      const float* xr = r.x + (int64_t)t * H;
      float amax = 0.0f;
      for (int h = tid; h < H; h += 256) amax = fmaxf(amax, fabsf(xr[h]));
      amax = warp_max(amax);
      if (lane == 0) red[warp] = amax;
      __syncthreads();
      const float m8 = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])),
                             fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
      const float s = __fdiv_rn(m8, 127.0f);
      for (int h = tid; h < H; h += 256) r.qx[(int64_t)t * H + h] = (int8_t)quant_code(xr[h], s, 127.0f);
      if (tid == 0) reinterpret_cast<float*>(r.sx)[t] = s;
      __syncthreads();
    }
  }
  // 2. zero y (the expert kernels accumulate into it)
  float4* y4 = reinterpret_cast<float4*>(r.y);
  for (int l = e * 256 + tid; l < T * H / 4; l += E * 256) y4[l] = make_float4(0.f, 0.f, 0.f, 0.f);

  // 3. router logits of expert e: chunk partials (fma chains from +0), then the
  //    partials added in chunk order
  const float* wrow = r.wr + (int64_t)e * H;
  for (int c = tid; c < C; c += 256) {
    float4 w4[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) w4[v] = __ldg(reinterpret_cast<const float4*>(wrow + 32 * c) + v);
    for (int t = 0; t < T; ++t) {
      const float4* xr = reinterpret_cast<const float4*>(r.x + (int64_t)t * H + 32 * c);
      float acc = 0.0f;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const float4 xv = __ldg(xr + v);
        acc = __fmaf_rn(xv.x, w4[v].x, acc);
        acc = __fmaf_rn(xv.y, w4[v].y, acc);
        acc = __fmaf_rn(xv.z, w4[v].z, acc);
        acc = __fmaf_rn(xv.w, w4[v].w, acc);
      }
      part[t * C + c] = acc;
    }
  }
  __syncthreads();
  for (int t = tid; t < T; t += 256) {
    const float* pt = part + t * C;
    float total = 0.0f;
    int c = 0;
    for (; c + 8 <= C; c += 8) {          // loads batched ahead of the in-order adds
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = pt[c + q];
#pragma unroll
      for (int q = 0; q < 8; ++q) total = __fadd_rn(total, v[q]);
    }
    for (; c < C; ++c) total = __fadd_rn(total, pt[c]);
    r.logits[(int64_t)t * E + e] = total;
  }

  // 4. the last CTA to arrive continues
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(r.ticket, 1u) == (unsigned)(E - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // 5. top-k per token
  if ((int64_t)T * E <= kRankKeys && (int64_t)T * E * E <= 256 * 4096) {
    // small problems: every key ranks itself against its token's keys in parallel
    // (rank = keys larger, or equal with a lower expert index: descending, ties low first)
    float* skey = rank_keys;
    float* slog = rank_keys + kRankKeys;
    for (int i = tid; i < T * E; i += 256) {
      const int x = i % E;
      const float L = __ldcg(r.logits + i);
      slog[i] = L;
      skey[i] = r.score == 0 ? L : __fadd_rn(csigmoid(L), r.bias ? r.bias[x] : 0.0f);
    }
    __syncthreads();
    for (int i = tid; i < T * E; i += 256) {
      const int t = i / E, x = i - t * E;
      const float kv = skey[i];
      const float* kt = skey + t * E;
      int rank = 0, j = 0;
      if ((E & 3) == 0) {
        const float4* kt4 = reinterpret_cast<const float4*>(kt);
#pragma unroll 4
        for (; j < E; j += 4) {
          const float4 q = kt4[j >> 2];
          rank += (q.x > kv) | ((q.x == kv) & (j < x));
          rank += (q.y > kv) | ((q.y == kv) & (j + 1 < x));
          rank += (q.z > kv) | ((q.z == kv) & (j + 2 < x));
          rank += (q.w > kv) | ((q.w == kv) & (j + 3 < x));
        }
      }
      for (; j < E; ++j) {
        const float kj = kt[j];
        rank += (kj > kv) | ((kj == kv) & (j < x));
      }
      if (rank < k) sel[t * k + rank] = x;
    }
    __syncthreads();
    for (int t = warp; t < T; t += 8) {
      const bool on = lane < k;
      int my_e = on ? sel[t * k + lane] : 0;
      const float myl = slog[t * E + my_e];
      float v, den;                      // slot mass, weight denominator (as topk.cuh)
      if (r.score == 0) {
        const float lmax = __shfl_sync(0xffffffffu, myl, 0);
        v = on ? cexp(myl - lmax) : 0.0f;
        if (r.renorm) {
          den = warp_sum(v);
        } else {
          float sacc = 0.0f;
          for (int x = lane; x < E; x += 32) sacc += cexp(slog[t * E + x] - lmax);
          den = warp_sum(sacc);
        }
      } else {
        v = on ? csigmoid(myl) : 0.0f;
        den = r.renorm ? warp_sum(v) : 1.0f;
      }
      float wv = v / den * r.rsf;
      if (r.top_p > 0.0f) {
        float cm;
        const int m = topp_keep(v, k, r.top_p, cm);
        if (lane >= m) {
          my_e = -1;
          wv = 0.0f;
        } else if (r.renorm) {
          wv = v / cm * r.rsf;
        }
      }
      if (on) {
        sel[t * k + lane] = my_e;
        r.idx[(int64_t)t * k + lane] = my_e;
        r.w[(int64_t)t * k + lane] = wv;
      }
    }
  } else {
    // one warp per token
    for (int t = warp; t < T; t += 8) {
      const int my_e = warp_topk<NE>(r.logits + (int64_t)t * E, r.bias, E, k, r.score, r.renorm,
                                     r.rsf, r.top_p, r.idx + (int64_t)t * k, r.w + (int64_t)t * k,
                                     r.status);
      if (lane < k) sel[t * k + lane] = my_e;
    }
  }
  __syncthreads();
  // expert parallelism: the grouping keeps the pairs whose expert is held here (global ids
  // e0 .. e0 + EL - 1), by local id; the idx / w views keep the global selection
  const int EL = r.EL;
  if (r.e0 != 0 || EL != E) {
    for (int p = tid; p < T * k; p += 256) {
      const int ee = sel[p];
      sel[p] = (ee >= r.e0 && ee < r.e0 + EL) ? ee - r.e0 : -1;
    }
    __syncthreads();
  }
  if (T == 1) {
    // one token: the active experts are its kept selections (all k, or the adaptive top-p
    // prefix; dropped slots hold -1), one slot each, in ascending expert order
    int nk = 0;
    for (int j = 0; j < k; ++j) nk += sel[j] >= 0;
    if (tid < k) {
      const int ee = sel[tid];
      int pos = 0;
      for (int j = 0; j < k; ++j) pos += (sel[j] >= 0) & (sel[j] < ee);
      if (ee >= 0 && ee < EL) {
        r.g.act_expert[pos] = ee;
        r.g.act_begin[pos] = pos;
        r.g.perm[pos] = tid;
        if (r.g.act_rows) r.g.act_rows[pos * 8] = 0;
      }
    }
    for (int x = tid; x < EL; x += 256) {
      int cnt = 0;
      for (int j = 0; j < k; ++j) cnt += (sel[j] >= 0) & (sel[j] < x);
      r.g.offsets[x] = cnt;
    }
    if (tid == 0) {
      r.g.offsets[EL] = nk;
      *r.g.n_active = nk;
      r.g.act_begin[nk] = nk;
      *r.ticket = 0u;
    }
    return;
  }
  for (int x = tid; x < EL; x += 256) masks[x] = 0u;
  __syncthreads();

  // 6. grouping: bit t of masks[e] = token t routes to e; pairs sorted by (expert, token)
  for (int p = tid; p < T * k; p += 256) {
    const int ee = sel[p];
    if (ee >= 0 && ee < EL) atomicOr(&masks[ee], 1u << (p / k));
  }
  __syncthreads();
  const int per = (EL + 255) / 256;
  const int lo = min(tid * per, EL), hi = min(lo + per, EL);
  int cnt = 0, nf = 0;
  for (int x = lo; x < hi; ++x) {
    const int c = __popc(masks[x]);
    cnt += c;
    nf += c > 0;
  }
  int incl = cnt, inclf = nf;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, incl, o);
    const int b = __shfl_up_sync(0xffffffffu, inclf, o);
    if (lane >= o) {
      incl += a;
      inclf += b;
    }
  }
  if (lane == 31) {
    wsum[warp] = incl;
    fsum[warp] = inclf;
  }
  __syncthreads();
  int base = 0, fbase = 0, total = 0, ftotal = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) {
      base += wsum[w];
      fbase += fsum[w];
    }
    total += wsum[w];
    ftotal += fsum[w];
  }
  int run = base + incl - cnt, frun = fbase + inclf - nf;
  for (int x = lo; x < hi; ++x) {
    const int c = __popc(masks[x]);
    offs[x] = run;
    r.g.offsets[x] = run;
    aidx[x] = frun;
    if (c > 0) {
      r.g.act_expert[frun] = x;
      r.g.act_begin[frun] = run;
      ++frun;
    }
    run += c;
  }
  if (tid == 0) {
    r.g.offsets[EL] = total;
    *r.g.n_active = ftotal;
    r.g.act_begin[ftotal] = total;
  }
  __syncthreads();
  for (int p = tid; p < T * k; p += 256) {
    const int ee = sel[p];
    if (ee < 0 || ee >= EL) continue;
    const int t = p / k;
    const int rank = __popc(masks[ee] & ((1u << t) - 1u));
    r.g.perm[offs[ee] + rank] = p;
    if (r.g.act_rows && rank < 8) r.g.act_rows[aidx[ee] * 8 + rank] = t;
  }
  if (tid == 0) *r.ticket = 0u;
}

cudaError_t launch_route_fused(const RouteArgs& r, cudaStream_t st) {
  const size_t smem = (size_t)r.T * (r.H / 32) * sizeof(float);
  int E = r.E;
#define MOE_ROUTE_CASE(N)                                                                  \
  do {                                                                                     \
    if (smem > 48 * 1024) {                                                                \
      const cudaError_t e = ensure_smem_attr((const void*)k_route_fused<N>, (int)smem);    \
      if (e != cudaSuccess) return e;                                                      \
    }                                                                                      \
    return launch_pdl(k_route_fused<N>, dim3(E), dim3(256), smem, st, r);                              \
  } while (0)
  if (E <= 32) MOE_ROUTE_CASE(1);
  if (E <= 64) MOE_ROUTE_CASE(2);
  if (E <= 128) MOE_ROUTE_CASE(4);
  if (E <= 256) MOE_ROUTE_CASE(8);
  if (E <= 512) MOE_ROUTE_CASE(16);
  MOE_ROUTE_CASE(32);
#undef MOE_ROUTE_CASE
}

}  // namespace moe
