// topk.cuh -- warp-level top-k selection and routing weights for one token.
//
// Softmax top-k ("top-8 of 64 experts/layer", OLMoE page, "Mixture-of-Experts") or
// DeepSeek-V3-style sigmoid noaux_tc: key = sigmoid(L) + bias for the selection only,
// weights s / sum_sel(s) * routed_scaling_factor (GLM-5.2 colibri page, "What's
// implemented"). Lane l holds the keys of experts l, l+32, ... (NE per lane); k
// rounds of a warp arg-max pick the largest key, equal keys going to the lower expert.
//
// Adaptive expert top-p (the colibri page's "--topp" knob): a token keeps only the shortest
// prefix of its top-k list whose share of the list's mass reaches top_p (topp_keep).
#pragma once

#include <cfloat>

#include "common.cuh"

namespace moe {

// Adaptive top-p cut, called by every lane of a warp in which lane j < k holds the mass v of
// slot j of a token's top-k list (v = exp(L_j - L_0) for softmax, sigmoid(L_j) for the sigmoid
// router; lanes >= k pass anything). Every lane runs the same fp32 sums in slot order:
// D = v_0 + ... + v_{k-1}, C_m = v_0 + ... + v_{m-1}; the result is the first m with
// C_m >= top_p * D (k if none), and cm = C_m, the kept mass (the renormalized weights' sum).
__device__ __forceinline__ int topp_keep(float v, int k, float top_p, float& cm) {
  float d = 0.0f;
  for (int j = 0; j < k; ++j) d = __fadd_rn(d, __shfl_sync(0xffffffffu, v, j));
  const float thr = __fmul_rn(top_p, d);
  float c = 0.0f;
  int m = k;
  for (int j = 0; j < k; ++j) {
    c = __fadd_rn(c, __shfl_sync(0xffffffffu, v, j));
    if (c >= thr) {                          // the same on every lane
      m = j + 1;
      break;
    }
  }
  cm = c;
  return m;
}

// Lt: the token's logits [E] (read through L2: they may have been written by other CTAs
// of the same grid). Writes idx_out[j], w_out[j] for j < k; returns lane j's expert (-1 for a
// slot that adaptive top-p drops: top_p in (0, 1), else 0 = off).
template <int NE>
__device__ __forceinline__ int warp_topk(const float* Lt, const float* __restrict__ bias, int E,
                                         int k, int score, int renorm, float rsf, float top_p,
                                         int32_t* idx_out, float* w_out, int* status) {
  const int lane = threadIdx.x & 31;
  float key[NE], lg[NE];
#pragma unroll
  for (int m = 0; m < NE; ++m) {
    const int e = lane + 32 * m;
    lg[m] = e < E ? __ldcg(Lt + e) : 0.0f;
    if (e >= E) key[m] = -FLT_MAX;
    else if (score == 0) key[m] = lg[m];
    else key[m] = __fadd_rn(csigmoid(lg[m]), bias ? bias[e] : 0.0f);
  }
  uint32_t taken = 0;
  int my_e = 0;
  float my_l = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bk = -FLT_MAX, bl = 0.0f;
    int be = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < NE; ++m) {
      const int e = lane + 32 * m;
      if (e < E && !((taken >> m) & 1u) && (key[m] > bk || be == 0x7fffffff)) {
        bk = key[m];
        be = e;
        bl = lg[m];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
        bl = ol;
      }
    }
    if (be < E && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_e = be;
      my_l = bl;
    }
  }
  const bool sel = lane < k;
  if (sel && (my_e < 0 || my_e >= E)) set_status(status, kStatusDeviceCheck);
  float v, den;                            // slot mass, weight denominator
  if (score == 0) {
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    v = sel ? cexp(my_l - lmax) : 0.0f;
    if (renorm) {
      den = warp_sum(v);
    } else {
      float s = 0.0f;
#pragma unroll
      for (int m = 0; m < NE; ++m)
        if (lane + 32 * m < E) s += cexp(lg[m] - lmax);
      den = warp_sum(s);
    }
  } else {
    v = sel ? csigmoid(my_l) : 0.0f;
    den = renorm ? warp_sum(v) : 1.0f;
  }
  float wv = v / den * rsf;
  if (top_p > 0.0f) {
    float cm;
    const int m = topp_keep(v, k, top_p, cm);
    if (lane >= m) {
      my_e = -1;
      wv = 0.0f;
    } else if (renorm) {
      wv = v / cm * rsf;
    }
  }
  if (sel) {
    idx_out[lane] = my_e;
    w_out[lane] = wv;
  }
  return my_e;
}

}  // namespace moe
