// topk.cuh -- warp-level top-k selection and routing weights for one token.
//
// Softmax top-k ("top-8 of 64 experts/layer", OLMoE page, "Mixture-of-Experts") or
// DeepSeek-V3-style sigmoid noaux_tc: key = sigmoid(L) + bias for the selection only,
// weights s / sum_sel(s) * routed_scaling_factor (GLM-5.2 colibri page, "What's
// implemented"). Lane l holds the keys of experts l, l+32, ... (NE per lane); k
// rounds of a warp arg-max pick the largest key, equal keys going to the lower expert.
#pragma once

#include <cfloat>

#include "common.cuh"

namespace moe {

// Lt: the token's logits [E] (read through L2: they may have been written by other CTAs
// of the same grid). Writes idx_out[j], w_out[j] for j < k; returns lane j's expert.
template <int NE>
__device__ __forceinline__ int warp_topk(const float* Lt, const float* __restrict__ bias, int E,
                                         int k, int score, int renorm, float rsf,
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
  float wv;
  if (score == 0) {
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    const float ex = sel ? cexp(my_l - lmax) : 0.0f;
    float den;
    if (renorm) {
      den = warp_sum(ex);
    } else {
      float s = 0.0f;
#pragma unroll
      for (int m = 0; m < NE; ++m)
        if (lane + 32 * m < E) s += cexp(lg[m] - lmax);
      den = warp_sum(s);
    }
    wv = ex / den * rsf;
  } else {
    const float s = sel ? csigmoid(my_l) : 0.0f;
    const float den = renorm ? warp_sum(s) : 1.0f;
    wv = s / den * rsf;
  }
  if (sel) {
    idx_out[lane] = my_e;
    w_out[lane] = wv;
  }
  return my_e;
}

}  // namespace moe
