// router.cu -- router logits, warp-level top-k selection and batch-union grouping.
//
// Router: "DeepSeek-V3-style sigmoid router (noaux_tc, routed_scaling_factor)"
// (GLM-5.2 colibri page, "What's implemented") or softmax top-k ("top-8 of 64
// experts/layer", OLMoE page, "Mixture-of-Experts"). Grouping: "Batch-union MoE:
// in prefill (and MTP verification), each unique expert of the batch is read
// once and applied to every position that routes to it" (GLM page).
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"
#include "topk.cuh"

namespace moe {

// ------------------------------------------------------------------ logits
// Small T: one CTA per (expert, block of TT tokens). Thread c owns 32-element
// chunk c: the expert's 32 weights stay in registers, each token's chunk partial
// is one fma chain; partials are then added in chunk order by one thread per token.
template <int TT>
__global__ void __launch_bounds__(256) k_router_small(const float* __restrict__ x,
                                                      const float* __restrict__ wr, int T, int E,
                                                      int H, float* __restrict__ logits) {
  extern __shared__ float part[];  // [TT][C]
  pdl_wait();
  const int e = blockIdx.x;
  const int t0 = blockIdx.y * TT;
  const int C = H / 32;
  const float* wrow = wr + (int64_t)e * H;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float4 w4[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) w4[v] = __ldg(reinterpret_cast<const float4*>(wrow + 32 * c) + v);
    for (int tt = 0; tt < TT && t0 + tt < T; ++tt) {
      const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)(t0 + tt) * H + 32 * c);
      float acc = 0.0f;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const float4 xv = __ldg(xr + v);
        acc = __fmaf_rn(xv.x, w4[v].x, acc);
        acc = __fmaf_rn(xv.y, w4[v].y, acc);
        acc = __fmaf_rn(xv.z, w4[v].z, acc);
        acc = __fmaf_rn(xv.w, w4[v].w, acc);
      }
      part[tt * C + c] = acc;
    }
  }
  __syncthreads();
  if (threadIdx.x < TT && t0 + (int)threadIdx.x < T) {
    const float* p = part + threadIdx.x * C;
    float total = 0.0f;
    for (int c = 0; c < C; ++c) total = __fadd_rn(total, p[c]);
    logits[(int64_t)(t0 + threadIdx.x) * E + e] = total;
  }
}

// Large T: a TT x 64 (tokens x experts) output tile per CTA, each thread a (TT/16) x 4
// register tile. The K loop walks the 32-element chunks in order; within a chunk every output
// runs its own fma chain from +0, which is then added to the output's running total. The
// next chunk's x and W_r slices are loaded (float4) into registers while the current one is
// computed, then stored into the other shared-memory buffer: one barrier per chunk.
template <int TT>
__global__ void __launch_bounds__(256) k_router_tiled(const float* __restrict__ x,
                                                      const float* __restrict__ wr, int T, int E,
                                                      int H, float* __restrict__ logits) {
  constexpr int RT = TT / 16;                      // token rows per thread
  constexpr int XV = TT * 8 / 256;                 // float4 of x per thread per chunk
  __shared__ __align__(16) float xs[2][32][TT + 4];
  __shared__ __align__(16) float ws[2][32][64 + 4];
  pdl_wait();
  const int tb = blockIdx.y * TT, eb = blockIdx.x * 64;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int C = H / 32;
  float4 xr[XV], wrg[2];
  auto load = [&](int c) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int l = threadIdx.x + 256 * v, rr = l >> 3, k4 = l & 7;
      const int t = tb + rr;
      xr[v] = t < T ? __ldg(reinterpret_cast<const float4*>(x + (int64_t)t * H + 32 * c) + k4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int l = threadIdx.x + 256 * v, rr = l >> 3, k4 = l & 7;
      const int e = eb + rr;
      wrg[v] = e < E ? __ldg(reinterpret_cast<const float4*>(wr + (int64_t)e * H + 32 * c) + k4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int b) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int l = threadIdx.x + 256 * v, rr = l >> 3, k = 4 * (l & 7);
      xs[b][k][rr] = xr[v].x;
      xs[b][k + 1][rr] = xr[v].y;
      xs[b][k + 2][rr] = xr[v].z;
      xs[b][k + 3][rr] = xr[v].w;
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int l = threadIdx.x + 256 * v, rr = l >> 3, k = 4 * (l & 7);
      ws[b][k][rr] = wrg[v].x;
      ws[b][k + 1][rr] = wrg[v].y;
      ws[b][k + 2][rr] = wrg[v].z;
      ws[b][k + 3][rr] = wrg[v].w;
    }
  };
  float total[RT][4];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) total[i][j] = 0.0f;
  load(0);
  store(0);
  __syncthreads();
  for (int c = 0; c < C; ++c) {
    const int b = c & 1;
    if (c + 1 < C) load(c + 1);
    float part[RT][4];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.0f;
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float av[RT];
      if constexpr (RT == 4) {
        const float4 a = *reinterpret_cast<const float4*>(&xs[b][kk][ty * 4]);
        av[0] = a.x;
        av[1] = a.y;
        av[2] = a.z;
        av[3] = a.w;
      } else {
        const float2 a = *reinterpret_cast<const float2*>(&xs[b][kk][ty * 2]);
        av[0] = a.x;
        av[1] = a.y;
      }
      const float4 bw = *reinterpret_cast<const float4*>(&ws[b][kk][tx * 4]);
      const float bv[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = __fmaf_rn(av[i], bv[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) total[i][j] = __fadd_rn(total[i][j], part[i][j]);
    if (c + 1 < C) store(b ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < RT; ++i) {
    const int t = tb + ty * RT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = eb + tx * 4 + j;
      if (e < E) logits[(int64_t)t * E + e] = total[i][j];
    }
  }
}

// The 32-token tile with the K loop split over two warp groups (512 threads): group g takes
// the chunks c = g (mod 2), each with the same thread tile as k_router_tiled, its own double
// buffer and one chunk of loads in flight. After each step (chunks 2s and 2s + 1) group 1 hands
// its chunk partials to group 0 through shared memory, and group 0 adds chunk 2s's partial and
// then chunk 2s + 1's to its running totals: the same chains and the same order of additions,
// with twice the warps per SM to cover the shared-memory load latency.
constexpr int kRouterKsTT = 32;
struct RouterKsSmem {
  float xs[2][2][32][kRouterKsTT + 4];   // [group][buffer][k][token]
  float ws[2][2][32][64 + 4];            // [group][buffer][k][expert]
  float pb[2][256][8];                   // [step parity][group-1 thread][output]
};

__global__ void __launch_bounds__(512) k_router_tiled_ks(const float* __restrict__ x,
                                                         const float* __restrict__ wr, int T,
                                                         int E, int H, float* __restrict__ logits) {
  constexpr int TT = kRouterKsTT, RT = TT / 16, XV = TT * 8 / 256;
  extern __shared__ __align__(16) uint8_t ks_raw[];
  RouterKsSmem& S = *reinterpret_cast<RouterKsSmem*>(ks_raw);
  pdl_wait();
  const int grp = threadIdx.x >> 8, gt = threadIdx.x & 255;
  const int tb = blockIdx.y * TT, eb = blockIdx.x * 64;
  const int ty = gt >> 4, tx = gt & 15;
  const int C = H / 32;
  float4 xr[XV], wrg[2];
  auto load = [&](int c) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int l = gt + 256 * v, rr = l >> 3, k4 = l & 7;
      const int t = tb + rr;
      xr[v] = t < T ? __ldg(reinterpret_cast<const float4*>(x + (int64_t)t * H + 32 * c) + k4)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int l = gt + 256 * v, rr = l >> 3, k4 = l & 7;
      const int e = eb + rr;
      wrg[v] = e < E ? __ldg(reinterpret_cast<const float4*>(wr + (int64_t)e * H + 32 * c) + k4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int b) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int l = gt + 256 * v, rr = l >> 3, k = 4 * (l & 7);
      S.xs[grp][b][k][rr] = xr[v].x;
      S.xs[grp][b][k + 1][rr] = xr[v].y;
      S.xs[grp][b][k + 2][rr] = xr[v].z;
      S.xs[grp][b][k + 3][rr] = xr[v].w;
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int l = gt + 256 * v, rr = l >> 3, k = 4 * (l & 7);
      S.ws[grp][b][k][rr] = wrg[v].x;
      S.ws[grp][b][k + 1][rr] = wrg[v].y;
      S.ws[grp][b][k + 2][rr] = wrg[v].z;
      S.ws[grp][b][k + 3][rr] = wrg[v].w;
    }
  };
  float total[RT][4];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) total[i][j] = 0.0f;
  if (grp < C) {
    load(grp);
    store(0);
  }
  __syncthreads();
  const int steps = (C + 1) / 2;
  for (int s = 0; s < steps; ++s) {
    const int b = s & 1;
    const int c = 2 * s + grp;                 // this group's chunk of the step
    const bool mine = c < C;
    if (c + 2 < C) load(c + 2);
    float part[RT][4];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.0f;
    if (mine) {
#pragma unroll 8
      for (int kk = 0; kk < 32; ++kk) {
        const float2 a = *reinterpret_cast<const float2*>(&S.xs[grp][b][kk][ty * 2]);
        const float av[RT] = {a.x, a.y};
        const float4 bw = *reinterpret_cast<const float4*>(&S.ws[grp][b][kk][tx * 4]);
        const float bv[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[i][j] = __fmaf_rn(av[i], bv[j], part[i][j]);
      }
    }
    if (grp == 1 && mine) {
      float4* pb = reinterpret_cast<float4*>(S.pb[b][gt]);
      pb[0] = make_float4(part[0][0], part[0][1], part[0][2], part[0][3]);
      pb[1] = make_float4(part[1][0], part[1][1], part[1][2], part[1][3]);
    }
    if (c + 2 < C) store(b ^ 1);
    __syncthreads();
    if (grp == 0) {
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) total[i][j] = __fadd_rn(total[i][j], part[i][j]);
      if (2 * s + 1 < C) {
        const float4* pb = reinterpret_cast<const float4*>(S.pb[b][gt]);
        const float4 p0 = pb[0], p1 = pb[1];
        const float q[RT][4] = {{p0.x, p0.y, p0.z, p0.w}, {p1.x, p1.y, p1.z, p1.w}};
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) total[i][j] = __fadd_rn(total[i][j], q[i][j]);
      }
    }
  }
  if (grp != 0) return;
#pragma unroll
  for (int i = 0; i < RT; ++i) {
    const int t = tb + ty * RT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = eb + tx * 4 + j;
      if (e < E) logits[(int64_t)t * E + e] = total[i][j];
    }
  }
}

void launch_router_logits(const float* x, const float* wr, int T, int E, int H, float* logits,
                          cudaStream_t st) {
  if (T <= 0) return;
  if (T <= 32) {
    constexpr int TT = 8;
    const int C = H / 32;
    dim3 grid(E, (T + TT - 1) / TT);
    const int threads = C >= 256 ? 256 : ((C + 31) / 32) * 32;
    launch_pdl(k_router_small<TT>, grid, dim3(threads), TT * C * sizeof(float), st, x, wr, T, E, H,
               logits);
  } else {
    // 32-token tiles when 64-token ones would leave SMs idle
    const int64_t tiles64 = (int64_t)((E + 63) / 64) * ((T + 63) / 64);
    if (tiles64 < 2 * 148) {
      dim3 grid((E + 63) / 64, (T + 31) / 32);
      // the K-split tile (68 KB of shared memory); the plain tile if that cannot be granted
      constexpr int smem = (int)sizeof(RouterKsSmem);
      if (ensure_smem_attr(reinterpret_cast<const void*>(k_router_tiled_ks), smem) == cudaSuccess)
        launch_pdl(k_router_tiled_ks, grid, dim3(512), (size_t)smem, st, x, wr, T, E, H, logits);
      else
        launch_pdl(k_router_tiled<32>, grid, dim3(256), 0, st, x, wr, T, E, H, logits);
    } else {
      dim3 grid((E + 63) / 64, (T + 63) / 64);
      launch_pdl(k_router_tiled<64>, grid, dim3(256), 0, st, x, wr, T, E, H, logits);
    }
  }
}

// ------------------------------------------------------------------- top-k
// One warp per token (warp_topk); for a single token the grouping is written too.
template <int NE>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits,
                                              const float* __restrict__ bias, int T, int E, int k,
                                              int score, int renorm, float rsf, float top_p,
                                              int32_t* __restrict__ idx, float* __restrict__ w,
                                              Grouping g1, int single, int* status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int my_e = warp_topk<NE>(logits + (int64_t)t * E, bias, E, k, score, renorm, rsf, top_p,
                                 idx + (int64_t)t * k, w + (int64_t)t * k, status);
  if (single) {
    // One token: the grouping is the kept selected experts (all k, or the top-p prefix: slots
    // with expert -1 are dropped) in ascending order.
    int rank = 0, nk = 0;
    for (int i = 0; i < k; ++i) {
      const int o = __shfl_sync(0xffffffffu, my_e, i);
      nk += o >= 0;
      rank += (o >= 0) & (o < my_e);
    }
    if (lane < k && my_e >= 0) {
      g1.act_expert[rank] = my_e;
      g1.act_begin[rank] = rank;
      g1.perm[rank] = lane;
    }
    if (lane == 0) {
      g1.act_begin[nk] = nk;
      *g1.n_active = nk;
      g1.offsets[E] = nk;
    }
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int cnt = 0;
      for (int i = 0; i < k; ++i) {
        const int o = __shfl_sync(0xffffffffu, my_e, i);
        cnt += (o >= 0) & (o < e);
      }
      if (e < E) g1.offsets[e] = cnt;
    }
  }
}

void launch_topk(const float* logits, const float* bias, int T, int E, int k, int score,
                 int renorm, float rsf, float top_p, int32_t* idx, float* w, const Grouping* single_token,
                 int* status, cudaStream_t st) {
  if (T <= 0) return;
  const int blocks = (T + 7) / 8;
  Grouping g{};
  if (single_token) g = *single_token;
  const int single = single_token != nullptr;
#define MOE_TOPK_CASE(N)                                                                     \
  launch_pdl(k_topk<N>, dim3(blocks), dim3(256), 0, st, logits, bias, T, E, k, score, renorm, rsf, \
             top_p, idx, w, g, single, status)
  if (E <= 32) MOE_TOPK_CASE(1);
  else if (E <= 64) MOE_TOPK_CASE(2);
  else if (E <= 128) MOE_TOPK_CASE(4);
  else if (E <= 256) MOE_TOPK_CASE(8);
  else if (E <= 512) MOE_TOPK_CASE(16);
  else MOE_TOPK_CASE(32);
#undef MOE_TOPK_CASE
}

// ----------------------------------------------------------------- grouping
// Stable counting sort of the T*k (token, slot) pairs by expert, one CTA.
//   A: per 32-token chunk c, masks[c][e] = bit set of the chunk's tokens routed to e;
//   B: per expert, base[c][e] = pairs of e in chunks before c (the chunks cut into
//      1024 / E parts, summed in parallel, then each part's sums scanned);
//   C: exclusive scan over experts -> offsets, list of distinct experts;
//   D: pos = offsets[e] + base[c][e] + (tokens of the chunk before this one routed to e).
// SM: masks and base live in dynamic shared memory (2 * C * E words) instead of the
// workspace. A token's k slots are read in batches of eight independent loads.
template <bool SM>
__global__ void __launch_bounds__(1024) k_permute(const int32_t* __restrict__ idx, int T, int k,
                                                  int E, int e0, int e_total, Grouping g,
                                                  uint32_t* masks_g, int32_t* base_g, int* status,
                                                  int reset_status) {
  extern __shared__ uint32_t dyn_s[];
  __shared__ int32_t off_s[1024];
  __shared__ int32_t aidx_s[1024];
  __shared__ int32_t psum[1024];            // [part][expert] pair counts
  __shared__ int32_t wsum[32], fsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = (T + 31) / 32;
  uint32_t* masks = SM ? dyn_s : masks_g;
  int32_t* base = SM ? reinterpret_cast<int32_t*>(dyn_s + (int64_t)C * E) : base_g;
  auto ldm = [&](int64_t i) -> uint32_t {
    if constexpr (SM) return masks[i];
    else return __ldcg(masks + i);
  };
  auto ldb = [&](int64_t i) -> int32_t {
    if constexpr (SM) return base[i];
    else return __ldcg(base + i);
  };
  pdl_wait();
  if (reset_status && tid == 0 && status) *status = 0;
  if (SM)
    for (int i = tid; i < C * E; i += 1024) masks[i] = 0u;
  __syncthreads();
  for (int c = warp; c < C; c += 32) {
    uint32_t* mrow = masks + (int64_t)c * E;
    if (!SM) {
      for (int e = lane; e < E; e += 32) mrow[e] = 0u;
      __syncwarp();
    }
    const int t = 32 * c + lane;
    if (t < T) {
      for (int j0 = 0; j0 < k; j0 += 8) {
        int ev[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) ev[u] = j0 + u < k ? __ldg(idx + (int64_t)t * k + j0 + u) : -1;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int eg = ev[u];
          if (eg == -1) continue;            // a slot dropped by adaptive top-p (or past k)
          if (eg < 0 || eg >= e_total) {
            set_status(status, kStatusDeviceCheck);
            continue;
          }
          const int e = eg - e0;             // local id; outside [0, E): held elsewhere
          if (e >= 0 && e < E) atomicOr(&mrow[e], 1u << lane);
        }
      }
    }
  }
  __syncthreads();
  // B: thread (part, e) counts its part's chunks, then writes their bases from the counts of
  //    the parts before it
  const int NP = E >= 1024 ? 1 : 1024 / E;  // parts per expert
  const int per = (C + NP - 1) / NP;         // chunks per part
  const int pe = tid % E, pp = tid / E;
  const int c0 = min(pp * per, C), c1 = min(c0 + per, C);
  if (pp < NP) {
    int cnt = 0;
    for (int c = c0; c < c1; ++c) cnt += __popc(ldm((int64_t)c * E + pe));
    psum[pp * E + pe] = cnt;
  }
  __syncthreads();
  int v = 0;
  if (pp < NP) {
    int run = 0;
    for (int q = 0; q < pp; ++q) run += psum[q * E + pe];
    for (int c = c0; c < c1; ++c) {
      base[(int64_t)c * E + pe] = run;
      run += __popc(ldm((int64_t)c * E + pe));
    }
  }
  if (tid < E)
    for (int q = 0; q < NP; ++q) v += psum[q * E + tid];
  const int f = (tid < E && v > 0) ? 1 : 0;
  int incl = v, inclf = f;
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
  if (warp == 0) {
    int a = wsum[lane], b = fsum[lane];
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, ia, o);
      const int y = __shfl_up_sync(0xffffffffu, ib, o);
      if (lane >= o) {
        ia += x;
        ib += y;
      }
    }
    wsum[lane] = ia - a;
    fsum[lane] = ib - b;
  }
  __syncthreads();
  incl += wsum[warp];
  inclf += fsum[warp];
  if (tid < E) {
    const int excl = incl - v;
    off_s[tid] = excl;
    g.offsets[tid] = excl;
    aidx_s[tid] = inclf - 1;
    if (f) {
      g.act_expert[inclf - 1] = tid;
      g.act_begin[inclf - 1] = excl;
    }
    if (tid == E - 1) {
      g.offsets[E] = incl;
      *g.n_active = inclf;
      g.act_begin[inclf] = incl;
    }
  }
  __syncthreads();
  for (int c = warp; c < C; c += 32) {
    const int t = 32 * c + lane;
    if (t >= T) continue;
    const uint32_t below = (1u << lane) - 1u;
    for (int j0 = 0; j0 < k; j0 += 8) {
      int ev[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ev[u] = j0 + u < k ? __ldg(idx + (int64_t)t * k + j0 + u) : -1;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int eg = ev[u];
        const int e = eg - e0;
        if (eg < 0 || eg >= e_total || e < 0 || e >= E) continue;
        const uint32_t m = ldm((int64_t)c * E + e);
        const int rank = ldb((int64_t)c * E + e) + __popc(m & below);
        g.perm[off_s[e] + rank] = t * k + j0 + u;
        if (g.act_rows && rank < 8) g.act_rows[aidx_s[e] * 8 + rank] = t;
      }
    }
  }
}

// Masks and bases in shared memory up to this many bytes (4096 tokens x 64 experts: 64 KB)
constexpr int64_t kPermuteSmemMax = 160 * 1024;

void launch_permute(const int32_t* idx, int T, int k, int E, int e0, int e_total, const Grouping& g,
                    uint32_t* masks, int32_t* base, int* status, int reset_status, cudaStream_t st) {
  if (T <= 0) return;
  const int64_t smem = 2 * (int64_t)((T + 31) / 32) * E * 4;
  if (smem <= kPermuteSmemMax &&
      ensure_smem_attr(reinterpret_cast<const void*>(k_permute<true>), (int)smem) == cudaSuccess) {
    launch_pdl(k_permute<true>, dim3(1), dim3(1024), (size_t)smem, st, idx, T, k, E, e0, e_total,
               g, masks, base, status, reset_status);
    return;
  }
  launch_pdl(k_permute<false>, dim3(1), dim3(1024), 0, st, idx, T, k, E, e0, e_total, g, masks,
             base, status, reset_status);
}

}  // namespace moe
