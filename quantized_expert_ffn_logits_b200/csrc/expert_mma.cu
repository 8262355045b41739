// expert_mma.cu -- tensor-core path for experts with many tokens (prefill, large batches).
//
// An expert that receives at least kMmaMinTokens (token, expert) pairs in a call is a dense
// contraction: its pairs are cut into tiles of 128 slots and every (tile, 128-row weight
// block) pair runs as an M = 128 (slots) x N = 128 (rows) GEMM on the sm_100a tensor cores.
// The codes enter as fp16 (exact: they are integers of at most 8 bits) and two tcgen05.mma
// kind::f16 with K = 16 and an fp32 accumulator cover one quantization group of 32: every
// product is an integer below 2^14 and every partial sum below 2^19, so the accumulator holds
// the exact group dot I_g as an fp32 value -- no integer-to-float step is left. The epilogue
// runs the ordered fp32 chain acc = fma((float)I_g, c_g, acc) with c_g = s_w,g * s_x,g per
// element, the same arithmetic as the weight-streaming path and the oracle (GLM-5.2 colibri
// page, "Integer-dot kernels"; "Batch-union MoE": every selected expert's weights are read once
// per tile of 128 of its tokens).
//
// Gate/up tiles (N = the 64 gate rows and 64 up rows of one block) end with SwiGLU and Q8_0
// h quantization per group of 32 -- one thread holds a slot's 32 indices of a group -- and
// write h (as fp16 codes) in the operand layout the down GEMM reads; down tiles (N = 128
// output rows) add w * v into y with 16-byte reductions.
//
// The per-group epilogue (two fp32 operations per element per group against one 32-wide
// step of the tensor cores) bounds this path, not the tensor cores: see the measurement notes.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace moe {

// -------------------------------------------------------------------- tile plan
// tiles[i] = {active expert index (-1: the shared expert), first slot, valid slots, expert}.
// Routed experts with at least min_tokens slots, in active order, then the shared expert's
// tokens (when has_shared and T >= min_tokens). One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) k_mma_plan(const int32_t* __restrict__ n_active,
                                                   const int32_t* __restrict__ act_expert,
                                                   const int32_t* __restrict__ act_begin, int E, int T,
                                                   int has_shared, int min_tokens, int max_tiles,
                                                   int4* __restrict__ tiles, int32_t* __restrict__ n_tiles,
                                                   int* status) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  const int na = min(*n_active, E);
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < na; base += 1024) {
    const int ai = base + tid;
    int cnt = 0, s0 = 0, n = 0, e = 0;
    if (ai < na) {
      s0 = act_begin[ai];
      n = act_begin[ai + 1] - s0;
      e = act_expert[ai];
      if (n >= min_tokens) cnt = (n + 127) / 128;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = wsum[lane];
      int iv = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, iv, o);
        if (lane >= o) iv += x;
      }
      wsum[lane] = iv - v;
    }
    __syncthreads();
    const int first = carry + wsum[warp] + incl - cnt;
    for (int j = 0; j < cnt; ++j) {
      if (first + j >= max_tiles) {
        set_status(status, kStatusDeviceCheck);
        break;
      }
      tiles[first + j] = make_int4(ai, s0 + 128 * j, min(128, n - 128 * j), e);
    }
    __syncthreads();
    if (tid == 1023) carry = first + cnt;
    __syncthreads();
  }
  if (tid == 0) {
    int total = carry;
    if (has_shared && T >= min_tokens)
      for (int s0 = 0; s0 < T; s0 += 128) {
        if (total >= max_tiles) {
          set_status(status, kStatusDeviceCheck);
          break;
        }
        tiles[total++] = make_int4(-1, s0, min(128, T - s0), 0);
      }
    *n_tiles = min(total, max_tiles);
  }
}

// Four signed int8 codes -> four exact fp16 values (two words): the bytes x ^ 0x80 = x + 128
// become the low mantissa bytes of fp16 1024 + (x + 128), then 1152 is subtracted (exact).
__device__ __forceinline__ void cvt_i8x4_f16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  const uint32_t x = w ^ 0x80808080u;
  uint32_t h0 = __byte_perm(x, 0x64646464u, 0x5140), h1 = __byte_perm(x, 0x64646464u, 0x7362);
  const __half2 k = __halves2half2(__float2half_rn(1152.0f), __float2half_rn(1152.0f));
  __half2 r0 = __hsub2(*reinterpret_cast<__half2*>(&h0), k), r1 = __hsub2(*reinterpret_cast<__half2*>(&h1), k);
  o0 = *reinterpret_cast<uint32_t*>(&r0);
  o1 = *reinterpret_cast<uint32_t*>(&r1);
}
// Four bytes holding v = n + BIAS (n a signed code: BIAS 8 for 4-bit, 2 for 2-bit codes) ->
// the four fp16 values n: the bytes become the low mantissa bytes of fp16 1024 + v, then
// 1024 + BIAS is subtracted (exact).
template <int BIAS = 8>
__device__ __forceinline__ void cvt_u4x4_f16(uint32_t v, uint32_t& o0, uint32_t& o1) {
  uint32_t h0 = __byte_perm(v, 0x64646464u, 0x5140), h1 = __byte_perm(v, 0x64646464u, 0x7362);
  const __half2 k = __halves2half2(__float2half_rn(1024.0f + BIAS), __float2half_rn(1024.0f + BIAS));
  __half2 r0 = __hsub2(*reinterpret_cast<__half2*>(&h0), k), r1 = __hsub2(*reinterpret_cast<__half2*>(&h1), k);
  o0 = *reinterpret_cast<uint32_t*>(&r0);
  o1 = *reinterpret_cast<uint32_t*>(&r1);
}

// -------------------------------------------------------------------- gather
// Operand A of the gate/up GEMM: for tile i, the q_x rows of its slots' tokens as fp16 (exact:
// the codes are integers) in the tensor-core operand layout [tile][K/8 pieces][128 slots][16 B],
// and their fp16 group scales [tile][K/32][128]; slots past the tile's valid count are zero.
// One thread per (tile, slot, group).
__global__ void __launch_bounds__(256) k_mma_gather(const int8_t* __restrict__ qx, const __half* __restrict__ sx,
                                                    const int4* __restrict__ tiles,
                                                    const int32_t* __restrict__ n_tiles,
                                                    const int32_t* __restrict__ perm, int k, int T, int K,
                                                    uint8_t* __restrict__ xa, __half* __restrict__ xs, int* status) {
  pdl_wait();
  const int G = K / 32;
  const int nt = *n_tiles;
  const int64_t per_tile = (int64_t)128 * G;
  for (int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; id < (int64_t)nt * per_tile;
       id += (int64_t)gridDim.x * blockDim.x) {
    const int ti = (int)(id / per_tile);
    const int rem = (int)(id - (int64_t)ti * per_tile);
    const int g = rem >> 7, t = rem & 127;
    const int4 tl = tiles[ti];
    uint4 o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) o[u] = make_uint4(0, 0, 0, 0);
    __half s = __float2half_rn(0.0f);
    if (t < tl.z) {
      const int slot = tl.y + t;
      int tok = slot;
      if (tl.x >= 0) {
        const int pr = perm[slot];
        tok = (pr >= 0 && pr < T * k) ? pr / k : -1;
      }
      if (tok >= 0 && tok < T) {
        const uint4* src = reinterpret_cast<const uint4*>(qx + (int64_t)tok * K + 32 * g);
        const uint4 v0 = src[0], v1 = src[1];
        cvt_i8x4_f16(v0.x, o[0].x, o[0].y);
        cvt_i8x4_f16(v0.y, o[0].z, o[0].w);
        cvt_i8x4_f16(v0.z, o[1].x, o[1].y);
        cvt_i8x4_f16(v0.w, o[1].z, o[1].w);
        cvt_i8x4_f16(v1.x, o[2].x, o[2].y);
        cvt_i8x4_f16(v1.y, o[2].z, o[2].w);
        cvt_i8x4_f16(v1.z, o[3].x, o[3].y);
        cvt_i8x4_f16(v1.w, o[3].z, o[3].w);
        s = sx[(int64_t)tok * G + g];
      } else if (g == 0) {
        set_status(status, kStatusDeviceCheck);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(xa) + ((int64_t)ti * 4 * G + 4 * g) * 128 + t;
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[u * 128] = o[u];
    xs[((int64_t)ti * G + g) * 128 + t] = s;
  }
}

// -------------------------------------------------------------------- GEMM kernel
constexpr int kMmaKC = 2;                  // quantization groups per pipeline stage
// Pipeline stages: a stage's way from the producer's copy to its release by the last epilogue
// warp (copy ~0.8 us, weight prep ~0.6 us, MMA hand-off, epilogue, the warps' skew) spans
// about four stage periods, so five stages (218 KB of shared memory) keep the copies ahead.
constexpr int kMmaNS = 5;
constexpr int kMmaNB = 4;                  // tensor-memory accumulators (128 fp32 columns each:
                                           // all 512; one CTA per SM), so MMAs run 4 groups ahead
constexpr int kMmaPrepWarps = 2;
// The roles that run ahead (producer, MMA issuer, prep) wait with try_wait's suspend hint: the
// thread wakes when the phase completes (measured: 1-2 % faster than polling with sleeps, which
// added up to a sleep period to every hand-off of the stage chain).
__device__ __forceinline__ bool mma_wait_ahead(uint64_t* bar, uint32_t parity) {
  return mbar_wait(bar, parity);
}
// One accumulator hand-off per 2-group stage: the MMA issuer fills a pair of accumulators
// (groups 2i, 2i + 1) and commits once; the epilogue waits once, drains both, releases once.
constexpr bool kMmaPairCommit = true;
// Weight blocks are re-read by every tile of their expert: normal L2 policy, not evict-first
// (measured: the same time either way at 4096 tokens).
constexpr bool kMmaWeightsEvictFirst = false;
constexpr int kMmaEpiWarps = 16;
constexpr int kMmaEpi0 = 2 + kMmaPrepWarps;                       // first epilogue warp
constexpr int kMmaThreads = (kMmaEpi0 + kMmaEpiWarps) * 32;       // producer, MMA, prep, epilogue

// One pipeline stage (two groups): operand A (the 128 slots' codes, already fp16 in the
// workspace), operand B as copied (the int8 or packed int4 codes of 128 weight rows) and as
// fp16 for the tensor cores, the fp16 scales of both and B's as fp32. Operand layout: K-major
// canonical without swizzle, [16-byte piece along K][128 rows][16 B].
struct MmaStage {
  static constexpr int AH = 0;             // [8 pieces][128][16] fp16
  static constexpr int BH = 16384;         // [8 pieces][128][16] fp16
  static constexpr int B8 = 32768;         // [4 pieces][128][16] int8 (int4: 2 pieces)
  static constexpr int AS = 40960;         // [2][128] fp16
  static constexpr int BS = 41472;         // [2][128] fp16
  static constexpr int BSF = 41984;        // [2][128] fp32
  static constexpr int BYTES = 43008;      // a multiple of 1024
};
// the stages, barriers (256 B), the h exchange (2 KB), 1 KB for aligning the base
constexpr int kMmaSmem = kMmaNS * MmaStage::BYTES + 256 + 2048 + 1024;
static_assert(kMmaSmem <= 227 * 1024, "shared memory per CTA");
static_assert((3 * kMmaNS + 2 * kMmaNB) * 8 + 8 <= 256, "barriers, tensor-memory slot, abort flag");

// Stage bytes the producer copies (A codes and scales, B codes and scales).
template <int WBITS>
__device__ __forceinline__ uint32_t mma_stage_bytes() {
  return 16384u + 512u + 1024u * WBITS + 512u;   // B: 2 groups x 128 rows x 32 codes
}

template <int WBITS, bool GATEUP>
__global__ void __launch_bounds__(kMmaThreads, 1) k_expert_mma(const __grid_constant__ MmaArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kMmaNS * MmaStage::BYTES);
  uint64_t* prep = full + kMmaNS;
  uint64_t* empty = prep + kMmaNS;
  uint64_t* acc_full = empty + kMmaNS;
  uint64_t* acc_empty = acc_full + kMmaNB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + kMmaNB);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* xchg = reinterpret_cast<int*>(base + kMmaNS * MmaStage::BYTES + 256);   // [2][2][128] h amax
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int PPU = WBITS / 2;           // 16-byte pieces of a 64-column down slab row
  constexpr int kKern = GATEUP ? 3 : 4;
  static_assert(kMmaKC == 2, "a stage is one 64-column down slab");

  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < kMmaNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&prep[s], kMmaPrepWarps);
      mbar_init(&empty[s], 1 + kMmaEpiWarps);
    }
    for (int b = 0; b < kMmaNB; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kMmaEpiWarps);
    }
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 2 * 2 * 128; i += kMmaThreads) xchg[i] = 0;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMmaNB * 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const BlobView& b0 = A.b[0];
  const int H = b0.H;
  const int nt = min(*A.n_tiles, A.max_tiles);
  // items = (tile, block): gate/up blocks of 64 intermediate indices, down blocks of 128 rows
  const int I_r = b0.I, I_s = A.b[1].I;
  const int per_r = GATEUP ? I_r / 64 : H / 128;
  const int per_s = GATEUP ? I_s / 64 : H / 128;
  const int per = max(per_r, per_s);        // items per tile (slots of a shorter tile idle)
  const int n_items = nt * per;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t c = 0;
      bool ok = true;
      const uint64_t once = policy_evict_first();
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int ti = it / per, blkn = it - ti * per;
        const int4 tl = A.tiles[ti];
        const int sh = tl.x < 0;
        const BlobView& bv = A.b[sh];
        if (blkn >= (sh ? per_s : per_r)) continue;
        const int K = GATEUP ? H : bv.I;
        const int G = K / 32, KB = kbytes(K, WBITS);
        const uint8_t* a_src = GATEUP ? A.a_ops + (int64_t)ti * 128 * K * 2 : A.h_ops + (int64_t)ti * 128 * A.hk * 2;
        const __half* as_src = GATEUP ? A.a_scales + (int64_t)ti * G * 128 : A.h_scales + (int64_t)ti * (A.hk / 32) * 128;
        for (int g0 = 0; g0 < G && ok; g0 += kMmaKC, ++c) {
          const int s = c % kMmaNS;
          if (c >= (uint32_t)kMmaNS && !mma_wait_ahead(&empty[s], ((c / kMmaNS) - 1) & 1)) {
            wait_failed(A.status, kKern, 0, s);
            ok = false;
            break;
          }
          uint8_t* st = base + s * MmaStage::BYTES;
          mbar_arrive_expect_tx(&full[s], mma_stage_bytes<WBITS>());
          bulk_load(st + MmaStage::AH, a_src + (int64_t)g0 * 4 * 2048, 16384, &full[s]);
          bulk_load(st + MmaStage::AS, as_src + (int64_t)g0 * 128, 512, &full[s]);
          auto load_w = [&](void* dst, const void* src, uint32_t bytes) {
            if (kMmaWeightsEvictFirst) bulk_load_hint(dst, src, bytes, &full[s], once);
            else bulk_load(dst, src, bytes, &full[s]);
          };
          if (GATEUP) {
            const int64_t blk = (int64_t)tl.w * 2 * bv.I + (int64_t)blkn * 128;
            // the stage's 2 groups: code bytes 4 WBITS g0 .. of each row = pieces WBITS g0 / 4 ..
            load_w(st + MmaStage::B8, bv.gu_w + blk * KB + (int64_t)g0 * WBITS / 4 * 2048, 1024u * WBITS);
            load_w(st + MmaStage::BS, bv.gu_s + (blk * G + (int64_t)g0 * 128) * 2, 512);
          } else {
            const int U = bv.I / 64, HB = bv.H / 128;
            const int64_t slab = ((int64_t)tl.w * U + g0 / 2) * HB + blkn;
            load_w(st + MmaStage::B8, bv.dn_w + slab * PPU * 2048, PPU * 2048);
            load_w(st + MmaStage::BS, bv.dn_s + slab * 512, 512);
          }
        }
      }
      // drain the copies still in flight before the CTA may exit
      const uint32_t c0 = c > (uint32_t)kMmaNS ? c - kMmaNS : 0;
      for (uint32_t d = c0; d < c; ++d)
        if (!mbar_wait(&full[d % kMmaNS], (d / kMmaNS) & 1)) {
          wait_failed(A.status, kKern, 2, d % kMmaNS);
          break;
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      uint32_t c = 0, gi = 0;
      constexpr uint32_t idesc = idesc_f16(128, 128);
      for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int ti = it / per, blkn = it - ti * per;
        const int4 tl = A.tiles[ti];
        const int sh = tl.x < 0;
        if (blkn >= (sh ? per_s : per_r)) continue;
        const int K = GATEUP ? H : A.b[sh].I;
        const int G = K / 32;
        for (int g0 = 0; g0 < G; g0 += kMmaKC, ++c) {
          const int s = c % kMmaNS;
          bool ok = *abort == 0;
          if (ok && !mma_wait_ahead(&prep[s], (c / kMmaNS) & 1)) {
            *abort = 1;
            wait_failed(A.status, kKern, 1, s);
            ok = false;
          }
          tc_fence_after();
          const uint8_t* st = base + s * MmaStage::BYTES;
          if constexpr (kMmaPairCommit) {
            // the stage's two groups into accumulator pair pr (buffers 2 pr, 2 pr + 1)
            const uint32_t pr = c & 1;
            if (ok && c >= 2 && !mma_wait_ahead(&acc_empty[pr], ((c >> 1) - 1) & 1)) {
              *abort = 1;
              wait_failed(A.status, kKern, 3, pr);
              ok = false;
            }
            tc_fence_after();
            if (ok)
              for (int j = 0; j < kMmaKC; ++j) {
                const uint8_t* a = st + MmaStage::AH + j * 8192;
                const uint8_t* b = st + MmaStage::BH + j * 8192;
                const uint32_t d = tmem + (2 * pr + j) * 128;
                mma_f16(d, smem_desc(a, 2048, 128), smem_desc(b, 2048, 128), idesc, 0);
                mma_f16(d, smem_desc(a + 4096, 2048, 128), smem_desc(b + 4096, 2048, 128), idesc, 1);
              }
            mma_commit(&acc_full[pr]);           // arrives (in order) even when skipped
            gi += kMmaKC;
          } else {
            for (int j = 0; j < kMmaKC; ++j, ++gi) {
              const int bb = gi % kMmaNB;
              if (ok && gi >= (uint32_t)kMmaNB && !mma_wait_ahead(&acc_empty[bb], ((gi / kMmaNB) - 1) & 1)) {
                *abort = 1;
                wait_failed(A.status, kKern, 3, bb);
                ok = false;
              }
              tc_fence_after();
              if (ok) {
                // group j: fp16 pieces 4j .. 4j + 3, two MMAs of K = 16 (exact integer dot)
                const uint8_t* a = st + MmaStage::AH + j * 8192;
                const uint8_t* b = st + MmaStage::BH + j * 8192;
                mma_f16(tmem + bb * 128, smem_desc(a, 2048, 128), smem_desc(b, 2048, 128), idesc, 0);
                mma_f16(tmem + bb * 128, smem_desc(a + 4096, 2048, 128), smem_desc(b + 4096, 2048, 128), idesc, 1);
              }
              mma_commit(&acc_full[bb]);         // arrives (in order) even when skipped
            }
          }
          mma_commit(&empty[s]);
        }
      }
    }
  } else if (warp < kMmaEpi0) {
    // ---------------------------------------------------------------- prep: weight codes -> fp16, scales
    uint32_t c = 0;
    const int pt = threadIdx.x - 64;        // [0, 32 * kMmaPrepWarps)
    constexpr int NPT = 32 * kMmaPrepWarps;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      const int ti = it / per, blkn = it - ti * per;
      const int4 tl = A.tiles[ti];
      const int sh = tl.x < 0;
      if (blkn >= (sh ? per_s : per_r)) continue;
      const int K = GATEUP ? H : A.b[sh].I;
      const int G = K / 32;
      for (int g0 = 0; g0 < G; g0 += kMmaKC, ++c) {
        const int s = c % kMmaNS;
        bool ok = *abort == 0;
        if (ok && !mma_wait_ahead(&full[s], (c / kMmaNS) & 1)) {
          *abort = 1;
          if (lane == 0) wait_failed(A.status, kKern, 4, s);
          ok = false;
        }
        uint8_t* st = base + s * MmaStage::BYTES;
        if (ok) {
          if (WBITS == 8) {
            // int8 piece p (16 codes of a row) -> fp16 pieces 2p, 2p + 1; every load of the
            // thread's share first (independent chains)
            constexpr int NQ = 4 * 128 / NPT;
            uint4 w[NQ];
#pragma unroll
            for (int u = 0; u < NQ; ++u) w[u] = *reinterpret_cast<const uint4*>(st + MmaStage::B8 + (pt + u * NPT) * 16);
#pragma unroll
            for (int u = 0; u < NQ; ++u) {
              const int q = pt + u * NPT, p = q >> 7, r = q & 127;
              uint4 lo, hi;
              cvt_i8x4_f16(w[u].x, lo.x, lo.y);
              cvt_i8x4_f16(w[u].y, lo.z, lo.w);
              cvt_i8x4_f16(w[u].z, hi.x, hi.y);
              cvt_i8x4_f16(w[u].w, hi.z, hi.w);
              *reinterpret_cast<uint4*>(st + MmaStage::BH + ((2 * p) * 128 + r) * 16) = lo;
              *reinterpret_cast<uint4*>(st + MmaStage::BH + ((2 * p + 1) * 128 + r) * 16) = hi;
            }
          }
          if (WBITS == 2) {
            // the packed int2 piece of a row (its 64 codes of the stage, element 4b + i in bits
            // 2i .. 2i + 1 of byte b) -> fp16 pieces 0 .. 7
            constexpr int NQ = 128 / NPT;
            uint4 w[NQ];
#pragma unroll
            for (int v = 0; v < NQ; ++v) w[v] = *reinterpret_cast<const uint4*>(st + MmaStage::B8 + (pt + v * NPT) * 16);
#pragma unroll
            for (int v = 0; v < NQ; ++v) {
              const int r = pt + v * NPT;
              const uint32_t wv[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {                          // elements 16 u .. 16 u + 15
                const uint32_t x = wv[u] ^ 0xAAAAAAAAu;               // fields n + 2
                const uint32_t m2 = 0x03030303u;
                const uint32_t f0 = x & m2, f1 = (x >> 2) & m2, f2 = (x >> 4) & m2, f3 = (x >> 6) & m2;
                const uint32_t a = __byte_perm(f0, f1, 0x5140), b = __byte_perm(f2, f3, 0x5140);   // 0 1 4 5, 2 3 6 7
                const uint32_t c = __byte_perm(f0, f1, 0x7362), d = __byte_perm(f2, f3, 0x7362);   // 8 9 12 13, 10 11 14 15
                uint4 o0, o1;
                cvt_u4x4_f16<2>(__byte_perm(a, b, 0x5410), o0.x, o0.y);
                cvt_u4x4_f16<2>(__byte_perm(a, b, 0x7632), o0.z, o0.w);
                cvt_u4x4_f16<2>(__byte_perm(c, d, 0x5410), o1.x, o1.y);
                cvt_u4x4_f16<2>(__byte_perm(c, d, 0x7632), o1.z, o1.w);
                *reinterpret_cast<uint4*>(st + MmaStage::BH + ((2 * u) * 128 + r) * 16) = o0;
                *reinterpret_cast<uint4*>(st + MmaStage::BH + ((2 * u + 1) * 128 + r) * 16) = o1;
              }
            }
          }
          if (WBITS == 4) {
            // packed int4 piece j (the 32 codes of group j of a row, element 2b in the low nibble
            // of byte b) -> fp16 pieces 4j .. 4j + 3
            constexpr int NQ = 2 * 128 / NPT;
            uint4 w[NQ];
#pragma unroll
            for (int v = 0; v < NQ; ++v) w[v] = *reinterpret_cast<const uint4*>(st + MmaStage::B8 + (pt + v * NPT) * 16);
#pragma unroll
            for (int v = 0; v < NQ; ++v) {
              const int q = pt + v * NPT, j = q >> 7, r = q & 127;
              const uint32_t wv[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint32_t x = wv[u] ^ 0x88888888u;            // nibbles n + 8
                const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
                uint4 o;
                cvt_u4x4_f16(__byte_perm(lo, hi, 0x5140), o.x, o.y);   // elements 8u .. 8u + 3
                cvt_u4x4_f16(__byte_perm(lo, hi, 0x7362), o.z, o.w);   // elements 8u + 4 .. 8u + 7
                *reinterpret_cast<uint4*>(st + MmaStage::BH + ((4 * j + u) * 128 + r) * 16) = o;
              }
            }
          }
          fence_async_smem();
          const __half* bs = reinterpret_cast<const __half*>(st + MmaStage::BS);
          float* bsf = reinterpret_cast<float*>(st + MmaStage::BSF);
          for (int q = pt; q < kMmaKC * 128; q += NPT) bsf[q] = __half2float(bs[q]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&prep[s]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // 16 warps: epilogue warp e reads tensor-memory lane quadrant warp % 4 (slots 32 q ..) and
    // column slice e / 4: gate/up -> gate columns 16 c .. 16 c + 15 and the matching up columns
    // 64 + 16 c ..; down -> output rows 32 c .. 32 c + 31 of the block.
    const int ew = warp - kMmaEpi0;         // [0, 16)
    const int quad = warp & 3;              // tensor-memory lane quadrant of this warp
    const int cs = ew >> 2;                 // column slice
    const int t = quad * 32 + lane;         // slot of the tile = tensor-memory lane
    const int colA = GATEUP ? 16 * cs : 32 * cs;
    const int colB = GATEUP ? 64 + 16 * cs : 32 * cs + 16;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    // gate/up: the two slices of one Q8_0 group of h meet here (per item parity, group, slot)
    int* amax_s = xchg;                     // [item parity][group][slot]
    uint32_t c = 0, gi = 0, nit = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      const int ti = it / per, blkn = it - ti * per;
      const int4 tl = A.tiles[ti];
      const int sh = tl.x < 0;
      if (blkn >= (sh ? per_s : per_r)) continue;
      const int K = GATEUP ? H : A.b[sh].I;
      const int G = K / 32;
      float2 acc2[16];                       // columns colA .. +15 (acc2[0..7]), colB .. (acc2[8..15])
#pragma unroll
      for (int q = 0; q < 16; ++q) acc2[q] = make_float2(0.0f, 0.0f);
      for (int g0 = 0; g0 < G; g0 += kMmaKC, ++c) {
        const int s = c % kMmaNS;
        bool ok = *abort == 0;
        if (ok && !mbar_wait(&prep[s], (c / kMmaNS) & 1)) {
          *abort = 1;
          if (lane == 0) wait_failed(A.status, kKern, 5, s);
          ok = false;
        }
        const uint8_t* st = base + s * MmaStage::BYTES;
        const __half* as = reinterpret_cast<const __half*>(st + MmaStage::AS);
        const float* bsf = reinterpret_cast<const float*>(st + MmaStage::BSF);
        const uint32_t pr = c & 1;            // pair mode: the stage's accumulator pair
        if (kMmaPairCommit) {
          if (ok && !mbar_wait(&acc_full[pr], (c >> 1) & 1)) {
            *abort = 1;
            if (lane == 0) wait_failed(A.status, kKern, 6, pr);
            ok = false;
          }
          ok = __all_sync(0xffffffffu, ok);
          tc_fence_after();
        }
#pragma unroll
        for (int j = 0; j < kMmaKC; ++j, ++gi) {
          const int bb = kMmaPairCommit ? (int)(2 * pr + j) : (int)(gi % kMmaNB);
          if (!kMmaPairCommit) {
            if (ok && !mbar_wait(&acc_full[bb], (gi / kMmaNB) & 1)) {
              *abort = 1;
              if (lane == 0) wait_failed(A.status, kKern, 6, bb);
              ok = false;
            }
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
          }
          uint32_t d0[16], d1[16];
          if (ok) {
            tmem_ld16(tq + bb * 128 + colA, d0);
            tmem_ld16(tq + bb * 128 + colB, d1);
            tmem_wait_ld();
          }
          if (!kMmaPairCommit || j == kMmaKC - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[kMmaPairCommit ? (int)pr : bb]);
          }
          if (!GATEUP && A.dbg_dots[sh] && ok && t < tl.z) {
            // debug: the down GEMM's exact group dots (fp32 integers) of output rows
            // n0 .. n0 + 31 for this slot, group g0 + j
            const int GI = K / 32, n0 = blkn * 128 + 32 * cs;
            int32_t* dd = A.dbg_dots[sh] + ((int64_t)(tl.y + t) * H + n0) * GI + g0 + j;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              dd[(int64_t)q * GI] = (int32_t)__uint_as_float(d0[q]);
              dd[(int64_t)(16 + q) * GI] = (int32_t)__uint_as_float(d1[q]);
            }
          }
          if (ok) {
            // acc = fma((float)I_g, s_w * s_x, acc) per element, two elements per packed op; the
            // tensor cores already produced (float)I_g exactly
            const float sx = __half2float(as[j * 128 + t]);
            const float2 sx2 = make_float2(sx, sx);
            const float4* sa = reinterpret_cast<const float4*>(bsf + j * 128 + colA);
            const float4* sb = reinterpret_cast<const float4*>(bsf + j * 128 + colB);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 wa = sa[q4], wb = sb[q4];
              const int q = 4 * q4;
              acc2[q / 2] = __ffma2_rn(make_float2(__uint_as_float(d0[q]), __uint_as_float(d0[q + 1])),
                                       __fmul2_rn(make_float2(wa.x, wa.y), sx2), acc2[q / 2]);
              acc2[q / 2 + 1] = __ffma2_rn(make_float2(__uint_as_float(d0[q + 2]), __uint_as_float(d0[q + 3])),
                                           __fmul2_rn(make_float2(wa.z, wa.w), sx2), acc2[q / 2 + 1]);
              acc2[8 + q / 2] = __ffma2_rn(make_float2(__uint_as_float(d1[q]), __uint_as_float(d1[q + 1])),
                                           __fmul2_rn(make_float2(wb.x, wb.y), sx2), acc2[8 + q / 2]);
              acc2[8 + q / 2 + 1] = __ffma2_rn(make_float2(__uint_as_float(d1[q + 2]), __uint_as_float(d1[q + 3])),
                                               __fmul2_rn(make_float2(wb.z, wb.w), sx2), acc2[8 + q / 2 + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      float acc[32];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        acc[2 * q] = acc2[q].x;
        acc[2 * q + 1] = acc2[q].y;
      }
      const bool live = *abort == 0;
      // ---- item output
      const bool valid = t < tl.z;
      const int slot = tl.y + t;
      if (GATEUP) {
        const int I = A.b[sh].I, IB = I / 32;
        const int i0 = blkn * 64 + 16 * cs;  // the thread's 16 intermediate indices
        const int par = nit & 1, gl = cs >> 1;
        int* am = amax_s + (par * 2 + gl) * 128 + t;
        float h[16];
        float amax = 0.0f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          h[q] = cswiglu(acc[q], acc[16 + q]);
          amax = fmaxf(amax, fabsf(h[q]));
        }
        atomicMax(am, __float_as_int(amax));             // non-negative: int order = float order
        named_bar(2, 32 * kMmaEpiWarps);
        const float sc = f16_round(__fdiv_rn(__int_as_float(*am), 127.0f));
        uint32_t pk[4];
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          uint32_t v = 0;
#pragma unroll
          for (int u = 0; u < 4; ++u) v |= (uint32_t)(uint8_t)(int8_t)quant_code(h[4 * w4 + u], sc, 127.0f) << (8 * u);
          pk[w4] = v;
        }
        if (live) {
          // the down GEMM's operand A: the 16 codes as fp16, pieces i0 / 8 and i0 / 8 + 1
          uint4 f0, f1;
          cvt_i8x4_f16(pk[0], f0.x, f0.y);
          cvt_i8x4_f16(pk[1], f0.z, f0.w);
          cvt_i8x4_f16(pk[2], f1.x, f1.y);
          cvt_i8x4_f16(pk[3], f1.z, f1.w);
          uint4* hd = reinterpret_cast<uint4*>(A.h_ops) + ((int64_t)ti * (A.hk / 8) + i0 / 8) * 128 + t;
          hd[0] = f0;
          hd[128] = f1;
          if (valid) {
            *reinterpret_cast<uint4*>(A.qh[sh] + (int64_t)slot * I + i0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (A.dbg_a[sh])
              for (int q = 0; q < 16; ++q) {
                A.dbg_a[sh][(int64_t)slot * I + i0 + q] = acc[q];
                A.dbg_b[sh][(int64_t)slot * I + i0 + q] = acc[16 + q];
              }
          }
        }
        named_bar(2, 32 * kMmaEpiWarps);
        if ((cs & 1) == 0) {
          if (live) {
            const int64_t hg = (int64_t)ti * (A.hk / 32) + i0 / 32;
            A.h_scales[hg * 128 + t] = __float2half_rn(sc);
            if (valid) A.sh[sh][(int64_t)slot * IB + i0 / 32] = __float2half_rn(sc);
          }
          *am = 0;                           // this parity's entry is next used two items on
        }
      } else if (valid && live) {
        int tok = slot;
        float wt = 1.0f;
        bool okp = true;
        if (!sh) {
          const int p = A.perm[slot];
          okp = p >= 0 && p < A.T * A.k;
          if (!okp) set_status(A.status, kStatusDeviceCheck);
          tok = okp ? p / A.k : 0;
          wt = okp ? A.wts[p] : 0.0f;
        }
        if (okp) {
          const int n0 = blkn * 128 + 32 * cs;
          float* yr = A.y + (int64_t)tok * H + n0;
#pragma unroll
          for (int q = 0; q < 32; q += 4)
            red_add_v4(yr + q, wt * acc[q], wt * acc[q + 1], wt * acc[q + 2], wt * acc[q + 3]);
          if (A.dbg_y[sh])
            for (int q = 0; q < 32; ++q) atomicAdd(A.dbg_y[sh] + (int64_t)slot * H + n0 + q, acc[q]);
        }
      }
      ++nit;
    }
  }
  // all tensor-memory reads done before the allocating warp frees it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kMmaNB * 128);
}

// -------------------------------------------------------------------- host side
namespace {

int sm_count_mma() { return device_sm_count(); }

template <int WBITS, bool GATEUP>
cudaError_t launch_mma_t(const MmaArgs& a, int max_items, cudaStream_t st) {
  {
    const cudaError_t e = ensure_smem_attr((const void*)k_expert_mma<WBITS, GATEUP>, kMmaSmem);
    if (e != cudaSuccess) return e;
  }
  const int grid = std::max(1, std::min(max_items, sm_count_mma()));
  return launch_pdl(k_expert_mma<WBITS, GATEUP>, dim3(grid), dim3(kMmaThreads), (size_t)kMmaSmem, st, a);
}

}  // namespace

cudaError_t launch_mma_plan(const Grouping& g, int E, int T, int has_shared, int min_tokens, int max_tiles,
                            int4* tiles, int32_t* n_tiles, int* status, cudaStream_t st) {
  return launch_pdl(k_mma_plan, dim3(1), dim3(1024), 0, st, (const int32_t*)g.n_active,
                    (const int32_t*)g.act_expert, (const int32_t*)g.act_begin, E, T, has_shared, min_tokens,
                    max_tiles, tiles, n_tiles, status);
}

cudaError_t launch_mma_gather(const int8_t* qx, const __half* sx, const int4* tiles, const int32_t* n_tiles,
                              const int32_t* perm, int k, int T, int K, int max_tiles, uint8_t* xa, __half* xs,
                              int* status, cudaStream_t st) {
  const int64_t work = (int64_t)max_tiles * 128 * (K / 32);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, (int64_t)sm_count_mma() * 8));
  return launch_pdl(k_mma_gather, dim3(grid), dim3(256), 0, st, qx, sx, tiles, n_tiles, perm, k, T, K, xa, xs,
                    status);
}

cudaError_t launch_expert_mma(bool gateup, const MmaArgs& a, cudaStream_t st) {
  const int per_r = gateup ? a.b[0].I / 64 : a.b[0].H / 128;
  const int per_s = gateup ? a.b[1].I / 64 : a.b[1].H / 128;
  const int max_items = a.max_tiles * std::max(per_r, per_s);
  if (a.b[0].wbits == 8)
    return gateup ? launch_mma_t<8, true>(a, max_items, st) : launch_mma_t<8, false>(a, max_items, st);
  if (a.b[0].wbits == 2)
    return gateup ? launch_mma_t<2, true>(a, max_items, st) : launch_mma_t<2, false>(a, max_items, st);
  return gateup ? launch_mma_t<4, true>(a, max_items, st) : launch_mma_t<4, false>(a, max_items, st);
}

}  // namespace moe
