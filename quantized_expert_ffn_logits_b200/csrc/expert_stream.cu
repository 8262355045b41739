// expert_stream.cu -- weight-streaming expert kernels (decode and small batches).
//
// Integer dots per group of 32, the canonical fp32 scale chain per row, SwiGLU and h
// quantization in the gate/up epilogue (GLM-5.2 colibri page, "Integer-dot kernels",
// "Quantization kernels: ... dequant-on-use"; "Batch-union MoE": every selected expert's
// weights are streamed once per call, whatever the number of tokens routed to it).
//
// Work unit = one selected expert x 64 intermediate indices: its gate/up block (64 gate rows
// and the 64 matching up rows, the whole K range contiguous in the blob as [piece][128
// rows][16 B]) and its down slab (all H output rows x those 64 columns). Grid = one
// persistent CTA per SM (at most one per unit), units round-robin; a unit with more tokens
// than fit one pass is streamed once per pass.
//
// CTA = one producer warp + eight consumer warps. The producer's lane 0 walks the CTA's
// passes and pushes 32 KB chunks (16 pieces) plus the matching scales into a four-stage
// shared-memory ring with cp.async.bulk ("full" mbarrier per stage, released on an "empty"
// mbarrier), and the pass's activation rows into one of two activation buffers right behind
// the pass's first chunk. Consumers, per block of 8 groups: warp w forms the exact int32 dots
// of group w for all 128 rows, a consumer barrier, then one thread per (row, token) runs the
// ordered fp32 chain acc = fma((float)I_g, c_g, acc). After the gate/up pass the gate and up
// values meet in shared memory, two warps apply SwiGLU and quantize h per group of 32, and
// the unit's down slab is consumed against those codes, each row's share added into y with
// 16-byte reductions. With one token and group-32 activations (MODE 3) the kernel also does
// the routing (route_one_token): the whole layer is one launch. Every wait is bounded: a
// wait that gives up sets the status word, the consumers skip the rest of their work but
// keep releasing stages (all warps take the same barriers), and the producer drains its
// copies before the CTA exits.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"
#include "topk.cuh"

namespace moe {

constexpr int kRows = 128;                 // rows per unit
constexpr int kPiece = kRows * 16;         // bytes of one 16-byte column of the unit: 2 KB
constexpr int kSP = 16;                    // pieces per ring stage (32 KB)
constexpr int kNS = 4;                     // ring stages
constexpr int kCW = 8;                     // consumer warps
constexpr int kNT = 32 * (kCW + 1);        // + the producer warp
constexpr int kTMP = 8;                    // most tokens per pass over a unit's weights
constexpr int kSmemMax = 227 * 1024;

// Shared-memory plan (offsets from a 1024-aligned base). Activation buffer b holds tm rows
// of K codes, then (g32 activations) tm rows of G fp16 scales.
// Single-token routing scratch (RingPlan::route): se, swt, sj, sidx, sw, own [32] each,
// then two flag words and the y-zero barrier target (8 bytes).
constexpr int kRouteBytes = 8 * 32 * 4;

struct RingPlan {
  int ring, sring, sstage, bars, abuf, abytes, ascale, xsum, sxf, idot, ubuf, hq, info, route, total;
};

// Bytes of one stage's scales: a chunk's fp16 group scales (16 pieces of codes hold 8, 16 or
// 32 groups of 128 rows for int8, int4, int2) or its down blocks' scales.
__host__ __device__ inline int ring_sstage(int wbits) { return wbits >= 4 ? 4096 : 16384 / wbits; }

// ring_min: bytes the ring region must at least have (the single-token routing scratch).
__host__ __device__ inline RingPlan ring_plan(int K, int tm, int wbits, int ring_min = 0) {
  RingPlan p;
  const int G = K / 32;
  int o = 0;
  // every region starts on a 128-byte boundary (128-bit and bulk-copy accesses)
  auto take = [&](int bytes) {
    const int at = o;
    o = (o + bytes + 127) & ~127;
    return at;
  };
  p.ring = take(kNS * kSP * kPiece > ring_min ? kNS * kSP * kPiece : ring_min);   // 128 KB or more
  p.sstage = ring_sstage(wbits);
  p.sring = take(kNS * p.sstage);               // group / row scales of a stage
  p.bars = take((2 * kNS + 4) * 8);
  p.ascale = tm * K;                            // offset of the scales inside a buffer
  p.abytes = (tm * K + tm * G * 2 + 127) & ~127;
  p.abuf = take(2 * p.abytes);
  p.xsum = take(2 * tm * G * 4);
  p.sxf = take(tm * G * 4);                     // scales not copied by the producer, as fp32
  p.idot = take(2 * 8 * tm * kRows * 4);        // int32 dots of a block of 8 groups, two buffers
  p.ubuf = take(2 * tm * 64 * 4);               // gate / up stage values of a pass
  p.hq = take(2 * tm * 64 + 2 * tm * 4 + 2 * tm * 4);   // h codes (+ de-interleaved), scales, sums
  p.info = take(3 * kTMP * 4 + 16);             // tokens, weights, abort flag
  p.route = take(kRouteBytes);                 // single-token routing (in-kernel selection)
  p.total = o + 1024;                           // slack for aligning the base
  return p;
}

// Tokens per pass: up to kTMP, as many as shared memory allows.
inline int ring_tokens(int K, int max_tokens, int wbits) {
  int tm = max_tokens < 1 ? 1 : (max_tokens > kTMP ? kTMP : max_tokens);
  while (tm > 1 && ring_plan(K, tm, wbits).total > kSmemMax) --tm;
  return tm;
}


// One work unit as the kernel sees it.
struct Unit {
  bool shd;      // the shared expert
  int ai;        // active-expert index (routed)
  int e;         // expert
  int s0, s1;    // slots [s0, s1) routed to it (shared: all tokens)
  int sub;       // row block inside the expert
  int rows8[8];  // tokens of slots s0 .. s0+7 (routed gate/up)
};

// Resolve grid work unit u (routed units first, then the shared expert's); false if idle.
// Routing data is read through L2 (written by an earlier kernel of the same stream); every
// load is issued before any is used, so resolving a unit costs one L2 round trip.
__device__ __forceinline__ bool unit_of(const ExpertArgs& r, const ExpertArgs& s, int has_shared,
                                        int routed_units, int per_expert_r, int u, Unit& U,
                                        bool want_rows, bool report, int mma_min) {
  if (u < routed_units) {
    U.shd = false;
    U.ai = u / per_expert_r;
    U.sub = u - U.ai * per_expert_r;
    const int na = __ldcg(r.n_active);
    U.e = __ldcg(r.act_expert + U.ai);
    U.s0 = __ldcg(r.act_begin + U.ai);
    U.s1 = __ldcg(r.act_begin + U.ai + 1);
    if (want_rows) {
      const int4 lo = __ldcg(reinterpret_cast<const int4*>(r.act_rows) + 2 * U.ai);
      const int4 hi = __ldcg(reinterpret_cast<const int4*>(r.act_rows) + 2 * U.ai + 1);
      U.rows8[0] = lo.x;
      U.rows8[1] = lo.y;
      U.rows8[2] = lo.z;
      U.rows8[3] = lo.w;
      U.rows8[4] = hi.x;
      U.rows8[5] = hi.y;
      U.rows8[6] = hi.z;
      U.rows8[7] = hi.w;
    }
    if (U.ai >= na) return false;
    if (U.s1 - U.s0 >= mma_min) return false;     // on the tensor-core path
    if (U.e < 0 || U.e >= r.b.E || U.s0 < 0 || U.s0 > U.s1 || U.s1 > r.T * r.k) {
      if (report) set_status(r.status, kStatusDeviceCheck);
      return false;
    }
    return true;
  }
  if (!has_shared || s.T >= mma_min) return false;
  U.shd = true;
  U.ai = 0;
  U.e = 0;
  U.s0 = 0;
  U.s1 = s.T;
  U.sub = u - routed_units;
  return true;
}

// Activation row of slot `slot`: gate/up reads the token's q_x row, down the slot's q_h
// row. Tokens of a routed unit's first 8 slots come with the unit; later ones from the
// pair list. A corrupt token or pair index is reported and read as row 0.
__device__ __forceinline__ int act_row(const ExpertArgs& a, bool gateup, const Unit& U, int slot) {
  if (!gateup || U.shd) return slot;
  const int j = slot - U.s0;
  int t;
  if (j < 8) {
    t = U.rows8[0];
#pragma unroll
    for (int q = 1; q < 8; ++q)
      if (j == q) t = U.rows8[q];
  } else {
    const int p = __ldcg(a.perm + slot);
    t = (p >= 0 && p < a.T * a.k) ? p / a.k : -1;
  }
  if (t < 0 || t >= a.T) {
    set_status(a.status, kStatusDeviceCheck);
    return 0;
  }
  return t;
}

// First chunk of a unit's down pass: units start at different 128-row blocks, so the
// CTAs' atomic adds into y spread over the output instead of meeting on the same lines.
__device__ __forceinline__ int down_rotation(const Unit& U, int nch) {
  return (int)(((unsigned)U.sub * 7u + (unsigned)U.ai * 3u) % (unsigned)nch);
}

struct Ring {
  uint8_t* ring;
  uint8_t* sring;     // [kNS][sstage]
  int sstage;
  uint64_t* full;     // [kNS]
  uint64_t* empty;    // [kNS]
  uint64_t* afull;    // [2]
  uint64_t* aempty;   // [2]
  uint8_t* abuf;      // [2][abytes]
  int* xsum;          // [2][tm][G]
  float* sxf;         // [tm][G] (or [tm] per-token scales)
};

// Single-token routing scratch in the (still idle) ring region: the router rows of the CTA's
// experts at a 144-byte chunk pitch (staged before the wait for the preceding kernel), the
// token's x at the same pitch, then the chunk partials (bytes; rows / x 0 = not staged).
struct RouteScratch {
  int rows, x, part;
};
__host__ __device__ inline int rs_total(const RouteScratch& s) { return s.rows + s.x + s.part; }

// Launch arguments. x[0][*] = gate/up (q_x activations, writes h), x[1][*] = down (reads h,
// adds into y); [*][0] routed experts, [*][1] the shared expert. Units are (expert,
// 64 intermediate indices) in every mode: MODE 0 runs the gate/up pass of each unit,
// MODE 1 its down pass (h from an earlier kernel), MODE 2 both, h staying on chip.
struct RingArgs {
  ExpertArgs x[2][2];
  int has_shared;
  int units;               // routed units first, then the shared expert's
  int routed;              // routed units
  int per;                 // units per routed expert (I / 64)
  int tm, kmax;
  int mma_min;             // experts with this many slots are left to the tensor-core path
  RouteArgs r;             // MODE 3 (one token): the routing done inside the kernel
  int cluster;             // MODE 3: logits shared per cluster of this many CTAs (0: grid barrier)
  RouteScratch rs;         // MODE 3: the routing scratch layout
};

// int4 weights: each 8-byte word of the activation rows de-interleaved into its even, then
// its odd elements (the order of a packed weight word's low and high nibbles), and the sum
// of every group's 32 codes (the unsigned-nibble correction of the int4 dot).
__device__ __forceinline__ void act_deinterleave(uint8_t* xs, int words, int tid, int nt) {
  for (int l = tid; l < words; l += nt) {
    uint2* wp = reinterpret_cast<uint2*>(xs) + l;
    const uint2 v = *wp;
    uint2 o;
    deinterleave8(v.x, v.y, o.x, o.y);
    *wp = o;
  }
}
// int2 weights: each 16-byte word of the activation rows de-interleaved into the order of a
// packed int2 word's fields (elements i, i + 4, i + 8, i + 12 for i = 0 .. 3).
__device__ __forceinline__ void act_deinterleave16(uint8_t* xs, int words, int tid, int nt) {
  for (int l = tid; l < words; l += nt) {
    uint4* wp = reinterpret_cast<uint4*>(xs) + l;
    *wp = deinterleave16(*wp);
  }
}
__device__ __forceinline__ void act_group_sums(const uint8_t* xs, int* xsum, int m, int K, int tid, int nt) {
  const int G = K / 32;
  for (int l = tid; l < m * G; l += nt) {
    const uint4* q4 = reinterpret_cast<const uint4*>(xs + (l / G) * K + 32 * (l % G));
    const uint4 a0 = q4[0], a1 = q4[1];
    int sacc = __dp4a((int)a0.x, 0x01010101, 0);
    sacc = __dp4a((int)a0.y, 0x01010101, sacc);
    sacc = __dp4a((int)a0.z, 0x01010101, sacc);
    sacc = __dp4a((int)a0.w, 0x01010101, sacc);
    sacc = __dp4a((int)a1.x, 0x01010101, sacc);
    sacc = __dp4a((int)a1.y, 0x01010101, sacc);
    sacc = __dp4a((int)a1.z, 0x01010101, sacc);
    sacc = __dp4a((int)a1.w, 0x01010101, sacc);
    xsum[l] = sacc;
  }
}

// ------------------------------------------------------------------ single-token routing
// MODE 3 (one token, group-32 activations) begins with the routing that other calls run as a
// separate kernel, so a decode step is one launch. Every CTA quantizes the token's
// activations (groups of 32: scale = fp16(max|x| / 127), code = x / scale rounded and
// clamped; GLM-5.2 colibri page, "Quantization kernels") straight into its activation
// buffer 0, computes the router logits of experts blockIdx.x, blockIdx.x + grid, ... in the
// fixed fp32 order (32-element fma chunks from +0, chunk partials added in chunk order) and
// zeroes its share of y. After a grid barrier every CTA reads the E logits and makes the
// same top-k selection (a chunked parallel rank; softmax or sigmoid weights as in
// topk.cuh); CTA 0 also writes the routing and grouping views of the workspace.
struct RouteSmem {
  int* se;        // [k] selected experts, ascending (active-expert order)
  float* swt;     // [k] their routing weights
  int* sj;        // [k] their positions in the token's top-k list (pair index)
  int* sidx;      // [k] the top-k list in selection order
  float* sw;      // [k] its weights
  float* own;     // [32] logits of this CTA's experts (cluster exchange)
  volatile int* flag;
  volatile unsigned long long* ytarget;   // y-zero barrier target (cluster exchange)
  volatile int* nk;                       // slots kept: k, or the adaptive top-p prefix
  volatile int* nl;                       // kept slots whose expert is held here (units)
  int* lsel;                              // [32] local id of each slot of the list, or -1
};

// Bounds of the cross-CTA waits (grid barrier, y-zero barrier): RouteArgs::wait_ns of
// %globaltimer time (about a second by default), and at most 2^22 polls (each an L2 round
// trip) whatever the timer reads.
constexpr uint32_t kGridWaitTries = 1u << 22;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long atom_add_release(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.release.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

// Poll until *p >= target; false once wait_ns have passed (checked every 32 polls) or the
// poll bound ran out.
__device__ __forceinline__ bool wait_counter(const unsigned long long* p, unsigned long long target,
                                             unsigned long long wait_ns) {
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 0; i < kGridWaitTries; ++i) {
    if (ld_acquire_u64(p) >= target) return true;
    if ((i & 31u) == 31u && globaltimer_ns() - t0 > wait_ns) return false;
  }
  return false;
}

// Grid barrier (thread 0 of every CTA, after a CTA barrier) in two halves: arrive, returning
// the target every CTA then waits for with wait_counter. The counter is a multiple of 1024
// when a call starts (grids are <= 1024 CTAs); this call's arrivals take base .. base + grid - 1
// and the last one moves the counter on to base + 1024 for the next call.
__device__ __forceinline__ unsigned long long grid_arrive(unsigned long long* ctr) {
  const unsigned long long old = atom_add_release(ctr, 1ull);   // the CTA's writes before it
  const unsigned long long target = (old & ~1023ull) + gridDim.x;
  if (old + 1 == target) atomicAdd(ctr, 1024ull - gridDim.x);
  return target;
}


// Scratch use of the (still idle) ring during the routing (RouteScratch). The logit of a
// 32-element chunk is one thread's fma chain, so threads read chunks 128 bytes apart; stored
// with a 144-byte chunk pitch instead, the eight lanes of a quarter warp hit eight different
// bank groups. Grid exchange: the 128 KB ring as [80 KB rows][28 KB x][20 KB partials], rows
// staged when they fit; cluster exchange: sized for the ne experts a CTA owns.
constexpr int kChunkPitch = 144;
constexpr int kRowBytes = 80 * 1024;
constexpr int kXBytes = 28 * 1024;
constexpr int kPartFloats = (kNS * kSP * kPiece - kRowBytes - kXBytes) / 4;
__host__ __device__ inline RouteScratch grid_scratch() { return RouteScratch{kRowBytes, kXBytes, kPartFloats * 4}; }
__host__ __device__ inline RouteScratch cluster_scratch(int ne, int C) {
  auto r128 = [](int v) { return (v + 127) & ~127; };
  RouteScratch s;
  s.rows = r128(ne * C * kChunkPitch);
  s.x = C * kChunkPitch <= kXBytes ? r128(C * kChunkPitch) : 0;
  s.part = r128((ne > 0 ? ne : 1) * C * 4);
  return s;
}

// Who computes which logits. Grid exchange: CTA b owns experts b, b + grid, ...; cluster
// exchange: cluster rank c owns experts c, c + cluster size, ... (every cluster computes all
// E logits and its CTAs share them through distributed shared memory).
struct Owners {
  int first, stride;
};
__device__ __forceinline__ Owners route_owners(bool cl) {
  Owners o;
  o.first = cl ? (int)cluster_rank() : (int)blockIdx.x;
  o.stride = cl ? (int)cluster_size() : (int)gridDim.x;
  return o;
}
__device__ __forceinline__ int owned_experts(int E, Owners o) {
  return o.first < E ? (E - 1 - o.first) / o.stride + 1 : 0;
}

// Every thread, before the wait for the preceding kernel: stage this CTA's router rows
// (model parameters, not written by the preceding kernel) into the ring, a 128-byte chunk
// per copy at the 144-byte pitch, completing on `bar`. Returns (to every thread) whether
// they fit; if not, the logits read them from global memory.
__device__ __forceinline__ bool stage_router_rows(const RouteArgs& r, bool cl, uint8_t* ring, uint64_t* bar,
                                                  volatile int* flag, int rows_bytes) {
  const Owners o = route_owners(cl);
  const int ne = owned_experts(r.E, o), C = r.H / 32;
  const bool fit = ne > 0 && (int64_t)ne * C * kChunkPitch <= rows_bytes;
  if (threadIdx.x == 0) {
    if (fit) mbar_arrive_expect_tx(bar, (uint32_t)(ne * C * 128));
    *flag = fit;
  }
  __syncthreads();                          // the expected bytes are set before any copy lands
  if (fit)
    for (int t = threadIdx.x; t < ne * C; t += kNT) {
      const int j = t / C, c = t - j * C;
      bulk_load(ring + (int64_t)t * kChunkPitch, r.wr + (int64_t)(o.first + j * o.stride) * r.H + 32 * c, 128, bar);
    }
  return fit;
}

// Slot j of the token's top-k list (S.sidx, global ids): its local expert id if the slot is
// kept (j < nk: adaptive top-p) and its expert held here (expert parallelism), else -1.
__device__ __forceinline__ int kept_local(const RouteArgs& r, const RouteSmem& S, int nk, int j) {
  const int ee = S.sidx[j];
  return (j < nk && ee >= r.e0 && ee < r.e0 + r.EL) ? ee - r.e0 : -1;
}
// Kept local slots with a local id below le (the position of le in ascending order).
__device__ __forceinline__ int kept_local_rank(const RouteArgs& r, const RouteSmem& S, int nk, int le) {
  int pos = 0;
  for (int j = 0; j < r.k; ++j) {
    const int o = kept_local(r, S, nk, j);
    pos += (o >= 0) & (o < le);
  }
  return pos;
}

// Grid exchange: 32-element chunk c (= the thread index) of the router rows of this CTA's
// first two experts, loaded into registers before the wait for the preceding kernel (model
// parameters, not written by it), so their latency overlaps the kernel's start.
struct RowChunks {
  float4 w[2][8];
};
__device__ __forceinline__ void prefetch_router_chunks(const RouteArgs& r, RowChunks& pf) {
  const int C = r.H / 32, c = threadIdx.x;
  const Owners o = route_owners(false);
  const int ne = owned_experts(r.E, o);
#pragma unroll
  for (int j = 0; j < 2; ++j)
    if (c < C && j < ne) {
      const float4* w4 = reinterpret_cast<const float4*>(r.wr + (int64_t)(o.first + j * o.stride) * r.H + 32 * c);
#pragma unroll
      for (int v = 0; v < 8; ++v) pf.w[j][v] = __ldg(w4 + v);
    }
}

// One 32-element router chunk against the token's same chunk: the fma chain from +0 in
// ascending index.
__device__ __forceinline__ float chunk_logit(const float4 (&xv)[8], const float4 (&wv)[8]) {
  float acc = 0.0f;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    acc = __fmaf_rn(xv[v].x, wv[v].x, acc);
    acc = __fmaf_rn(xv[v].y, wv[v].y, acc);
    acc = __fmaf_rn(xv[v].z, wv[v].z, acc);
    acc = __fmaf_rn(xv[v].w, wv[v].w, acc);
  }
  return acc;
}

// Q8_0 codes and group scales of the token into activation buffer 0 (and, CTA 0, the q_x /
// s_x views): 8 threads per group, 4 elements each, every load of a round in flight at once
// (8 G is a multiple of 32, so a warp's lanes are all in range or all out). xpad (optional):
// x also stored at the routing scratch's chunk pitch.
__device__ __forceinline__ void quantize_token(const RouteArgs& r, const RingPlan& P, const Ring& R,
                                               uint8_t* xpad, int tid, int nt) {
  const int G = r.H / 32;
  const bool cta0 = blockIdx.x == 0;
  uint8_t* xs = R.abuf;
  __half* sxs = reinterpret_cast<__half*>(xs + P.ascale);
  for (int l0 = tid; l0 < 8 * G; l0 += 4 * nt) {
    float4 xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (l0 + u * nt < 8 * G) xv[u] = __ldg(reinterpret_cast<const float4*>(r.x) + l0 + u * nt);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int l = l0 + u * nt;
      if (l >= 8 * G) break;                   // warp-uniform (nt a multiple of 32)
      const int g = l >> 3;
      const float4 v = xv[u];
      float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const float sc = f16_round(__fdiv_rn(m, 127.0f));
      const uint32_t word = (uint32_t)(uint8_t)(int8_t)quant_code(v.x, sc, 127.0f) |
                            (uint32_t)(uint8_t)(int8_t)quant_code(v.y, sc, 127.0f) << 8 |
                            (uint32_t)(uint8_t)(int8_t)quant_code(v.z, sc, 127.0f) << 16 |
                            (uint32_t)(uint8_t)(int8_t)quant_code(v.w, sc, 127.0f) << 24;
      reinterpret_cast<uint32_t*>(xs)[l] = word;
      if ((l & 7) == 0) sxs[g] = __float2half_rn(sc);
      if (xpad) *reinterpret_cast<float4*>(xpad + (l >> 3) * kChunkPitch + (l & 7) * 16) = v;
      if (cta0) {
        reinterpret_cast<uint32_t*>(r.qx)[l] = word;
        if ((l & 7) == 0) reinterpret_cast<__half*>(r.sx)[g] = __float2half_rn(sc);
      }
    }
  }
}

// Grid exchange, the logits (step 3 of route_one_token) first: thread c loads the token's
// chunk c and forms the chunk partials of every expert this CTA owns (the first two from the
// prefetched registers); the partials are added in chunk order per expert, and the CTA's
// share of y is zeroed. Ends with a CTA barrier.
__device__ __forceinline__ void grid_logits(const RouteArgs& r, const Ring& R, const RowChunks& pf) {
  const int tid = threadIdx.x, H = r.H, C = H / 32;
  const Owners own = route_owners(false);
  const int ne = owned_experts(r.E, own);
  float* part = reinterpret_cast<float*>(R.ring);          // [ne][C]
  for (int c = tid; c < C && ne > 0; c += kNT) {
    float4 xv[8];
    const float4* x4 = reinterpret_cast<const float4*>(r.x + 32 * c);
#pragma unroll
    for (int v = 0; v < 8; ++v) xv[v] = __ldg(x4 + v);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (j < ne) {
        float4 wv[8];
        if (c == tid) {
#pragma unroll
          for (int v = 0; v < 8; ++v) wv[v] = pf.w[j][v];
        } else {
          const float4* w4 = reinterpret_cast<const float4*>(r.wr + (int64_t)(own.first + j * own.stride) * H + 32 * c);
#pragma unroll
          for (int v = 0; v < 8; ++v) wv[v] = __ldg(w4 + v);
        }
        part[j * C + c] = chunk_logit(xv, wv);
      }
    for (int j = 2; j < ne; ++j) {
      float4 wv[8];
      const float4* w4 = reinterpret_cast<const float4*>(r.wr + (int64_t)(own.first + j * own.stride) * H + 32 * c);
#pragma unroll
      for (int v = 0; v < 8; ++v) wv[v] = __ldg(w4 + v);
      part[j * C + c] = chunk_logit(xv, wv);
    }
  }
  // this CTA's share of y = 0 (ordered before every CTA's adds by the grid barrier)
  float4* y4 = reinterpret_cast<float4*>(r.y);
  for (int l = blockIdx.x * kNT + tid; l < H / 4; l += gridDim.x * kNT) y4[l] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  for (int j = tid; j < ne; j += kNT) {
    const float* pj = part + j * C;
    float total = 0.0f;
    int c = 0;
    for (; c + 8 <= C; c += 8) {
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = pj[c + q];
#pragma unroll
      for (int q = 0; q < 8; ++q) total = __fadd_rn(total, v[q]);
    }
    for (; c < C; ++c) total = __fadd_rn(total, pj[c]);
    r.logits[own.first + j * own.stride] = total;
  }
  __syncthreads();
}

// Every thread of the CTA. False when a wait gave up (status recorded; with the cluster
// exchange the CTA has still taken both cluster-barrier arrivals, and must wait on the
// second before it exits). reg_rows: grid exchange with the router chunks prefetched in pf;
// else the router rows were staged and complete on rows_bar (or, null, are read from global
// memory).
template <bool TOPP>
__device__ bool route_one_token(const RouteArgs& r, const RingPlan& P, const Ring& R, const RouteSmem& S,
                                uint64_t* rows_bar, bool cl, const RouteScratch& rs, const RowChunks& pf,
                                bool reg_rows) {
  volatile int* flag = S.flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = r.H, G = H / 32, C = H / 32, E = r.E, k = r.k;
  const bool cta0 = blockIdx.x == 0;
  const Owners own = route_owners(cl);
  if (cta0 && tid == 0) {
    r.status[0] = 0;
    r.status[2] = 0;
    r.status[3] = 0;
  }
  bool good = true;
  unsigned long long gtarget = 0;
  if (reg_rows) {
    // logits, y share zeroed, then warp 0 arrives at the grid barrier and waits (below) while
    // the other warps quantize the token
    grid_logits(r, R, pf);
    if (tid == 0) gtarget = grid_arrive(r.gbar);
    if (warp > 0) quantize_token(r, P, R, nullptr, tid - 32, kNT - 32);
  } else {
  // 1. the token's Q8_0 codes, and x at the chunk pitch for the staged logits (cluster
  //    exchange, or grid exchange with more than two experts per CTA)
  uint8_t* xpad = (rs.x && C * kChunkPitch <= rs.x) ? R.ring + rs.rows : nullptr;
  quantize_token(r, P, R, xpad, tid, kNT);
  // 2. this CTA's share of y = 0 (ordered before every CTA's adds by a grid barrier: the
  //    routing's, or with the cluster exchange one whose wait comes before the first add)
  float4* y4 = reinterpret_cast<float4*>(r.y);
  for (int l = blockIdx.x * kNT + tid; l < H / 4; l += gridDim.x * kNT) y4[l] = make_float4(0.f, 0.f, 0.f, 0.f);
  // 3. logits of this CTA's experts, as many at a time as their chunk partials fit the ring
  //    (idle until the selection): partials first, then each expert's added in chunk order
  float* part = reinterpret_cast<float*>(R.ring + rs.rows + rs.x);
  const int ne = owned_experts(E, own);
  const int nb = rs.part / 4 / C;
  if (rows_bar) {
    // the router rows (copied while the preceding kernel finished): polled, not suspended on
    bool ok = false;
    for (uint32_t i = 0; i < (1u << 24) && !ok; ++i) ok = mbar_try_wait(rows_bar, 0);
    if (tid == 0) *flag = ok;
  }
  __syncthreads();                          // x at the chunk pitch, the rows' wait result
  if (rows_bar) {
    good = *flag != 0;
    if (!good && tid == 0) wait_failed(r.status, 1, 7, 0);
  }
  for (int j0 = 0; good && j0 < ne; j0 += nb) {
    const int nj = min(nb, ne - j0);
    for (int l = tid; l < nj * C; l += kNT) {
      const int j = l / C, c = l - j * C;
      const int e = own.first + (j0 + j) * own.stride;
      float4 wv[8], xv4[8];
      if (rows_bar) {
        const float4* w4 = reinterpret_cast<const float4*>(R.ring + ((j0 + j) * C + c) * kChunkPitch);
#pragma unroll
        for (int v = 0; v < 8; ++v) wv[v] = w4[v];
      } else {
        const float4* w4 = reinterpret_cast<const float4*>(r.wr + (int64_t)e * H + 32 * c);
#pragma unroll
        for (int v = 0; v < 8; ++v) wv[v] = __ldg(w4 + v);
      }
      if (xpad) {
        const float4* x4 = reinterpret_cast<const float4*>(xpad + c * kChunkPitch);
#pragma unroll
        for (int v = 0; v < 8; ++v) xv4[v] = x4[v];
      } else {
        const float4* x4 = reinterpret_cast<const float4*>(r.x + 32 * c);
#pragma unroll
        for (int v = 0; v < 8; ++v) xv4[v] = __ldg(x4 + v);
      }
      float acc = 0.0f;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const float4 xv = xv4[v];
        acc = __fmaf_rn(xv.x, wv[v].x, acc);
        acc = __fmaf_rn(xv.y, wv[v].y, acc);
        acc = __fmaf_rn(xv.z, wv[v].z, acc);
        acc = __fmaf_rn(xv.w, wv[v].w, acc);
      }
      part[l] = acc;
    }
    __syncthreads();
    for (int j = tid; j < nj; j += kNT) {
      const float* pj = part + j * C;
      float total = 0.0f;
      int c = 0;
      for (; c + 8 <= C; c += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = pj[c + q];
#pragma unroll
        for (int q = 0; q < 8; ++q) total = __fadd_rn(total, v[q]);
      }
      for (; c < C; ++c) total = __fadd_rn(total, pj[c]);
      const int e = own.first + (j0 + j) * own.stride;
      if (!cl || (int)blockIdx.x < own.stride) r.logits[e] = total;   // the fp32 logit view
      if (cl) S.own[j0 + j] = total;
    }
    __syncthreads();
  }
  __syncthreads();
  }   // cluster exchange: steps 1-3 from the staged router rows
  // 4. every logit into this CTA's shared memory
  float* slog = reinterpret_cast<float*>(R.ring);           // scratch again: [E] logits
  float* skey = slog + 512;                                  //                [E] selection keys
  if (!cl) {
    if (tid == 0) {
      if (!reg_rows) gtarget = grid_arrive(r.gbar);
      *flag = wait_counter(r.gbar, gtarget, r.wait_ns) ? 1 : 0;
    }
    __syncthreads();
    if (!*flag) {
      if (tid == 0) wait_failed(r.status, 1, 6, 0);
      return false;
    }
    if (!good) return false;
    for (int i = tid; i < E; i += kNT) slog[i] = __ldcg(r.logits + i);
  } else {
    if (tid == 0) {
      // y-zero barrier, first half: this CTA's share of y is zero; the wait is taken before
      // the CTA's first add into y
      __threadfence();
      const unsigned long long old = atomicAdd(r.gbar, 1ull);
      const unsigned long long target = (old & ~1023ull) + gridDim.x;
      if (old + 1 == target) atomicAdd(r.gbar, 1024ull - gridDim.x);
      *S.ytarget = target;
    }
    cluster_arrive();
    cluster_wait();
    for (int i = tid; i < E; i += kNT) slog[i] = ld_dsmem_f32(S.own + i / own.stride, (uint32_t)(i % own.stride));
    cluster_arrive();                                       // this CTA's remote reads are done
    if (!good) return false;
  }
  if (tid < 32) S.sidx[tid] = -1;
  if (TOPP && tid == 0) *S.nk = k;
  // 5. top-k (every CTA, same result): keys ranked by (keys larger, or equal with a lower
  //    expert index): descending, ties to the lower expert. The logits also go to activation
  //    buffer 1 (idle in this mode): the routing weights are formed there after the producer
  //    has started.
  float* slogk = reinterpret_cast<float*>(R.abuf + P.abytes);
  float* ckey = skey + 512;                                 // [E / 64 * k] candidate keys
  int* cidx = reinterpret_cast<int*>(ckey + 512);           //              their experts
  for (int i = tid; i < E; i += kNT) {
    const float L = slog[i];
    slogk[i] = L;
    skey[i] = r.score == 0 ? L : __fadd_rn(csigmoid(L), r.bias ? r.bias[i] : 0.0f);
  }
  const int nch = (E + 63) / 64, ncand = nch * k;
  for (int t = tid; t < ncand; t += kNT) cidx[t] = -1;     // chunks with fewer than k keys
  __syncthreads();
  // Two phases, O(64 E + (k E / 64)^2) comparisons instead of O(E^2): (a) every key ranks
  // itself within its chunk of 64 keys (one thread per key); with one chunk that is the
  // answer, else a key of chunk rank < k is a candidate, kept (key and expert) at slot
  // chunk * k + rank; (b) every candidate ranks itself against all candidates. A key of the
  // global top k is among its chunk's top k, and every key ranked above it is too, so its rank
  // among the candidates is its global rank (same tie rule throughout).
  // (a): four adjacent lanes per key, each counting one quarter (16 keys) of the key's chunk
  // with four independent counters; two xor-shuffles add the quarters. Warps step through the
  // (key, quarter) pairs together so every shuffle has its whole warp.
  for (int l0 = warp * 32; l0 < 4 * E; l0 += kNT) {
    const int l = l0 + lane, i = l >> 2, qt = l & 3;
    const bool on = l < 4 * E;
    const int base = i & ~63, n = on ? min(64, E - base) : 0;
    const float kv = on ? skey[i] : 0.0f;
    const int j0 = 16 * qt, j1 = min(j0 + 16, n);
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0, j = j0;
    if (j1 - j0 == 16) {
      const float4* k4 = reinterpret_cast<const float4*>(skey + base + j0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 q = k4[u];
        const int jj = base + j0 + 4 * u;
        r0 += (q.x > kv) | ((q.x == kv) & (jj < i));
        r1 += (q.y > kv) | ((q.y == kv) & (jj + 1 < i));
        r2 += (q.z > kv) | ((q.z == kv) & (jj + 2 < i));
        r3 += (q.w > kv) | ((q.w == kv) & (jj + 3 < i));
      }
      j = j1;
    }
    for (; j < j1; ++j) r0 += (skey[base + j] > kv) | ((skey[base + j] == kv) & (base + j < i));
    int rank = (r0 + r1) + (r2 + r3);
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    rank += __shfl_xor_sync(0xffffffffu, rank, 2);
    if (on && qt == 0 && rank < k) {
      if (nch == 1) {
        S.sidx[rank] = i;
      } else {
        ckey[(i >> 6) * k + rank] = kv;
        cidx[(i >> 6) * k + rank] = i;
      }
    }
  }
  if (nch > 1) {
    __syncthreads();
    for (int t = tid; t < ncand; t += kNT) {
      const int i = cidx[t];
      if (i < 0) continue;
      const float kv = ckey[t];
      int rank = 0;
      for (int u = 0; u < ncand; ++u) {
        const float q = ckey[u];
        const int j = cidx[u];
        rank += (j >= 0) & ((q > kv) | ((q == kv) & (j < i)));
      }
      if (rank < k) S.sidx[rank] = i;
    }
  }
  fence_async_smem();                       // this thread's ring accesses precede the bulk copies
  __syncthreads();
  // 5b. adaptive top-p: the kept prefix of the list (topk.cuh's rule; every CTA, same result)
  if constexpr (TOPP) {
    if (warp == 0) {
      const bool on = lane < k;
      const int ee = on ? S.sidx[lane] : 0;
      const float myl = (ee >= 0 && ee < E) ? slog[ee] : 0.0f;
      float v;
      if (r.score == 0) {
        const float lmax = __shfl_sync(0xffffffffu, myl, 0);
        v = on ? cexp(myl - lmax) : 0.0f;
      } else {
        v = on ? csigmoid(myl) : 0.0f;
      }
      float cm;
      const int m = topp_keep(v, k, r.top_p, cm);
      if (lane == 0) *S.nk = m;
    }
    __syncthreads();
  }
  // 6. the kept selection whose experts are held here (all of them without expert
  //    parallelism), by local id, in ascending order (all the producer needs): warp 0, one
  //    lane per slot of the list
  const int nk = TOPP ? *S.nk : k;
  if (warp == 0) {
    const int ee = lane < k ? S.sidx[lane] : -1;
    const int le = (lane < nk && ee >= r.e0 && ee < r.e0 + r.EL) ? ee - r.e0 : -1;
    int pos = 0;
    for (int i = 0; i < k; ++i) {
      const int o = __shfl_sync(0xffffffffu, le, i);
      pos += (o >= 0) & (o < le);
    }
    const int nl = __popc(__ballot_sync(0xffffffffu, le >= 0));
    S.lsel[lane] = le;
    if (le >= 0) {
      S.se[pos] = le;
      S.sj[pos] = lane;
      if (cta0) {
        r.g.act_expert[pos] = le;
        r.g.act_begin[pos] = pos;
        r.g.perm[pos] = lane;
        if (r.g.act_rows) r.g.act_rows[pos * 8] = 0;
      }
    }
    if (cta0 && lane < k) r.idx[lane] = lane < nk ? ee : -1;
    if (lane == 0) *S.nl = nl;
    __syncwarp();
    if (cta0) {
      for (int x = lane; x < r.EL; x += 32) {
        int cnt = 0;
        for (int i = 0; i < k; ++i) {
          const int o = S.lsel[i];
          cnt += (o >= 0) & (o < x);
        }
        r.g.offsets[x] = cnt;
      }
      if (lane == 0) {
        r.g.offsets[r.EL] = nl;
        *r.g.n_active = nl;
        r.g.act_begin[nl] = nl;
      }
    }
  }
  __syncthreads();
  return true;
}

// Warp 0 of the consumers, after route_one_token: routing weights of the k selected experts
// from the logits kept in activation buffer 1 -- softmax over the selected (renormalized) or
// over all E, or sigmoid scores (normalized over the selected), times the routed scaling
// factor (as in topk.cuh) -- into S.sw (selection order) and S.swt (ascending order).
template <bool TOPP>
__device__ __forceinline__ void route_weights(const RouteArgs& r, const RingPlan& P, const Ring& R,
                                              const RouteSmem& S) {
  const float* slogk = reinterpret_cast<const float*>(R.abuf + P.abytes);
  const int lane = threadIdx.x & 31, E = r.E, k = r.k;
  const bool on = lane < k;
  const int my_e = on ? S.sidx[lane] : 0;
  const float myl = (my_e >= 0 && my_e < E) ? slogk[my_e] : 0.0f;
  float v, den;                             // slot mass, weight denominator
  if (r.score == 0) {
    const float lmax = __shfl_sync(0xffffffffu, myl, 0);
    v = on ? cexp(myl - lmax) : 0.0f;
    if (r.renorm) {
      den = warp_sum(v);
    } else {
      float sacc = 0.0f;
      for (int x = lane; x < E; x += 32) sacc += cexp(slogk[x] - lmax);
      den = warp_sum(sacc);
    }
  } else {
    v = on ? csigmoid(myl) : 0.0f;
    den = r.renorm ? warp_sum(v) : 1.0f;
  }
  float wv = v / den * r.rsf;
  const int nk = TOPP ? *S.nk : k;          // adaptive top-p: the kept prefix (route_one_token)
  if (TOPP && r.renorm) {
    float cm;
    topp_keep(v, k, r.top_p, cm);
    wv = v / cm * r.rsf;
  }
  if (lane < nk) {
    S.sw[lane] = wv;
    const int le = kept_local(r, S, nk, lane);   // its weight goes with its unit (held here)
    if (le >= 0) S.swt[kept_local_rank(r, S, nk, le)] = wv;
  }
  if (on && blockIdx.x == 0) r.w[lane] = lane < nk ? wv : 0.0f;
  __syncwarp();
}

// Work unit u of a MODE 3 grid: routed units (the token's k experts, ascending) first, then
// the shared expert's. Slot of the routed pair = its active-expert index.
// nl: the token's kept slots whose experts are held here (all k without adaptive top-p or
// expert parallelism); units of the others are none.
template <bool TOPP>
__device__ __forceinline__ bool unit_of_token(const RingArgs& A, const RouteSmem& S, int nl, int u, Unit& U,
                                              bool report) {
  if (u < A.routed) {
    U.shd = false;
    U.ai = u / A.per;
    if (U.ai < A.r.k && U.ai >= nl) return false;   // dropped by top-p, or held elsewhere
    U.sub = u - U.ai * A.per;
    U.e = S.se[U.ai];
    U.s0 = U.ai;
    U.s1 = U.ai + 1;
#pragma unroll
    for (int q = 0; q < 8; ++q) U.rows8[q] = 0;
    if (U.ai >= A.r.k || U.e < 0 || U.e >= A.r.EL) {
      if (report) set_status(A.r.status, kStatusDeviceCheck);
      return false;
    }
    return true;
  }
  if (!A.has_shared) return false;
  U.shd = true;
  U.ai = 0;
  U.e = 0;
  U.s0 = 0;
  U.s1 = 1;
  U.sub = u - A.routed;
  return true;
}

// ------------------------------------------------------------------ producer
// Lane 0 of the producer warp: every chunk of every pass of every unit of this CTA, in the
// order the consumers take them. Gate/up pass: the unit's 128 rows over K = H (codes at
// gu_w + blk * KB, fp16 group scales at gu_s + blk * G * 2, blk = first row of the block),
// with the pass's activation rows right after the first chunk. Down pass: the unit's slab
// (all H rows x its 64 columns) in chunks of whole 128-row blocks, with their scales
// (fp16 [block][2][128] or fp32 per row).
template <int WBITS, bool WG32, bool AG32, int MODE, bool TOPP>
__device__ void ring_producer(const RingArgs& A, const RingPlan& P, const Ring& R, const RouteSmem& S) {
  constexpr int GPP4 = 16 / WBITS;          // 4 x groups per 16-byte piece (int8 2, int4 4, int2 8)
  constexpr int PPU = WBITS / 2;            // pieces of a row's 64-column down slice
  constexpr int NBC = kSP / PPU;            // 128-row down blocks per chunk
  constexpr int kern = MODE == 1 ? 2 : 1;
  int* status = A.x[0][0].status;
  uint32_t c = 0, pidx = 0, nacts = 0;      // chunks, passes, activation copies issued
  bool ok = true;
  const uint64_t once = policy_evict_first();
  auto push = [&](const uint8_t* w, uint32_t wbytes, const uint8_t* sc, uint32_t sbytes) -> bool {
    const int st = c % kNS;
    if (c >= (uint32_t)kNS && !mbar_wait(&R.empty[st], ((c / kNS) - 1) & 1)) {
      wait_failed(status, kern, 0, st);
      return false;
    }
    mbar_arrive_expect_tx(&R.full[st], wbytes + sbytes);
    bulk_load_hint(R.ring + st * (kSP * kPiece), w, wbytes, &R.full[st], once);
    if (sbytes) bulk_load_hint(R.sring + st * R.sstage, sc, sbytes, &R.full[st], once);
    ++c;
    return true;
  };
  const int nl = MODE == 3 ? *S.nl : 0;
  for (int u = blockIdx.x; u < A.units && ok; u += gridDim.x) {
    Unit U;
    if (MODE == 3 ? !unit_of_token<TOPP>(A, S, nl, u, U, false)
                  : !unit_of(A.x[0][0], A.x[0][1], A.has_shared, A.routed, A.per, u, U, MODE != 1, false,
                             A.mma_min))
      continue;
    const ExpertArgs& g = A.x[0][U.shd ? 1 : 0];
    const ExpertArgs& d = A.x[1][U.shd ? 1 : 0];
    for (int c0 = U.s0; c0 < U.s1 && ok; c0 += A.tm, ++pidx) {
      const int m = min(A.tm, U.s1 - c0);
      if (MODE != 1) {
        const int K = g.b.H, KB = kbytes(K, WBITS), NP = KB / 16, G = K / 32;
        const bool copy_scales = AG32 && (G % 8) == 0;
        const int64_t blk = (int64_t)U.e * 2 * g.b.I + (int64_t)U.sub * kRows;
        const uint8_t* wsrc = g.b.gu_w + blk * KB;
        const uint8_t* ssrc = g.b.gu_s + blk * G * 2;
        for (int p0 = 0; p0 < NP && ok; p0 += kSP) {
          const int np = min(kSP, NP - p0);
          ok = push(wsrc + (int64_t)p0 * kPiece, (uint32_t)np * kPiece,
                    ssrc + (int64_t)(p0 * GPP4 / 4) * 256, WG32 ? (uint32_t)(np * GPP4 / 4) * 256 : 0u);
          if (!ok || p0 != 0) continue;
          if (MODE == 3) continue;   // the CTA quantized the token's activations itself
          // this pass's activation rows, behind its first chunk
          const int b = pidx & 1;
          if (pidx >= 2 && !mbar_wait(&R.aempty[b], ((pidx >> 1) - 1) & 1)) {
            wait_failed(status, kern, 3, b);
            ok = false;
            break;
          }
          uint8_t* dst = R.abuf + b * P.abytes;
          const uint32_t bytes = (uint32_t)(m * K + (copy_scales ? m * G * 2 : 0));
          mbar_arrive_expect_tx(&R.afull[b], bytes);
          ++nacts;
          for (int tt = 0; tt < m; ++tt) {
            const int row = act_row(g, true, U, c0 + tt);
            bulk_load(dst + tt * K, g.qa + (int64_t)row * K, (uint32_t)K, &R.afull[b]);
            if (copy_scales)
              bulk_load(dst + P.ascale + tt * G * 2,
                        reinterpret_cast<const uint8_t*>(g.sa) + (int64_t)row * G * 2, (uint32_t)(G * 2),
                        &R.afull[b]);
          }
        }
      }
      if (MODE != 0 && ok) {
        const int HB = d.b.H / kRows;
        const int64_t slab0 = ((int64_t)U.e * (d.b.I / 64) + U.sub) * HB;   // first 128-row block
        const uint8_t* wsrc = d.b.dn_w + slab0 * PPU * kPiece;
        const uint8_t* ssrc = WG32 ? d.b.dn_s + slab0 * 512 : d.b.dn_s + (int64_t)U.e * d.b.H * 4;
        const int nch = (HB + NBC - 1) / NBC;
        const int rot = down_rotation(U, nch);
        for (int j = 0; j < nch && ok; ++j) {
          const int hb0 = ((j + rot) % nch) * NBC;
          const int nb = min(NBC, HB - hb0);
          ok = push(wsrc + (int64_t)hb0 * PPU * kPiece, (uint32_t)(nb * PPU * kPiece), ssrc + (int64_t)hb0 * 512,
                    (uint32_t)nb * 512);
        }
      }
    }
  }
  // drain: no copy may still be writing into this CTA's shared memory when it exits
  const uint32_t c0 = c > (uint32_t)kNS ? c - kNS : 0;
  for (uint32_t dd = c0; dd < c; ++dd)
    if (!mbar_wait(&R.full[dd % kNS], (dd / kNS) & 1)) {
      wait_failed(status, kern, 2, dd % kNS);
      break;
    }
  const uint32_t q0 = nacts > 2 ? nacts - 2 : 0;
  for (uint32_t dd = q0; dd < nacts; ++dd)
    if (!mbar_wait(&R.afull[dd & 1], (dd >> 1) & 1)) {
      wait_failed(status, kern, 4, dd & 1);
      break;
    }
}

// ------------------------------------------------------------------ consumers
// A chunk is consumed in blocks of 8 consecutive groups (int8: one block per chunk, int4:
// two). Dots: warp w takes group w of the block for all 128 rows (lane l: rows l, l+32,
// l+64, l+96), loads the block's activations once per token and writes each exact int32
// dot to idot[buffer][w][token][row]. One consumer barrier later, thread (row, token set)
// runs the ordered fp32 chain of its row over the block's 8 groups for its tokens
// (tokens ts, ts+2, ... with ts = thread / 128). idot is double-buffered, so the barrier
// after the next block's dots also orders this block's chain before the buffer is reused.
template <int WBITS, bool WG32, bool AG32, int TM>
__device__ __forceinline__ void block_dots(const uint8_t* stage, int j0, int gbase, int m, int tm,
                                           const uint8_t* xs, int K, const int* xsum, int G, int* idot) {
  constexpr int PPG = WBITS == 8 ? 2 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gg = j0 + warp;                            // this warp's group inside the chunk
  const int g = gbase + gg;                            // ... and inside the row
  // int8: two pieces per group, int4: one, int2: 8 bytes (half of one) of each row
  const uint8_t* wp = WBITS == 2 ? stage + (gg >> 1) * kPiece + lane * 16 + (gg & 1) * 8
                                 : stage + gg * PPG * kPiece + lane * 16;
  uint4 w[4 * PPG];
  uint2 w2[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (WBITS == 2) {
      w2[r] = *reinterpret_cast<const uint2*>(wp + r * 512);
    } else {
      w[r * PPG] = *reinterpret_cast<const uint4*>(wp + r * 512);
      if (WBITS == 8) w[r * PPG + 1] = *reinterpret_cast<const uint4*>(wp + kPiece + r * 512);
    }
  }
  int* out = idot + warp * tm * kRows + lane;
  const int mq = TM == 1 ? 1 : m;          // TM: compile-time bound on the pass's tokens
  for (int q = 0; q < mq; ++q) {
    const uint8_t* xg = xs + q * K + 32 * g;
    const uint4 x0 = *reinterpret_cast<const uint4*>(xg);
    const uint4 x1 = *reinterpret_cast<const uint4*>(xg + 16);
    int xsg = 0;
    if (WBITS != 8) xsg = xsum[q * G + g];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int d;
      if (WBITS == 8)
        d = group_dot_i8(w[2 * r], w[2 * r + 1], x0, x1);
      else if (WBITS == 4)
        d = group_dot_i4(w[r], make_uint4(x0.x, x0.z, x1.x, x1.z), make_uint4(x0.y, x0.w, x1.y, x1.w), xsg);
      else
        d = group_dot_i2(w2[r], x0, x1, xsg);   // activations de-interleaved per 16
      out[q * kRows + r * 32] = d;
    }
  }
}

template <int WBITS, bool WG32, bool AG32, int TM>
__device__ __forceinline__ void block_chain(const __half* sst, int j0, int gbase, int m, int tm, int G,
                                            const int* idot, const __half* sxh, const float* sxf,
                                            float acc[kTMP / 2], int isum[kTMP / 2]) {
  const int row = threadIdx.x & 127, ts = threadIdx.x >> 7;
  float sw[8];
  if (WG32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) sw[j] = __half2float(sst[(j0 + j) * 128 + row]);
  }
#pragma unroll
  for (int qq = 0; qq < (TM == 1 ? 1 : kTMP / 2); ++qq) {
    const int q = ts + 2 * qq;
    if (TM != 1 && q >= m) break;
    int d[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = idot[(j * tm + q) * kRows + row];
    if (!WG32 && !AG32) {
#pragma unroll
      for (int j = 0; j < 8; ++j) isum[qq] += d[j];
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int g = gbase + j0 + j;
        float sxg = 0.0f;
        if (AG32) sxg = sxh ? __half2float(sxh[q * G + g]) : sxf[q * G + g];
        float cg;
        if (WG32 && AG32) cg = __fmul_rn(sw[j], sxg);
        else if (WG32) cg = sw[j];
        else cg = sxg;
        acc[qq] = __fmaf_rn(exact_i2f(d[j]), cg, acc[qq]);
      }
    }
  }
}

// Consumes one pass (all chunks of the unit) and leaves the stage values of row
// (thread & 127) for tokens ts + 2 qq in v[qq]. After a wait gives up (`abort` set by any
// consumer), waits and compute are skipped but every stage is still released and every
// barrier taken, so the producer is never left waiting.
template <int WBITS, bool WG32, bool AG32, int TM>
__device__ __forceinline__ void ring_consume(int K, int m, int tm, const Ring& R, uint32_t& c, uint32_t& nblk,
                                             const uint8_t* xs, const __half* sxh, const float* sxf,
                                             const int* xsum, int* idot, float sw_row,
                                             float v[kTMP / 2], volatile int* abort, int* status,
                                             int kernel) {
  constexpr int GPP4 = 16 / WBITS;          // 4 x groups per 16-byte piece
  const int lane = threadIdx.x & 31;
  const int ts = threadIdx.x >> 7;
  const bool chain_thread = ts < m;
  const int KB = kbytes(K, WBITS), NP = KB / 16, G = K / 32;
  float acc[kTMP / 2];
  int isum[kTMP / 2];
#pragma unroll
  for (int q = 0; q < kTMP / 2; ++q) {
    acc[q] = 0.0f;
    isum[q] = 0;
  }
  for (int p0 = 0; p0 < NP; p0 += kSP, ++c) {
    const int np = min(kSP, NP - p0);
    const int st = c % kNS;
    bool ok = *abort == 0;
    if (ok && !mbar_wait(&R.full[st], (c / kNS) & 1)) {
      *abort = 1;
      if (lane == 0) wait_failed(status, kernel, 1, st);
      ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    const uint8_t* stage = R.ring + st * (kSP * kPiece);
    const __half* sst = reinterpret_cast<const __half*>(R.sring + st * R.sstage);
    const int gbase = p0 * GPP4 / 4, ng = np * GPP4 / 4;
    // blocks of 8 groups; a short last chunk (K a multiple of 128 but not of 256 / 512)
    // ends with a block of 4, handled by the first four warps and chain steps
    for (int j0 = 0; j0 < ng; j0 += 8, ++nblk) {
      const int nb = min(8, ng - j0);
      int* ib = idot + (nblk & 1) * (8 * tm * kRows);
      if (ok && (threadIdx.x >> 5) < nb) block_dots<WBITS, WG32, AG32, TM>(stage, j0, gbase, m, tm, xs, K, xsum, G, ib);
      named_bar(1, 32 * kCW);
      if (ok && chain_thread) {
        if (nb == 8) {
          block_chain<WBITS, WG32, AG32, TM>(sst, j0, gbase, m, tm, G, ib, sxh, sxf, acc, isum);
        } else {
          // 4-group tail: same chain, groups j0 .. j0+3 only
          const int row = threadIdx.x & 127;
          for (int qq = 0; qq < kTMP / 2; ++qq) {
            const int q = ts + 2 * qq;
            if (q >= m) break;
            for (int j = 0; j < nb; ++j) {
              const int g = gbase + j0 + j;
              const int d = ib[(j * tm + q) * kRows + row];
              if (!WG32 && !AG32) {
                isum[qq] += d;
              } else {
                const float swg = WG32 ? __half2float(sst[(j0 + j) * 128 + row]) : 0.0f;
                float sxg = 0.0f;
                if (AG32) sxg = sxh ? __half2float(sxh[q * G + g]) : sxf[q * G + g];
                float cg;
                if (WG32 && AG32) cg = __fmul_rn(swg, sxg);
                else if (WG32) cg = swg;
                else cg = sxg;
                acc[qq] = __fmaf_rn(exact_i2f(d), cg, acc[qq]);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&R.empty[st]);
  }
#pragma unroll
  for (int qq = 0; qq < kTMP / 2; ++qq) {
    const int q = ts + 2 * qq;
    const float sxt = (!AG32 && q < m) ? sxf[q] : 0.0f;
    if (WG32 && AG32) v[qq] = acc[qq];
    else if (WG32) v[qq] = __fmul_rn(acc[qq], sxt);
    else if (AG32) v[qq] = __fmul_rn(acc[qq], sw_row);
    else v[qq] = __fmul_rn(__fmaf_rn(__int2float_rn(isum[qq]), sxt, 0.0f), sw_row);
  }
}

// Down pass of one unit: the slab's 128-row blocks arrive a chunk at a time; thread t takes
// rows t, t + 256, ... of the chunk (int8: 2 rows, int4: 4). Per (row, token) the two group
// dots against the unit's 64 h codes give this unit's share of the row's down value
// (fp32, any order), weighted and added into y (and, for inspection, into the pair's
// down value, and its two exact group dots into the debug view [slot][H][I/32] at groups
// 2 sub, 2 sub + 1). hx: the pass's h codes [tm][64] (int4 weights: each 8-byte word
// de-interleaved), hxs: per-group code sums [tm][2] (int4), hs: h scales [tm][2].
template <int WBITS, bool WG32, bool AG32, int TM>
__device__ __forceinline__ void down_consume(int H, int m, int rot, const Ring& R, uint32_t& c, const uint8_t* hx,
                                             const int* hxs, const float* hs, const int* toks,
                                             const float* wts, float* y, float* dbg, int32_t* ddots, int GI,
                                             int sub, int slot0, volatile int* abort, int* status) {
  constexpr int PPU = WBITS / 2;                  // pieces of a row's 64 columns
  constexpr int NBC = kSP / PPU;
  constexpr int RPT = NBC * kRows / (32 * kCW);   // rows per thread of a full chunk
  const int lane = threadIdx.x & 31;
  const int HB = H / kRows;
  const int nch = (HB + NBC - 1) / NBC;
  for (int j = 0; j < nch; ++j, ++c) {
    const int hb0 = ((j + rot) % nch) * NBC;
    const int nb = min(NBC, HB - hb0);
    const int st = c % kNS;
    bool ok = *abort == 0;
    if (ok && !mbar_wait(&R.full[st], (c / kNS) & 1)) {
      *abort = 1;
      if (lane == 0) wait_failed(status, 2, 1, st);
      ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      const uint8_t* stage = R.ring + st * (kSP * kPiece);
      const uint8_t* sst = R.sring + st * R.sstage;
      uint4 w[RPT][PPU];
      float c0s[RPT], c1s[RPT];
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int rr = threadIdx.x + 32 * kCW * k, b = rr >> 7, r = rr & 127;
        if (b < nb) {
#pragma unroll
          for (int p = 0; p < PPU; ++p)
            w[k][p] = *reinterpret_cast<const uint4*>(stage + ((b * PPU + p) * kRows + r) * 16);
          if (WG32) {
            const __half* sh = reinterpret_cast<const __half*>(sst);
            c0s[k] = __half2float(sh[(b * 2) * kRows + r]);
            c1s[k] = __half2float(sh[(b * 2 + 1) * kRows + r]);
          } else {
            c0s[k] = c1s[k] = reinterpret_cast<const float*>(sst)[b * kRows + r];
          }
        }
      }
      for (int q = 0; q < (TM == 1 ? 1 : m); ++q) {
        const uint4* xq = reinterpret_cast<const uint4*>(hx + q * 64);
        const uint4 x0 = xq[0], x1 = xq[1], x2 = xq[2], x3 = xq[3];
        const float hs0 = hs[2 * q], hs1 = hs[2 * q + 1];
        const float wq = wts[q];
        float* yq = y + (int64_t)toks[q] * H;
        float* dq = dbg ? dbg + (int64_t)(slot0 + q) * H : nullptr;
        int32_t* tq = ddots ? ddots + (int64_t)(slot0 + q) * H * GI + 2 * sub : nullptr;
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
          const int rr = threadIdx.x + 32 * kCW * k, b = rr >> 7, r = rr & 127;
          if (b >= nb) break;
          int d0, d1;
          if (WBITS == 8) {
            d0 = group_dot_i8(w[k][0], w[k][1], x0, x1);
            d1 = group_dot_i8(w[k][2], w[k][3], x2, x3);
          } else if (WBITS == 4) {
            d0 = group_dot_i4(w[k][0], make_uint4(x0.x, x0.z, x1.x, x1.z), make_uint4(x0.y, x0.w, x1.y, x1.w),
                              hxs[2 * q]);
            d1 = group_dot_i4(w[k][1], make_uint4(x2.x, x2.z, x3.x, x3.z), make_uint4(x2.y, x2.w, x3.y, x3.w),
                              hxs[2 * q + 1]);
          } else {
            // int2: the row's 64 codes are one piece, h de-interleaved per 16
            d0 = group_dot_i2(make_uint2(w[k][0].x, w[k][0].y), x0, x1, hxs[2 * q]);
            d1 = group_dot_i2(make_uint2(w[k][0].z, w[k][0].w), x2, x3, hxs[2 * q + 1]);
          }
          float v;
          if (WG32 && AG32)
            v = __fmaf_rn(__int2float_rn(d1), __fmul_rn(c1s[k], hs1), __fmul_rn(__int2float_rn(d0), __fmul_rn(c0s[k], hs0)));
          else if (WG32)
            v = __fmul_rn(__fmaf_rn(__int2float_rn(d1), c1s[k], __fmul_rn(__int2float_rn(d0), c0s[k])), hs0);
          else if (AG32)
            v = __fmul_rn(__fmaf_rn(__int2float_rn(d1), hs1, __fmul_rn(__int2float_rn(d0), hs0)), c0s[k]);
          else
            v = __fmul_rn(__fmul_rn(__int2float_rn(d0 + d1), hs0), c0s[k]);
          const int n = (hb0 + b) * kRows + r;
          // lanes 4j .. 4j+3 hold rows n .. n+3: one 16-byte reduction per four rows
          const float wv = wq * v;
          const float w1 = __shfl_down_sync(0xffffffffu, wv, 1);
          const float w2 = __shfl_down_sync(0xffffffffu, wv, 2);
          const float w3 = __shfl_down_sync(0xffffffffu, wv, 3);
          if ((lane & 3) == 0) red_add_v4(yq + n, wv, w1, w2, w3);
          if (dq) atomicAdd(dq + n, v);
          if (tq) {
            tq[(int64_t)n * GI] = d0;
            tq[(int64_t)n * GI + 1] = d1;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&R.empty[st]);
  }
}

// ------------------------------------------------------------------ kernel
// Per unit and pass: the gate/up pass (consumer warps of ring_consume; after it the gate and
// up stage values meet in shared memory and warps 0 and 1 apply SwiGLU and quantize h per
// group of 32 -- one warp per group), then the down pass over the unit's slab with the
// pass's h codes from shared memory (MODE 2) or from the workspace (MODE 1).
template <int WBITS, bool WG32, bool AG32, int MODE, int TM, bool TOPP>
__global__ void __launch_bounds__(kNT, 1) k_expert_ring(const __grid_constant__ RingArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  const RingPlan P = ring_plan(A.kmax, A.tm, WBITS, MODE == 3 ? rs_total(A.rs) : 0);
  Ring R;
  R.ring = base + P.ring;
  R.sring = base + P.sring;
  R.sstage = P.sstage;
  R.full = reinterpret_cast<uint64_t*>(base + P.bars);
  R.empty = R.full + kNS;
  R.afull = R.empty + kNS;
  R.aempty = R.afull + 2;
  R.abuf = base + P.abuf;
  R.xsum = reinterpret_cast<int*>(base + P.xsum);
  R.sxf = reinterpret_cast<float*>(base + P.sxf);
  int* idot = reinterpret_cast<int*>(base + P.idot);
  float* gbuf = reinterpret_cast<float*>(base + P.ubuf);
  float* ubuf = gbuf + A.tm * 64;
  uint8_t* hq = base + P.hq;                       // [tm][64] h codes of the pass
  uint8_t* hqd = hq + A.tm * 64;                   // [tm][64] de-interleaved (int4 weights)
  float* hs = reinterpret_cast<float*>(hqd + A.tm * 64);   // [tm][2] h scales
  int* hxs = reinterpret_cast<int*>(hs + 2 * A.tm);        // [tm][2] code sums
  int* toks = reinterpret_cast<int*>(base + P.info);
  float* wts = reinterpret_cast<float*>(toks + kTMP);
  volatile int* abort = toks + 3 * kTMP;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = A.x[0][0].status;

  // single-token routing, grid exchange with at most two experts per CTA: the CTA's router
  // chunks straight into registers; else (cluster exchange, or more experts) staged rows
  RowChunks pf;
  const bool reg_rows = MODE == 3 && !A.cluster && owned_experts(A.r.E, route_owners(false)) <= 2;
  if (reg_rows) prefetch_router_chunks(A.r, pf);   // in flight during the start-up
  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&R.full[s], 1);
      mbar_init(&R.empty[s], kCW);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&R.afull[b], 1);
      mbar_init(&R.aempty[b], kCW);
    }
    fence_barrier_init();
  }
  RouteSmem S;
  S.se = reinterpret_cast<int*>(base + P.route);
  S.swt = reinterpret_cast<float*>(S.se + 32);
  S.sj = S.se + 64;
  S.sidx = S.se + 96;
  S.sw = S.swt + 96;
  S.own = S.swt + 128;
  S.flag = reinterpret_cast<volatile int*>(S.se + 192);
  volatile int* rows_flag = S.se + 193;
  S.ytarget = reinterpret_cast<volatile unsigned long long*>(S.se + 194);
  S.nk = S.se + 196;
  S.nl = S.se + 197;
  S.lsel = S.se + 200;
  __syncthreads();
  bool rows = false;
  if (MODE == 3) {
    if (!reg_rows) rows = stage_router_rows(A.r, A.cluster != 0, R.ring, &R.afull[0], rows_flag, A.rs.rows);
  }
  pdl_wait();
  if (MODE == 3) {
    // one token: routing first. Its grid barrier also means every CTA of this grid is
    // resident before any CTA lets the next kernel launch (and take SMs).
    if (!route_one_token<TOPP>(A.r, P, R, S, rows ? &R.afull[0] : nullptr, A.cluster != 0, A.rs, pf, reg_rows)) {
      if (A.cluster) cluster_wait();
      return;
    }
  }
  // single token: the next kernel may launch once every CTA of this grid is resident, after
  // the routing's grid barrier (with the cluster exchange after the y-zero barrier, consumers,
  // below). The batch modes let it launch when this grid completes: launched early, its CTAs
  // took SMs this grid still needed (measured on graph-replayed steps: -2.1 % at OLMoE int8
  // T = 8, -2.6 % at GLM int4 T = 4, no change at T = 4096) -- except before the host-buffer
  // path's small output copy, which is better launched early
  if (MODE == 3 ? !A.cluster : A.x[0][0].early_trigger != 0) pdl_trigger();

  if (warp == kCW) {
    if (lane == 0) ring_producer<WBITS, WG32, AG32, MODE, TOPP>(A, P, R, S);
    if (MODE == 3 && A.cluster) {
      __syncwarp();
      cluster_wait();                      // peers are done reading this CTA's logits
    }
    return;
  }

  const int ctid = threadIdx.x;             // consumer thread index, [0, 256)
  const int row = ctid & 127, ts = ctid >> 7;  // chain row, first token (tokens ts + 2 qq)
  const int tm = A.tm;
  uint32_t c = 0, pidx = 0, nblk = 0;       // chunks, gate/up passes, 8-group blocks consumed
  bool ywait = !(MODE == 3 && A.cluster);   // cluster exchange: y-zero barrier still to wait on
  if (MODE == 3) {
    // off the path to the first weight copy: the routing weights (read only by this warp's
    // ctid 0) and, int4 / int2 weights, the token's de-interleaved codes and group sums
    if (warp == 0) route_weights<TOPP>(A.r, P, R, S);
    if (WBITS != 8) {
      if (WBITS == 4) act_deinterleave(R.abuf, A.kmax / 8, ctid, 32 * kCW);
      else act_deinterleave16(R.abuf, A.kmax / 16, ctid, 32 * kCW);
      named_bar(1, 32 * kCW);
      act_group_sums(R.abuf, R.xsum, 1, A.kmax, ctid, 32 * kCW);
    }
  }
  const int nl = MODE == 3 ? *S.nl : 0;
  for (int u = blockIdx.x; u < A.units; u += gridDim.x) {
    Unit U;
    if (MODE == 3 ? !unit_of_token<TOPP>(A, S, nl, u, U, ctid == 0)
                  : !unit_of(A.x[0][0], A.x[0][1], A.has_shared, A.routed, A.per, u, U, MODE != 1, ctid == 0,
                             A.mma_min))
      continue;
    const ExpertArgs& g = A.x[0][U.shd ? 1 : 0];
    const ExpertArgs& d = A.x[1][U.shd ? 1 : 0];
    const int I = g.b.I, IB = I / 32;
    for (int c0 = U.s0; c0 < U.s1; c0 += tm) {
      const int m = min(tm, U.s1 - c0);
      named_bar(1, 32 * kCW);              // previous pass done with the per-pass arrays
      if (ctid < m) {
        const int slot = c0 + ctid;
        if (MODE == 3) {
          toks[ctid] = 0;
          wts[ctid] = U.shd ? 1.0f : S.swt[U.ai];
        } else if (MODE != 0) {
          int p = U.shd ? slot : __ldcg(d.perm + slot);
          if (p < 0 || p >= (U.shd ? d.T : d.T * d.k)) {
            set_status(status, kStatusDeviceCheck);
            p = 0;
          }
          toks[ctid] = U.shd ? slot : p / d.k;
          wts[ctid] = U.shd ? 1.0f : d.wts[p];
        }
        if (MODE != 1 && !AG32) R.sxf[ctid] = reinterpret_cast<const float*>(g.sa)[act_row(g, true, U, slot)];
      }
      if (MODE == 1) {
        // h of this unit's 64 columns, written by the gate/up and h-quantization kernels
        if (ctid < 4 * m) {
          const int q = ctid >> 2, part = ctid & 3;
          reinterpret_cast<uint4*>(hq + q * 64)[part] =
              *reinterpret_cast<const uint4*>(d.qa + (int64_t)(c0 + q) * I + U.sub * 64 + part * 16);
        }
        if (ctid < 2 * m) {
          const int q = ctid >> 1, j = ctid & 1;
          hs[ctid] = AG32 ? __half2float(reinterpret_cast<const __half*>(d.sa)[(int64_t)(c0 + q) * IB + 2 * U.sub + j])
                          : reinterpret_cast<const float*>(d.sa)[c0 + q];
        }
      }
      if (MODE != 1) {
        const int K = g.b.H, G = K / 32;
        // MODE 3: buffer 0 holds the token's codes and fp16 scales (and int4 prep) already
        const bool copy_scales = MODE == 3 || (AG32 && (G % 8) == 0);
        const int b = MODE == 3 ? 0 : pidx & 1;
        if (AG32 && !copy_scales)
          for (int l = ctid; l < m * G; l += 32 * kCW) {
            const int tt = l / G, gg = l - tt * G;
            const int r = act_row(g, true, U, c0 + tt);
            R.sxf[l] = __half2float(reinterpret_cast<const __half*>(g.sa)[(int64_t)r * G + gg]);
          }
        uint8_t* xs = R.abuf + b * P.abytes;
        int* xsum = R.xsum + b * tm * G;
        bool aok = *abort == 0;
        if (MODE != 3 && aok && !mbar_wait(&R.afull[b], (pidx >> 1) & 1)) {
          *abort = 1;
          if (lane == 0) wait_failed(status, 1, 5, b);
          aok = false;
        }
        if (WBITS != 8 && MODE != 3) {
          // de-interleave each 8-byte word into even / odd elements (int4) or each 16-byte
          // word by fours (int2); per-group sums (barriers taken by every consumer thread,
          // whatever its wait returned)
          if (aok) {
            if (WBITS == 4) act_deinterleave(xs, m * (K / 8), ctid, 32 * kCW);
            else act_deinterleave16(xs, m * (K / 16), ctid, 32 * kCW);
          }
          named_bar(1, 32 * kCW);
          if (aok) act_group_sums(xs, xsum, m, K, ctid, 32 * kCW);
        }
        named_bar(1, 32 * kCW);
        const __half* sxh = copy_scales ? reinterpret_cast<const __half*>(xs + P.ascale) : nullptr;
        const int64_t blk = (int64_t)U.e * 2 * I + (int64_t)U.sub * kRows;
        const float sw_row = WG32 ? 0.0f : reinterpret_cast<const float*>(g.b.gu_s)[blk + row];
        float v[kTMP / 2];
        ring_consume<WBITS, WG32, AG32, TM>(K, m, tm, R, c, nblk, xs, sxh, R.sxf, xsum, idot, sw_row, v, abort,
                                        status, 1);
        __syncwarp();
        if (MODE != 3 && lane == 0) mbar_arrive(&R.aempty[b]);
        ++pidx;
        const bool is_up = row >= 64;
#pragma unroll
        for (int qq = 0; qq < kTMP / 2; ++qq) {
          const int q = ts + 2 * qq;
          if (q < m) {
            if (g.dbg_a) (is_up ? g.dbg_b : g.dbg_a)[(int64_t)(c0 + q) * I + U.sub * 64 + (row & 63)] = v[qq];
            (is_up ? ubuf : gbuf)[q * 64 + (row & 63)] = v[qq];
          }
        }
        named_bar(1, 32 * kCW);
        if (warp < 2) {
          // SwiGLU and h quantization: warp w takes the group of 32 indices w * 32 ..
          const int il = warp * 32 + lane, i = U.sub * 64 + il;
          for (int q = 0; q < m; ++q) {
            const int slot = c0 + q;
            const float h = cswiglu(gbuf[q * 64 + il], ubuf[q * 64 + il]);
            if (AG32) {
              const float sc = f16_round(__fdiv_rn(warp_max(fabsf(h)), 127.0f));
              const int code = quant_code(h, sc, 127.0f);
              g.qh[(int64_t)slot * I + i] = (int8_t)code;
              if (lane == 0) g.sh[(int64_t)slot * IB + i / 32] = __float2half_rn(sc);
              if (MODE >= 2) {              // h stays on chip for the down pass
                hq[q * 64 + il] = (uint8_t)(int8_t)code;
                if (lane == 0) hs[2 * q + warp] = sc;
              }
            } else {
              g.hbuf[(int64_t)slot * I + i] = h;
            }
          }
        }
      }
      if (MODE != 0) {
        if (!ywait) {
          // y-zero barrier, second half, before this CTA's first add into y (long done by now:
          // every CTA arrived right after zeroing its share, before its first gate/up pass)
          if (ctid == 0) {
            const bool ok = wait_counter(A.r.gbar, *S.ytarget, A.r.wait_ns);
            if (!ok) {
              *abort = 1;
              wait_failed(status, 1, 8, 0);
            }
          }
          ywait = true;
          named_bar(1, 32 * kCW);
          pdl_trigger();
        }
        named_bar(1, 32 * kCW);            // h codes / scales of the pass in shared memory
        const uint8_t* hx = hq;
        if (WBITS != 8) {
          // the h codes in the order of the packed weights' fields, and their group sums
          if (WBITS == 4 && ctid < 8 * m) {
            const uint2 v = reinterpret_cast<const uint2*>(hq)[ctid];
            uint2 o;
            deinterleave8(v.x, v.y, o.x, o.y);
            reinterpret_cast<uint2*>(hqd)[ctid] = o;
          }
          if (WBITS == 2 && ctid < 4 * m)
            reinterpret_cast<uint4*>(hqd)[ctid] = deinterleave16(reinterpret_cast<const uint4*>(hq)[ctid]);
          if (ctid < 2 * m) {
            const uint4* q4 = reinterpret_cast<const uint4*>(hq + ctid * 32);
            hxs[ctid] = code_sum32(q4[0], q4[1]);
          }
          named_bar(1, 32 * kCW);
          hx = hqd;
        }
        constexpr int NBC = kSP / (WBITS / 2);   // 128-row down blocks per chunk
        const int rot = down_rotation(U, (d.b.H / kRows + NBC - 1) / NBC);
        down_consume<WBITS, WG32, AG32, TM>(d.b.H, m, rot, R, c, hx, hxs, hs, toks, wts, d.y, d.dbg_a, d.dbg_dots,
                                            d.b.I / 32, U.sub, c0, abort, status);
      }
    }
  }
  if (MODE == 3 && A.cluster) cluster_wait();   // peers are done reading this CTA's logits
}

// ------------------------------------------------------------------ host side
namespace {

int sm_count() { return device_sm_count(); }

// MODE 3 grid: every unit its CTA, and at least one CTA per expert for the router logits (up
// to one CTA per SM: the grid barrier needs all of them resident at once).
int decode_grid(int units, int E) { return std::min(sm_count(), std::max(units, E)); }

template <int WBITS, bool WG32, bool AG32, int MODE, int TM, bool TOPP = false>
cudaError_t launch_ring_t(const RingArgs& A, cudaStream_t st) {
  const RingPlan P = ring_plan(A.kmax, A.tm, WBITS);
  if constexpr (MODE != 3) {
    const cudaError_t e = ensure_smem_attr((const void*)k_expert_ring<WBITS, WG32, AG32, MODE, TM, TOPP>, P.total);
    if (e != cudaSuccess) return e;
  }
  if constexpr (MODE == 3) {
    // one token: the logits shared per cluster (of 16 or 8 CTAs, every CTA staging the router
    // rows of E / cluster experts) when every cluster of the grid can be resident at
    // once (the y-zero barrier waits on all CTAs) with no fewer CTAs than the grid exchange
    // would use; else every CTA computes some logits and a grid barrier follows
    auto kern = k_expert_ring<WBITS, WG32, AG32, MODE, TM, TOPP>;
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    const int C = A.r.H / 32, sms = sm_count();
    const int grid_x = decode_grid(A.units, A.r.E);          // grid exchange
    const int need = std::min(std::max(A.units, 1), sms);
    int cs_best = 0, cgrid = 0, csmem = 0;
    RouteScratch crs{};
    // (clusters of 4 were measured slower at the OLMoE shape: staging 16 experts' router rows
    // as 128-byte copies takes ~5 us of copy issue per CTA)
    for (int cs : {16, 8}) {
      const int ne = (A.r.E + cs - 1) / cs;
      if (ne > 32) continue;                                   // S.own holds 32 logits
      const RouteScratch rs = cluster_scratch(ne, C);
      const int smem = ring_plan(A.kmax, A.tm, WBITS, rs_total(rs)).total;
      if (smem > kSmemMax) continue;
      const int mc = max_active_clusters((const void*)kern, dev, cs, smem, kNT);
      const int want = (std::max(A.units, 1) + cs - 1) / cs;
      const int g = cs * std::min({want, mc, sms / cs});
      if (g >= need && (cs_best == 0 || g < cgrid)) {
        cs_best = cs;
        cgrid = g;
        csmem = smem;
        crs = rs;
      }
    }
    RingArgs B = A;
    B.cluster = cs_best;
    if (!B.cluster) {
      // Plain (programmatic) launch: the grid is at most one CTA per SM and one CTA fits an SM,
      // so on an otherwise idle GPU every CTA is resident; if other work holds SMs, the
      // bounded grid-barrier wait returns MOE_ERR_TIMEOUT rather than hanging. (A cooperative
      // launch would guarantee residency, but measured it cannot start while the host path's
      // input-copy kernel still holds SMs: 3 us more per step there.)
      B.rs = grid_scratch();
      const int smem = ring_plan(A.kmax, A.tm, WBITS, rs_total(B.rs)).total;
      const cudaError_t e = ensure_smem_attr((const void*)kern, smem);
      if (e != cudaSuccess) return e;
      return launch_pdl(kern, dim3(grid_x), dim3(kNT), (size_t)smem, st, B);
    }
    B.rs = crs;
    {
      const cudaError_t e = ensure_smem_attr((const void*)kern, csmem);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs_best;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(cgrid);
    cfg.blockDim = dim3(kNT);
    cfg.dynamicSmemBytes = (size_t)csmem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = kUsePdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, B);
  } else {
    const int grid = std::min(A.units, sm_count());
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(k_expert_ring<WBITS, WG32, AG32, MODE, TM, TOPP>, dim3(grid), dim3(kNT), (size_t)P.total, st,
                      A);
  }
}

template <int WBITS, bool WG32, bool AG32, int TM>
cudaError_t launch_mode_tm(int mode, const RingArgs& A, cudaStream_t st) {
  if (mode == 0) return launch_ring_t<WBITS, WG32, AG32, 0, TM>(A, st);
  if (mode == 1) return launch_ring_t<WBITS, WG32, AG32, 1, TM>(A, st);
  if constexpr (AG32) return launch_ring_t<WBITS, WG32, AG32, 2, TM>(A, st);
  return cudaErrorInvalidValue;               // the fused mode needs group-32 activations
}

// One token per pass (decode) gets consumers compiled for exactly one token.
template <int WBITS, bool WG32, bool AG32>
cudaError_t launch_mode(int mode, const RingArgs& A, cudaStream_t st) {
  return A.tm == 1 ? launch_mode_tm<WBITS, WG32, AG32, 1>(mode, A, st)
                   : launch_mode_tm<WBITS, WG32, AG32, kTMP>(mode, A, st);
}

// Adaptive top-p gets its own instantiation, so the plain single-token kernel carries none of it.
template <int WBITS, bool WG32>
cudaError_t launch_decode_t(const RingArgs& A, cudaStream_t st) {
  return A.r.top_p > 0.0f ? launch_ring_t<WBITS, WG32, true, 3, 1, true>(A, st)
                          : launch_ring_t<WBITS, WG32, true, 3, 1, false>(A, st);
}

}  // namespace

bool experts_fusable(const ExpertArgs& r, const ExpertArgs* s) {
  (void)s;
  return r.ag32 != 0;
}

cudaError_t launch_experts(int mode, const ExpertArgs& gr, const ExpertArgs* gs, const ExpertArgs& dr,
                           const ExpertArgs* ds, int mma_min, cudaStream_t st) {
  RingArgs A;
  std::memset(&A, 0, sizeof(A));
  A.x[0][0] = gr;
  A.x[0][1] = gs ? *gs : gr;
  A.x[1][0] = dr;
  A.x[1][1] = ds ? *ds : dr;
  A.has_shared = gs != nullptr;
  A.per = gr.b.I / 64;
  A.routed = gr.max_active * A.per;
  A.units = A.routed + (gs ? gs->b.I / 64 : 0);
  A.kmax = mode == 1 ? 64 : gr.b.H;           // K of the staged activation rows
  A.tm = ring_tokens(A.kmax, gr.T, gr.b.wbits);
  A.mma_min = mma_min;
  const int sel = (gr.b.wbits == 8 ? 4 : gr.b.wbits == 2 ? 8 : 0) | (gr.b.wg32 ? 2 : 0) | (gr.ag32 ? 1 : 0);
  switch (sel) {
    case 11: return launch_mode<2, true, true>(mode, A, st);
    case 10: return launch_mode<2, true, false>(mode, A, st);
    case 9: return launch_mode<2, false, true>(mode, A, st);
    case 8: return launch_mode<2, false, false>(mode, A, st);
    case 7: return launch_mode<8, true, true>(mode, A, st);
    case 6: return launch_mode<8, true, false>(mode, A, st);
    case 5: return launch_mode<8, false, true>(mode, A, st);
    case 4: return launch_mode<8, false, false>(mode, A, st);
    case 3: return launch_mode<4, true, true>(mode, A, st);
    case 2: return launch_mode<4, true, false>(mode, A, st);
    case 1: return launch_mode<4, false, true>(mode, A, st);
    default: return launch_mode<4, false, false>(mode, A, st);
  }
}

bool decode_fusable(const RouteArgs& r, const ExpertArgs& gr, const ExpertArgs* gs) {
  if (r.T != 1 || !experts_fusable(gr, gs) || !r.ag32 || r.E > 512 || r.k > 32 || r.H != gr.b.H ||
      r.H % 128 != 0 || 4 * r.E > r.H || !r.gbar)   // the logits also fit activation buffer 1
    return false;
  return r.H / 32 <= kPartFloats;   // one expert's chunk partials fit the ring scratch
}

cudaError_t launch_decode(const RouteArgs& r, const ExpertArgs& gr, const ExpertArgs* gs, const ExpertArgs& dr,
                          const ExpertArgs* ds, cudaStream_t st) {
  if (!decode_fusable(r, gr, gs)) return cudaErrorInvalidValue;
  RingArgs A;
  std::memset(&A, 0, sizeof(A));
  A.x[0][0] = gr;
  A.x[0][1] = gs ? *gs : gr;
  A.x[1][0] = dr;
  A.x[1][1] = ds ? *ds : dr;
  A.has_shared = gs != nullptr;
  A.per = gr.b.I / 64;
  A.routed = r.k * A.per;
  A.units = A.routed + (gs ? gs->b.I / 64 : 0);
  A.kmax = gr.b.H;
  A.tm = 1;
  A.mma_min = 0x7fffffff;
  A.r = r;
  const int sel = (gr.b.wbits == 8 ? 2 : gr.b.wbits == 2 ? 4 : 0) | (gr.b.wg32 ? 1 : 0);
  switch (sel) {
    case 5: return launch_decode_t<2, true>(A, st);
    case 4: return launch_decode_t<2, false>(A, st);
    case 3: return launch_decode_t<8, true>(A, st);
    case 2: return launch_decode_t<8, false>(A, st);
    case 1: return launch_decode_t<4, true>(A, st);
    default: return launch_decode_t<4, false>(A, st);
  }
}

}  // namespace moe
