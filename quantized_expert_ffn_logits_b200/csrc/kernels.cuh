// kernels.cuh -- launch wrappers of the device kernels (host-side declarations).
#pragma once

#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

// ---- host_setup.cu: per-device host-side setup (attributes and properties are per device;
// the caches are keyed by the current device and guarded by setup_mutex())
constexpr int kMaxDevices = 64;
int current_device();                                   // -1 if unknown or >= kMaxDevices
int device_sm_count();                                  // SMs of the current device
cudaError_t ensure_smem_attr(const void* kernel, int bytes);   // dynamic smem limit >= bytes
// Most co-resident clusters of `cluster` CTAs of `threads` threads and `smem` bytes (cached).
int max_active_clusters(const void* kernel, int dev, int cluster, int smem, int threads);
std::mutex& setup_mutex();

// ---- quantize.cu
void launch_quantize_experts(const float* w_gu, const float* w_dn, const BlobView& b,
                             uint8_t* gu_w, uint8_t* dn_w, uint8_t* gu_s, uint8_t* dn_s,
                             cudaStream_t st);
// FP8 checkpoint weights: E4M3 codes [E][2I][H] / [E][H][I] with fp32 inverse scales per
// 128 x 128 block, [E][ceil(2I/128)][ceil(H/128)] / [E][ceil(H/128)][ceil(I/128)].
void launch_quantize_experts_fp8(const uint8_t* w_gu, const float* s_gu, const uint8_t* w_dn,
                                 const float* s_dn, const BlobView& b, uint8_t* gu_w, uint8_t* dn_w,
                                 uint8_t* gu_s, uint8_t* dn_s, cudaStream_t st);
// y_zero (optional): output rows to zero; status (optional): status word to reset.
void launch_quantize_act(const float* x, int T, int H, int g32, int8_t* q, void* scales,
                         float* y_zero, int* status, cudaStream_t st);
void launch_quantize_rows_token(const float* h, int rows, int K, int8_t* q, float* scales,
                                cudaStream_t st);

// ---- router.cu
void launch_router_logits(const float* x, const float* wr, int T, int E, int H, float* logits,
                          cudaStream_t st);

struct Grouping {            // batch-union grouping outputs (all device pointers)
  int32_t* offsets;          // [E+1]
  int32_t* perm;             // [T*k]
  int32_t* n_active;         // [1]
  int32_t* act_expert;       // [E]
  int32_t* act_begin;        // [E+1]
  int32_t* act_rows;         // [E][8] token of each active expert's first 8 slots (or null)
};

// top_p: adaptive expert top-p threshold in (0, 1), 0 = off (dropped slots: idx -1, w 0).
void launch_topk(const float* logits, const float* bias, int T, int E, int k, int score,
                 int renorm, float rsf, float top_p, int32_t* idx, float* w, const Grouping* single_token,
                 int* status, cudaStream_t st);
// Pairs with expert -1 (dropped by adaptive top-p) are left out of the grouping, and so are
// pairs whose global expert id lies outside e0 .. e0 + E - 1 (held elsewhere: expert
// parallelism); the grouping uses local ids (global - e0). Ids outside [0, e_total) are
// reported (device check) and dropped. masks/base: scratch [ceil(T/32)][E] each.
// reset_status: clear the status word first (stand-alone use).
void launch_permute(const int32_t* idx, int T, int k, int E, int e0, int e_total, const Grouping& g,
                    uint32_t* masks, int32_t* base, int* status, int reset_status, cudaStream_t st);

// ---- expert_stream.cu (weight-streaming expert kernels)
struct ExpertArgs {
  BlobView b;
  // activation rows: gate/up reads q_x rows (one per token); down reads q_h rows (one per slot)
  const int8_t* qa;
  const void* sa;            // fp16 [rows][K/32] or fp32 [rows]
  int ag32;
  // grouping: routed experts when act_expert != nullptr, else one expert (index 0) applied
  // to slots [0, T) where slot t is token t
  const int32_t* n_active;
  const int32_t* act_expert;
  const int32_t* act_begin;
  const int32_t* perm;
  const int32_t* act_rows;   // [E][8] tokens of the first 8 slots of each active expert
  const float* wts;          // routing weights [T*k] (down, routed)
  int T, k;
  int max_active;            // grid bound on active experts
  // outputs
  int8_t* qh;                // gate/up, g32 act: [slots][I] codes
  __half* sh;                // gate/up, g32 act: [slots][I/32]
  float* hbuf;               // gate/up, token act: [slots][I] fp32 h
  float* dbg_a;              // gate/up: gate values [slots][I]; down: pair values [slots][H]
  float* dbg_b;              // gate/up: up values
  int32_t* dbg_dots;         // down: int32 group dots [slots][H][I/32] (debug)
  float* y;                  // down: [T][H] accumulated
  int* status;
  int early_trigger;         // streaming kernel, batch modes: let the next kernel launch early
                             // (the host-buffer path, where a small output copy follows)
};

// Routed experts and (optional) shared expert: gate/up args gr/gs, down args dr/ds. Work
// unit = (expert, 64 intermediate indices). mode 0: gate/up pass of every unit (h to the
// workspace), 1: down pass (h from the workspace), 2: both, h kept on chip -- needs
// experts_fusable() (group-32 activations: h of a unit is quantized without the rest).
bool experts_fusable(const ExpertArgs& r, const ExpertArgs* s);
// Experts (the shared one: T) with mma_min or more slots are skipped (tensor-core path).
cudaError_t launch_experts(int mode, const ExpertArgs& gr, const ExpertArgs* gs, const ExpertArgs& dr,
                           const ExpertArgs* ds, int mma_min, cudaStream_t st);

// ---- expert_mma.cu: tensor-core GEMMs for experts with many tokens
// Pairs an expert needs in a call to take this path. A tensor-core call costs about the same
// whatever its tiles' fill (~510 us for the 64 OLMoE-shaped int4 experts at one tile each),
// while streaming an expert costs in proportion to its pairs: measured, streaming wins below
// ~12-16 pairs per expert.
constexpr int kMmaMinTokens = 16;

struct MmaArgs {
  BlobView b[2];                           // routed experts, shared expert
  const int4* tiles;
  const int32_t* n_tiles;
  int max_tiles;
  const uint8_t* a_ops;                    // operand A of every tile, fp16: [tile][K/8][128][16]
  const __half* a_scales;                  // [tile][K/32][128]
  // gate/up outputs: h of every tile in operand layout for the down GEMM, and the per-slot
  // views of the workspace (q_h, s_h; gate / up values when debugging)
  uint8_t* h_ops;                          // fp16: [tile][hk/8][128][16]
  __half* h_scales;                        // [tile][hk/32][128]
  int hk;                                  // row length of a tile's h: max(I, I_shared)
  int8_t* qh[2];
  __half* sh[2];
  float* dbg_a[2];
  float* dbg_b[2];
  // down outputs
  const int32_t* perm;
  const float* wts;
  float* y;
  float* dbg_y[2];
  int32_t* dbg_dots[2];                    // down: int32 group dots [slot][H][K/32] (debug)
  int T, k;
  int* status;
};

// Tile list of the experts with >= min_tokens slots (+ the shared expert's tokens).
cudaError_t launch_mma_plan(const Grouping& g, int E, int T, int has_shared, int min_tokens, int max_tiles,
                            int4* tiles, int32_t* n_tiles, int* status, cudaStream_t st);
// Operand A (q_x rows of each tile's tokens, [tile][K/16][128][16]) and its scales.
cudaError_t launch_mma_gather(const int8_t* qx, const __half* sx, const int4* tiles, const int32_t* n_tiles,
                              const int32_t* perm, int k, int T, int K, int max_tiles, uint8_t* xa, __half* xs,
                              int* status, cudaStream_t st);
// Gate/up (+ SwiGLU, Q8_0 h) or down (+ weighted combine) of every tile x weight block.
cudaError_t launch_expert_mma(bool gateup, const MmaArgs& a, cudaStream_t st);

// ---- route_fused.cu (T <= 32)
struct RouteArgs {
  const float* x;
  const float* wr;
  const float* bias;      // sigmoid mode only, may be null
  int T, E, H, k, score, renorm, ag32;     // E: the router's experts (all of them)
  int e0, EL;             // experts held here: global ids e0 .. e0 + EL - 1 (local 0 .. EL - 1);
                          // the grouping keeps only pairs in that range, with local ids
  float rsf;
  float top_p;            // adaptive expert top-p in (0, 1); 0 = off
  int8_t* qx;
  void* sx;
  float* y;               // zeroed here
  float* logits;
  int32_t* idx;
  float* w;
  Grouping g;
  int* status;
  unsigned* ticket;       // zero between calls; the last CTA resets it
  // grid barrier of the single-token expert kernel: a multiple of 1024 between calls (each
  // call's CTAs arrive at base .. base + grid - 1, the last one moves it to base + 1024)
  unsigned long long* gbar;
  unsigned long long wait_ns;   // bound of the single-token kernel's cross-CTA waits (ns)
};
cudaError_t launch_route_fused(const RouteArgs& r, cudaStream_t st);

// One token, group-32 activations: the routing (activation quantization, router logits, top-k,
// grouping) runs inside the expert kernel -- every CTA computes some experts' logits, then
// a grid barrier -- so the whole layer is one launch. decode_fusable() says whether
// the call qualifies (T == 1, E <= 512, fused mode).
bool decode_fusable(const RouteArgs& r, const ExpertArgs& gr, const ExpertArgs* gs);
cudaError_t launch_decode(const RouteArgs& r, const ExpertArgs& gr, const ExpertArgs* gs, const ExpertArgs& dr,
                          const ExpertArgs* ds, cudaStream_t st);

#ifdef MOE_NO_PDL
constexpr bool kUsePdl = false;
#else
constexpr bool kUsePdl = true;
#endif

// Launch with programmatic stream serialization (the kernel calls griddepcontrol.wait
// before touching its predecessor's outputs).
template <typename Kern, typename... Args>
inline cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---- host_io.cu: n floats between page-locked host memory (device-mapped address) and the
// device, as programmatically chained kernels (n a multiple of 4, both addresses 16-aligned).
cudaError_t launch_copy_in(const float* x_host_mapped, float* x_dev, int64_t n, cudaStream_t st);
cudaError_t launch_copy_out(const float* y_dev, float* y_host_mapped, int64_t n, cudaStream_t st);

// ---- expert_gemv.cu (debug entry point)
void launch_group_dots(const BlobView& b, int which, int n, const int32_t* expert,
                       const int32_t* row, const int8_t* act, int32_t* dots, cudaStream_t st);

}  // namespace moe
