// api.cu -- the C ABI (include/moe_b200.h): argument checks, workspace layout and
// the launch sequence of the layer forward.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <cstring>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "kernels.cuh"

namespace {

using moe::BlobView;

inline int64_t al256(int64_t v) { return (v + 255) & ~int64_t(255); }

// Bounds of the single-token kernel's cross-CTA waits (grid barrier, y-zero barrier): about
// a second, or 2 ms with MOE_FLAG_SHORT_WAITS.
constexpr unsigned long long kWaitNs = 1000000000ull;
constexpr unsigned long long kShortWaitNs = 2000000ull;

// Batches up to this many tokens take the single-launch routing kernel.
constexpr int32_t kFusedRouteMaxT = 32;
// Control block at the start of a layer workspace: status word, routing ticket, wait record
// (words 0-3), single-token grid-barrier counter (bytes 16-23).
constexpr int64_t kControlBytes = 256;
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct BlobOffsets {
  int64_t gu_w, dn_w, gu_s, dn_s, total;
};

bool blob_offsets(int32_t wtype, int32_t wscale, int32_t E, int32_t H, int32_t I, BlobOffsets& o) {
  if ((wtype != MOE_W_INT8 && wtype != MOE_W_INT4 && wtype != MOE_W_INT2) ||
      (wscale != MOE_SCALE_ROW_F32 && wscale != MOE_SCALE_G32_F16))
    return false;
  if (E < 1 || E > 1024 || H < 128 || I < 128 || H % 128 || I % 128) return false;
  const int64_t bits = wtype == MOE_W_INT8 ? 8 : wtype == MOE_W_INT4 ? 4 : 2;
  const int64_t kb_gu = H * bits / 8, kb_dn = I * bits / 8;
  const int64_t s_gu = wscale == MOE_SCALE_G32_F16 ? (int64_t)(H / 32) * 2 : 4;
  const int64_t s_dn = wscale == MOE_SCALE_G32_F16 ? (int64_t)(I / 32) * 2 : 4;
  o.gu_w = 0;
  o.dn_w = al256(o.gu_w + (int64_t)E * 2 * I * kb_gu);
  o.gu_s = al256(o.dn_w + (int64_t)E * H * kb_dn);
  o.dn_s = al256(o.gu_s + (int64_t)E * 2 * I * s_gu);
  o.total = al256(o.dn_s + (int64_t)E * H * s_dn);
  return true;
}

moe_status check_blob(const moe_expert_blob* b, BlobOffsets& o) {
  if (!b || !b->data) return MOE_ERR_INVALID_ARG;
  if (!blob_offsets(b->wtype, b->wscale, b->n_experts, b->hidden, b->inter, o))
    return MOE_ERR_UNSUPPORTED;
  if (!aligned(b->data, 256)) return MOE_ERR_INVALID_ARG;
  if ((int64_t)b->bytes < o.total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

BlobView view(const moe_expert_blob* b, const BlobOffsets& o) {
  const uint8_t* d = static_cast<const uint8_t*>(b->data);
  BlobView v;
  v.gu_w = d + o.gu_w;
  v.dn_w = d + o.dn_w;
  v.gu_s = d + o.gu_s;
  v.dn_s = d + o.dn_s;
  v.E = b->n_experts;
  v.H = b->hidden;
  v.I = b->inter;
  v.wbits = b->wtype == MOE_W_INT8 ? 8 : b->wtype == MOE_W_INT4 ? 4 : 2;
  v.wg32 = b->wscale == MOE_SCALE_G32_F16;
  return v;
}

// The router's experts: all of them (n_experts_total, or the blob's when 0).
int32_t experts_total(const moe_route_cfg* c, int32_t E_local) {
  return c->n_experts_total > 0 ? c->n_experts_total : E_local;
}

moe_status check_cfg(const moe_route_cfg* c, int32_t E_local) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID_NOAUX_TC) return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_ACT_TOKEN_F32 && c->act != MOE_ACT_G32_F16) return MOE_ERR_INVALID_ARG;
  if (c->n_experts_total < 0 || c->expert_begin < 0) return MOE_ERR_UNSUPPORTED;
  const int32_t E = experts_total(c, E_local);
  if (E > 1024 || (int64_t)c->expert_begin + E_local > E) return MOE_ERR_UNSUPPORTED;
  if (c->top_k < 1 || c->top_k > 32 || c->top_k > E) return MOE_ERR_UNSUPPORTED;
  if (!(c->top_p >= 0.0f) || !std::isfinite(c->top_p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// The adaptive top-p threshold the kernels take: 0 when off.
float topp_of(const moe_route_cfg* c) { return (c->top_p > 0.0f && c->top_p < 1.0f) ? c->top_p : 0.0f; }

// Workspace of one layer forward: every region starts at a multiple of 256 bytes.
struct Layout {
  int64_t status, qx, sx, logits, idx, w, offsets, perm, n_active, act_expert, act_begin, act_rows;
  int64_t masks, base, qh, sh, hbuf, dbg_gate, dbg_up, dbg_y, dbg_dots, total;
  // tensor-core path (T > 32, group-32 weights and activations)
  int64_t mm_tiles, mm_ntiles, mm_xa, mm_xs, mm_ha, mm_hs;
  int32_t mm_max_tiles, mm_min_tokens, mm_hk;
  int64_t qh_sh, sh_sh, hbuf_sh, dbg_gate_sh, dbg_up_sh, dbg_y_sh, dbg_dots_sh;   // shared-expert rows
};

// E: experts held here (grouping), E_total: the router's experts (logits).
Layout layout(int32_t T, int32_t E, int32_t E_total, int32_t H, int32_t I, int32_t Is, int32_t k, int32_t ag32,
              bool debug, bool mma, bool force_mma) {
  Layout L;
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o = al256(o + (bytes > 0 ? bytes : 0));
    return at;
  };
  const int64_t P = (int64_t)T * k;
  const int64_t C = (T + 31) / 32;
  L.status = take(kControlBytes);
  L.qx = take((int64_t)T * H);
  L.sx = take(ag32 ? (int64_t)T * (H / 32) * 2 : (int64_t)T * 4);
  L.logits = take((int64_t)T * E_total * 4);
  L.idx = take(P * 4);
  L.w = take(P * 4);
  L.offsets = take((int64_t)(E + 1) * 4);
  L.perm = take(P * 4);
  L.n_active = take(4);
  L.act_expert = take((int64_t)(E + 1) * 4);
  L.act_begin = take((int64_t)(E + 2) * 4);
  L.act_rows = take((int64_t)E * 8 * 4);
  L.masks = take(T > 1 ? C * E * 4 : 0);
  L.base = take(T > 1 ? C * E * 4 : 0);
  const int64_t rows_h = P * I + (int64_t)T * Is;
  L.qh = take(rows_h);
  L.qh_sh = L.qh + P * I;
  if (ag32) {
    L.sh = take((P * (I / 32) + (int64_t)T * (Is / 32)) * 2);
    L.sh_sh = L.sh + P * (I / 32) * 2;
  } else {
    L.sh = take((P + T) * 4);
    L.sh_sh = L.sh + P * 4;
  }
  if (!ag32) {
    L.hbuf = take(rows_h * 4);
    L.hbuf_sh = L.hbuf + P * I * 4;
  } else {
    L.hbuf = L.hbuf_sh = -1;
  }
  if (debug) {
    L.dbg_gate = take(rows_h * 4);
    L.dbg_gate_sh = L.dbg_gate + P * I * 4;
    L.dbg_up = take(rows_h * 4);
    L.dbg_up_sh = L.dbg_up + P * I * 4;
    L.dbg_y = take((P + T) * H * 4);
    L.dbg_y_sh = L.dbg_y + P * H * 4;
    L.dbg_dots = take((P * (I / 32) + (int64_t)T * (Is / 32)) * H * 4);
    L.dbg_dots_sh = L.dbg_dots + P * H * (I / 32) * 4;
  } else {
    L.dbg_gate = L.dbg_up = L.dbg_y = L.dbg_dots = -1;
    L.dbg_gate_sh = L.dbg_up_sh = L.dbg_y_sh = L.dbg_dots_sh = -1;
  }
  L.mm_max_tiles = 0;
  L.mm_min_tokens = force_mma ? 1 : moe::kMmaMinTokens;
  L.mm_hk = std::max(I, Is);
  L.mm_tiles = L.mm_ntiles = L.mm_xa = L.mm_xs = L.mm_ha = L.mm_hs = -1;
  if (mma) {
    // tiles of 128 slots: every qualifying expert wastes at most one partial tile
    const int64_t n_exp = std::min<int64_t>(E, P / L.mm_min_tokens);
    const int64_t mt = (P + 127) / 128 + n_exp + (Is ? (T + 127) / 128 : 0) + 1;
    L.mm_max_tiles = (int32_t)mt;
    L.mm_tiles = take(mt * 16);
    L.mm_ntiles = take(4);
    L.mm_xa = take(mt * 128 * H * 2);                     // fp16 operands
    L.mm_xs = take(mt * (H / 32) * 128 * 2);
    L.mm_ha = take(mt * 128 * L.mm_hk * 2);
    L.mm_hs = take(mt * (L.mm_hk / 32) * 128 * 2);
  }
  L.total = o;
  return L;
}

// Calls with more than kFusedRouteMaxT tokens, group-32 weights and activations send experts
// with many pairs to the tensor-core GEMMs.
bool use_mma(int32_t T, const moe_expert_blob* experts, const moe_route_cfg* cfg) {
  return T > kFusedRouteMaxT && cfg->act == MOE_ACT_G32_F16 && experts->wscale == MOE_SCALE_G32_F16 &&
         (cfg->flags & MOE_FLAG_FORCE_GEMV) == 0;
}

// One token with group-32 activations: routing and every expert in one launch (the expert
// kernel routes the token itself before a grid barrier).
bool use_decode(int32_t T, const moe_expert_blob* experts, const moe_route_cfg* cfg) {
  const int32_t E = experts_total(cfg, experts->n_experts);
  return T == 1 && cfg->act == MOE_ACT_G32_F16 && E <= 512 && experts->hidden % 128 == 0 &&
         4 * E <= experts->hidden;
}

struct LayerPlan {
  BlobOffsets eo, so;
  int32_t Is;
  bool mma;      // experts with many tokens take the tensor-core path
  Layout L;
};

moe_status plan_layer(int32_t T, const moe_expert_blob* experts, const moe_expert_blob* shared,
                      const moe_route_cfg* cfg, LayerPlan& p) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  moe_status s = check_blob(experts, p.eo);
  if (s != MOE_OK) return s;
  s = check_cfg(cfg, experts->n_experts);
  if (s != MOE_OK) return s;
  p.Is = 0;
  if (shared) {
    s = check_blob(shared, p.so);
    if (s != MOE_OK) return s;
    if (shared->n_experts != 1 || shared->hidden != experts->hidden ||
        shared->wtype != experts->wtype || shared->wscale != experts->wscale)
      return MOE_ERR_UNSUPPORTED;
    p.Is = shared->inter;
  }
  p.mma = use_mma(T, experts, cfg);
  p.L = layout(T, experts->n_experts, experts_total(cfg, experts->n_experts), experts->hidden,
               experts->inter, p.Is, cfg->top_k,
               cfg->act == MOE_ACT_G32_F16, (cfg->flags & MOE_FLAG_DEBUG) != 0, p.mma,
               (cfg->flags & MOE_FLAG_FORCE_MMA) != 0);
  return MOE_OK;
}

thread_local char g_last_error[256] = "";

moe_status cuda_fail(const char* where, cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
  return MOE_ERR_CUDA;
}

moe_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail("launch", e);
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_last_error(void) { return g_last_error; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

size_t moe_expert_blob_bytes(int32_t wtype, int32_t wscale, int32_t n_experts, int32_t hidden,
                             int32_t inter) {
  BlobOffsets o;
  if (!blob_offsets(wtype, wscale, n_experts, hidden, inter, o)) return 0;
  return (size_t)o.total;
}

moe_status moe_quantize_experts(const float* w_gate_up, const float* w_down,
                                const moe_expert_blob* out, void* stream) {
  if (!w_gate_up || !w_down) return MOE_ERR_INVALID_ARG;
  BlobOffsets o;
  const moe_status s = check_blob(out, o);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t me = cudaMemsetAsync(out->data, 0, (size_t)o.total, st);
  if (me != cudaSuccess) return cuda_fail("blob memset", me);
  const BlobView b = view(out, o);
  uint8_t* d = static_cast<uint8_t*>(out->data);
  moe::launch_quantize_experts(w_gate_up, w_down, b, d + o.gu_w, d + o.dn_w, d + o.gu_s,
                               d + o.dn_s, st);
  return launch_status();
}

moe_status moe_quantize_experts_fp8(const uint8_t* w_gate_up, const float* s_gate_up,
                                    const uint8_t* w_down, const float* s_down,
                                    const moe_expert_blob* out, void* stream) {
  if (!w_gate_up || !s_gate_up || !w_down || !s_down) return MOE_ERR_INVALID_ARG;
  BlobOffsets o;
  const moe_status s = check_blob(out, o);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t me = cudaMemsetAsync(out->data, 0, (size_t)o.total, st);
  if (me != cudaSuccess) return cuda_fail("blob memset", me);
  const BlobView b = view(out, o);
  uint8_t* d = static_cast<uint8_t*>(out->data);
  moe::launch_quantize_experts_fp8(w_gate_up, s_gate_up, w_down, s_down, b, d + o.gu_w, d + o.dn_w,
                                   d + o.gu_s, d + o.dn_s, st);
  return launch_status();
}

moe_status moe_quantize_activations(const float* x, int32_t T, int32_t H, int32_t act, int8_t* q,
                                    void* scales, void* stream) {
  if (T < 0 || H <= 0 || H % 32) return T < 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  if (act != MOE_ACT_TOKEN_F32 && act != MOE_ACT_G32_F16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !q || !scales || !aligned(x, 16) || !aligned(q, 4) || !aligned(scales, 4))
    return MOE_ERR_INVALID_ARG;
  moe::launch_quantize_act(x, T, H, act == MOE_ACT_G32_F16, q, scales, nullptr, nullptr,
                           static_cast<cudaStream_t>(stream));
  return launch_status();
}

moe_status moe_router_logits(const float* x, const float* router_w, int32_t T, int32_t E,
                             int32_t H, float* logits, void* stream) {
  if (T < 0 || E < 1) return MOE_ERR_INVALID_ARG;
  if (H <= 0 || H % 32) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !logits || !aligned(x, 16) || !aligned(router_w, 16))
    return MOE_ERR_INVALID_ARG;
  moe::launch_router_logits(x, router_w, T, E, H, logits, static_cast<cudaStream_t>(stream));
  return launch_status();
}

moe_status moe_route_topk(const float* logits, const float* bias, int32_t T, int32_t E,
                          const moe_route_cfg* cfg, int32_t* idx, float* w, void* stream) {
  if (T < 0 || E < 1 || E > 1024) return E > 1024 ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (!cfg) return MOE_ERR_INVALID_ARG;
  moe_route_cfg c = *cfg;                 // selection over the E logits given: no expert range
  c.n_experts_total = 0;
  c.expert_begin = 0;
  const moe_status s = check_cfg(&c, E);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !w) return MOE_ERR_INVALID_ARG;
  moe::launch_topk(logits, cfg->score == MOE_SCORE_SIGMOID_NOAUX_TC ? bias : nullptr, T, E,
                   cfg->top_k, cfg->score, cfg->renormalize != 0, cfg->routed_scaling_factor,
                   topp_of(cfg), idx, w, nullptr, nullptr, static_cast<cudaStream_t>(stream));
  return launch_status();
}

size_t moe_permute_workspace_bytes(int32_t T, int32_t k, int32_t E) {
  if (T < 0 || k < 1 || E < 1 || E > 1024) return 0;
  const int64_t C = (T + 31) / 32;
  return (size_t)(256 + al256(C * E * 4) * 2 + 256 + al256((int64_t)(E + 1) * 4) +
                  al256((int64_t)(E + 2) * 4));
}

moe_status moe_permute(const int32_t* idx, int32_t T, int32_t k, int32_t E, int32_t* offsets,
                       int32_t* perm, void* workspace, size_t ws_bytes, void* stream) {
  if (T < 0 || k < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!idx || !offsets || !perm || !workspace) return MOE_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_bytes(T, k, E)) return MOE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t C = (T + 31) / 32;
  int64_t o = 256;
  uint32_t* masks = reinterpret_cast<uint32_t*>(ws + o);
  o += al256(C * E * 4);
  int32_t* base = reinterpret_cast<int32_t*>(ws + o);
  o += al256(C * E * 4);
  moe::Grouping g{};
  g.offsets = offsets;
  g.perm = perm;
  g.n_active = reinterpret_cast<int32_t*>(ws + o);
  o += 256;
  g.act_expert = reinterpret_cast<int32_t*>(ws + o);
  o += al256((int64_t)(E + 1) * 4);
  g.act_begin = reinterpret_cast<int32_t*>(ws + o);
  moe::launch_permute(idx, T, k, E, 0, E, g, masks, base, reinterpret_cast<int*>(ws), 1,
                      static_cast<cudaStream_t>(stream));
  return launch_status();
}

size_t moe_layer_workspace_bytes(int32_t T, const moe_expert_blob* experts,
                                 const moe_expert_blob* shared, const moe_route_cfg* cfg) {
  LayerPlan p;
  if (!experts || !cfg) return 0;
  // sizes only: a blob without data is fine here
  moe_expert_blob e = *experts;
  if (!e.data) e.data = reinterpret_cast<void*>(256);
  moe_expert_blob sh;
  if (shared) {
    sh = *shared;
    if (!sh.data) sh.data = reinterpret_cast<void*>(256);
  }
  e.bytes = e.bytes ? e.bytes : (size_t)-1;
  if (shared) sh.bytes = sh.bytes ? sh.bytes : (size_t)-1;
  if (plan_layer(T, &e, shared ? &sh : nullptr, cfg, p) != MOE_OK) return 0;
  return (size_t)p.L.total;
}

moe_status moe_layer_debug_views(int32_t T, const moe_expert_blob* experts,
                                 const moe_expert_blob* shared, const moe_route_cfg* cfg,
                                 moe_debug_views* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  const size_t total = moe_layer_workspace_bytes(T, experts, shared, cfg);
  if (total == 0) return MOE_ERR_UNSUPPORTED;
  const int32_t Is = shared ? shared->inter : 0;
  const Layout L = layout(T, experts->n_experts, experts_total(cfg, experts->n_experts), experts->hidden,
                          experts->inter, Is, cfg->top_k,
                          cfg->act == MOE_ACT_G32_F16, (cfg->flags & MOE_FLAG_DEBUG) != 0,
                          use_mma(T, experts, cfg), (cfg->flags & MOE_FLAG_FORCE_MMA) != 0);
  out->status = L.status;
  out->q_x = L.qx;
  out->s_x = L.sx;
  out->logits = L.logits;
  out->idx = L.idx;
  out->w = L.w;
  out->offsets = L.offsets;
  out->perm = L.perm;
  out->n_active = L.n_active;
  out->act_expert = L.act_expert;
  out->q_h = L.qh;
  out->s_h = L.sh;
  out->gate = L.dbg_gate;
  out->up = L.dbg_up;
  out->y_pair = L.dbg_y;
  out->dn_dots = L.dbg_dots;
  out->total = L.total;
  return MOE_OK;
}

}  // extern "C"

namespace {

struct StageMarks {
  const moe_stage_events* ev;
  cudaStream_t st;
  bool capturing;
  cudaError_t err = cudaSuccess;
  void mark(void* e) {
    if (!e) return;
    cudaError_t r = capturing ? cudaEventRecordWithFlags(static_cast<cudaEvent_t>(e), st, cudaEventRecordExternal)
                              : cudaEventRecord(static_cast<cudaEvent_t>(e), st);
    if (r != cudaSuccess) err = r;
  }
  void begin(int s) { if (ev) mark(ev->begin[s]); }
  void end(int s) { if (ev) mark(ev->end[s]); }
};

// host_copy: the host-buffer entry, whose output copy kernel follows the layer's last kernel.
moe_status forward_impl(const float* x, int32_t T, const float* router_w, const float* router_bias,
                        const moe_expert_blob* experts, const moe_expert_blob* shared,
                        const moe_route_cfg* cfg, float* y, void* workspace, size_t ws_bytes,
                        void* stream, const moe_stage_events* events, bool host_copy = false) {
  LayerPlan p;
  moe_status s = plan_layer(T, experts, shared, cfg, p);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(y, 16)) return MOE_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < (size_t)p.L.total) return MOE_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  StageMarks mk{events, st, false};
  if (events) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t ce = cudaStreamIsCapturing(st, &cs);
    if (ce != cudaSuccess) return cuda_fail("cudaStreamIsCapturing", ce);
    mk.capturing = cs == cudaStreamCaptureStatusActive;
  }
  const Layout& L = p.L;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto at = [&](int64_t off) -> void* { return off < 0 ? nullptr : ws + off; };
  // E: experts held here (grouping, blob), E_total: the router's (logits, top-k)
  const int32_t E = experts->n_experts, H = experts->hidden, I = experts->inter, k = cfg->top_k;
  const int32_t E_total = experts_total(cfg, E), e0 = cfg->expert_begin;
  const int ag32 = cfg->act == MOE_ACT_G32_F16;
  int* status = static_cast<int*>(at(L.status));
  const BlobView bv = view(experts, p.eo);

  moe::Grouping g{};
  g.offsets = static_cast<int32_t*>(at(L.offsets));
  g.perm = static_cast<int32_t*>(at(L.perm));
  g.n_active = static_cast<int32_t*>(at(L.n_active));
  g.act_expert = static_cast<int32_t*>(at(L.act_expert));
  g.act_begin = static_cast<int32_t*>(at(L.act_begin));
  g.act_rows = static_cast<int32_t*>(at(L.act_rows));
  int32_t* idx = static_cast<int32_t*>(at(L.idx));
  float* wts = static_cast<float*>(at(L.w));
  float* logits = static_cast<float*>(at(L.logits));
  const float* bias = cfg->score == MOE_SCORE_SIGMOID_NOAUX_TC ? router_bias : nullptr;
  cudaError_t err = cudaSuccess;
  const char* err_where = "";
  auto keep = [&](cudaError_t e, const char* where) {
    if (e != cudaSuccess && err == cudaSuccess) {
      err = e;
      err_where = where;
    }
  };

  moe::RouteArgs r;
  std::memset(&r, 0, sizeof(r));
  const bool decode = use_decode(T, experts, cfg);
  if (T <= kFusedRouteMaxT) {
    // 1-3. activation quantization, router logits, top-k and grouping in one launch (one
    //      token: inside the expert kernel, launched below)
    r.x = x;
    r.wr = router_w;
    r.bias = bias;
    r.T = T;
    r.E = E_total;
    r.e0 = e0;
    r.EL = E;
    r.H = H;
    r.k = k;
    r.score = cfg->score;
    r.renorm = cfg->renormalize != 0;
    r.ag32 = ag32;
    r.rsf = cfg->routed_scaling_factor;
    r.top_p = topp_of(cfg);
    r.qx = static_cast<int8_t*>(at(L.qx));
    r.sx = at(L.sx);
    r.y = y;
    r.logits = logits;
    r.idx = idx;
    r.w = wts;
    r.g = g;
    r.status = status;
    r.ticket = reinterpret_cast<unsigned*>(ws + L.status + 4);
    r.gbar = reinterpret_cast<unsigned long long*>(ws + L.status + 16);
    r.wait_ns = (cfg->flags & MOE_FLAG_SHORT_WAITS) ? kShortWaitNs : kWaitNs;
    mk.begin(MOE_STAGE_QUANT_X);
    if (!decode) keep(moe::launch_route_fused(r, st), "routing kernel");
    mk.end(MOE_STAGE_QUANT_X);
    for (int sg = MOE_STAGE_ROUTER; sg <= MOE_STAGE_GROUP; ++sg) {
      mk.begin(sg);
      mk.end(sg);
    }
  } else {
    // 1. Q8_0 activations (also zeroes y and the status word)
    mk.begin(MOE_STAGE_QUANT_X);
    moe::launch_quantize_act(x, T, H, ag32, static_cast<int8_t*>(at(L.qx)), at(L.sx), y, status, st);
    mk.end(MOE_STAGE_QUANT_X);
    // 2. router logits
    mk.begin(MOE_STAGE_ROUTER);
    moe::launch_router_logits(x, router_w, T, E_total, H, logits, st);
    mk.end(MOE_STAGE_ROUTER);
    // 3. top-k selection and weights, batch-union grouping
    mk.begin(MOE_STAGE_TOPK);
    moe::launch_topk(logits, bias, T, E_total, k, cfg->score, cfg->renormalize != 0,
                     cfg->routed_scaling_factor, topp_of(cfg), idx, wts, nullptr, status, st);
    mk.end(MOE_STAGE_TOPK);
    mk.begin(MOE_STAGE_GROUP);
    moe::launch_permute(idx, T, k, E, e0, E_total, g, static_cast<uint32_t*>(at(L.masks)),
                        static_cast<int32_t*>(at(L.base)), status, 0, st);
    mk.end(MOE_STAGE_GROUP);
  }

  // 4. gate/up + SwiGLU (+ h quantization for group-32 activations); routed and shared
  //    experts in one grid
  moe::ExpertArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  ra.early_trigger = host_copy ? 1 : 0;
  ra.b = bv;
  ra.qa = static_cast<const int8_t*>(at(L.qx));
  ra.sa = at(L.sx);
  ra.ag32 = ag32;
  ra.n_active = g.n_active;
  ra.act_expert = g.act_expert;
  ra.act_begin = g.act_begin;
  ra.perm = g.perm;
  ra.act_rows = g.act_rows;
  ra.wts = wts;
  ra.T = T;
  ra.k = k;
  ra.max_active = (int)((int64_t)T * k < E ? (int64_t)T * k : E);
  ra.qh = static_cast<int8_t*>(at(L.qh));
  ra.sh = static_cast<__half*>(at(L.sh));
  ra.hbuf = static_cast<float*>(at(L.hbuf));
  ra.dbg_a = static_cast<float*>(at(L.dbg_gate));
  ra.dbg_b = static_cast<float*>(at(L.dbg_up));
  ra.y = y;
  ra.status = status;
  moe::ExpertArgs sa;
  std::memset(&sa, 0, sizeof(sa));
  if (shared) {
    sa = ra;
    sa.b = view(shared, p.so);
    sa.n_active = nullptr;
    sa.act_expert = nullptr;
    sa.act_begin = nullptr;
    sa.perm = nullptr;
    sa.act_rows = nullptr;
    sa.max_active = 1;
    sa.qh = static_cast<int8_t*>(at(L.qh_sh));
    sa.sh = static_cast<__half*>(at(L.sh_sh));
    sa.hbuf = static_cast<float*>(at(L.hbuf_sh));
    sa.dbg_a = static_cast<float*>(at(L.dbg_gate_sh));
    sa.dbg_b = static_cast<float*>(at(L.dbg_up_sh));
  }
  // 5. down projection + weighted combine into y; routed and shared experts in one grid
  moe::ExpertArgs rd = ra;
  rd.qa = static_cast<const int8_t*>(at(L.qh));
  rd.sa = at(L.sh);
  rd.dbg_a = static_cast<float*>(at(L.dbg_y));
  rd.dbg_b = nullptr;
  rd.dbg_dots = static_cast<int32_t*>(at(L.dbg_dots));
  moe::ExpertArgs sd = sa;
  if (shared) {
    sd.qa = static_cast<const int8_t*>(at(L.qh_sh));
    sd.sa = at(L.sh_sh);
    sd.dbg_a = static_cast<float*>(at(L.dbg_y_sh));
    sd.dbg_b = nullptr;
    sd.dbg_dots = static_cast<int32_t*>(at(L.dbg_dots_sh));
  }
  const moe::ExpertArgs* sap = shared ? &sa : nullptr;
  const moe::ExpertArgs* sdp = shared ? &sd : nullptr;
  // the down kernels add each unit's share of a pair's down value into the pair's view
  if (L.dbg_y >= 0)
    keep(cudaMemsetAsync(ws + L.dbg_y, 0, (size_t)((int64_t)(T * k + T) * H * 4), st), "debug view reset");
  if (L.dbg_dots >= 0)
    keep(cudaMemsetAsync(ws + L.dbg_dots, 0, (size_t)(((int64_t)T * k * (I / 32) + (int64_t)T * (p.Is / 32)) * H * 4), st),
         "debug dots reset");
  // experts with many slots: tensor-core GEMMs (tile list, operand gather, gate/up, down)
  const int mma_min = p.mma ? L.mm_min_tokens : 0x7fffffff;
  auto launch_mma = [&](bool down) {
    moe::MmaArgs m;
    std::memset(&m, 0, sizeof(m));
    m.b[0] = bv;
    m.b[1] = shared ? sa.b : bv;
    m.tiles = static_cast<const int4*>(at(L.mm_tiles));
    m.n_tiles = static_cast<const int32_t*>(at(L.mm_ntiles));
    m.max_tiles = L.mm_max_tiles;
    m.a_ops = static_cast<const uint8_t*>(at(L.mm_xa));
    m.a_scales = static_cast<const __half*>(at(L.mm_xs));
    m.h_ops = static_cast<uint8_t*>(at(L.mm_ha));
    m.h_scales = static_cast<__half*>(at(L.mm_hs));
    m.hk = L.mm_hk;
    m.qh[0] = ra.qh;
    m.qh[1] = shared ? sa.qh : ra.qh;
    m.sh[0] = ra.sh;
    m.sh[1] = shared ? sa.sh : ra.sh;
    m.dbg_a[0] = ra.dbg_a;
    m.dbg_a[1] = shared ? sa.dbg_a : nullptr;
    m.dbg_b[0] = ra.dbg_b;
    m.dbg_b[1] = shared ? sa.dbg_b : nullptr;
    m.perm = g.perm;
    m.wts = wts;
    m.y = y;
    m.dbg_y[0] = rd.dbg_a;
    m.dbg_y[1] = shared ? sd.dbg_a : nullptr;
    m.dbg_dots[0] = rd.dbg_dots;
    m.dbg_dots[1] = shared ? sd.dbg_dots : nullptr;
    m.T = T;
    m.k = k;
    m.status = status;
    if (!down) {
      keep(moe::launch_mma_plan(g, E, T, shared ? 1 : 0, L.mm_min_tokens, L.mm_max_tiles,
                                static_cast<int4*>(at(L.mm_tiles)), static_cast<int32_t*>(at(L.mm_ntiles)),
                                status, st),
           "tensor-core tile plan");
      keep(moe::launch_mma_gather(static_cast<const int8_t*>(at(L.qx)), static_cast<const __half*>(at(L.sx)),
                                  m.tiles, m.n_tiles, g.perm, k, T, H, L.mm_max_tiles,
                                  static_cast<uint8_t*>(at(L.mm_xa)), static_cast<__half*>(at(L.mm_xs)),
                                  status, st),
           "tensor-core operand gather");
      keep(moe::launch_expert_mma(true, m, st), "tensor-core gate/up kernel");
    } else {
      keep(moe::launch_expert_mma(false, m, st), "tensor-core down kernel");
    }
  };
  if (decode) {
    // one token: routing (1-3) and 4+5 in one persistent grid
    mk.begin(MOE_STAGE_GATE_UP);
    keep(moe::launch_decode(r, ra, sap, rd, sdp, st), "decode kernel");
    mk.end(MOE_STAGE_GATE_UP);
    for (int sg : {MOE_STAGE_DOWN, MOE_STAGE_QUANT_H}) {
      mk.begin(sg);
      mk.end(sg);
    }
  } else if (moe::experts_fusable(ra, sap)) {
    // 4+5 in one persistent grid: per unit (expert, 64 intermediate indices) the gate/up
    // pass, SwiGLU and h quantization, then the unit's share of the down projection
    mk.begin(MOE_STAGE_GATE_UP);
    if (p.mma) launch_mma(false);
    keep(moe::launch_experts(2, ra, sap, rd, sdp, mma_min, st), "expert kernel");
    mk.end(MOE_STAGE_GATE_UP);
    mk.begin(MOE_STAGE_DOWN);
    if (p.mma) launch_mma(true);
    mk.end(MOE_STAGE_DOWN);
    mk.begin(MOE_STAGE_QUANT_H);
    mk.end(MOE_STAGE_QUANT_H);
  } else {
    mk.begin(MOE_STAGE_GATE_UP);
    if (p.mma) launch_mma(false);
    keep(moe::launch_experts(0, ra, sap, rd, sdp, mma_min, st), "gate/up kernel");
    mk.end(MOE_STAGE_GATE_UP);
    mk.begin(MOE_STAGE_QUANT_H);
    if (!ag32) {
      moe::launch_quantize_rows_token(static_cast<const float*>(at(L.hbuf)), T * k, I,
                                      static_cast<int8_t*>(at(L.qh)), static_cast<float*>(at(L.sh)), st);
      if (shared)
        moe::launch_quantize_rows_token(static_cast<const float*>(at(L.hbuf_sh)), T, p.Is,
                                        static_cast<int8_t*>(at(L.qh_sh)),
                                        static_cast<float*>(at(L.sh_sh)), st);
    }
    mk.end(MOE_STAGE_QUANT_H);
    mk.begin(MOE_STAGE_DOWN);
    keep(moe::launch_experts(1, ra, sap, rd, sdp, mma_min, st), "down kernel");
    if (p.mma) launch_mma(true);
    mk.end(MOE_STAGE_DOWN);
  }
  if (err != cudaSuccess) return cuda_fail(err_where, err);
  if (mk.err != cudaSuccess) return cuda_fail("stage event record", mk.err);
  return launch_status();
}

}  // namespace

extern "C" {

moe_status moe_layer_forward(const float* x, int32_t T, const float* router_w,
                             const float* router_bias, const moe_expert_blob* experts,
                             const moe_expert_blob* shared, const moe_route_cfg* cfg, float* y,
                             void* workspace, size_t ws_bytes, void* stream) {
  return forward_impl(x, T, router_w, router_bias, experts, shared, cfg, y, workspace, ws_bytes,
                      stream, nullptr);
}

moe_status moe_layer_forward_host(const float* x_host, int32_t T, const float* router_w,
                                  const float* router_bias, const moe_expert_blob* experts,
                                  const moe_expert_blob* shared, const moe_route_cfg* cfg, float* x_dev,
                                  float* y_dev, float* y_host, void* workspace, size_t ws_bytes, void* stream) {
  if (T < 0 || !experts) return MOE_ERR_INVALID_ARG;
  if (T == 0) return forward_impl(x_dev, T, router_w, router_bias, experts, shared, cfg, y_dev, workspace,
                                  ws_bytes, stream, nullptr);
  if (!x_host || !y_host || !x_dev || !y_dev) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = (int64_t)T * experts->hidden;
  const size_t bytes = (size_t)n * sizeof(float);
  // page-locked host buffers with device-mapped addresses: the SMs move x and y (kernels
  // chained to the layer's); otherwise copy-engine copies
  void* xm = nullptr;
  void* ym = nullptr;
  const bool mapped = aligned(x_host, 16) && aligned(y_host, 16) && aligned(x_dev, 16) && aligned(y_dev, 16) &&
                      cudaHostGetDevicePointer(&xm, const_cast<float*>(x_host), 0) == cudaSuccess &&
                      cudaHostGetDevicePointer(&ym, y_host, 0) == cudaSuccess;
  if (!mapped) (void)cudaGetLastError();   // the lookup's error is not the call's
  cudaError_t e = mapped ? moe::launch_copy_in(static_cast<const float*>(xm), x_dev, n, st)
                         : cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail("x host-to-device copy", e);
  const moe_status s = forward_impl(x_dev, T, router_w, router_bias, experts, shared, cfg, y_dev, workspace,
                                    ws_bytes, stream, nullptr, true);
  if (s != MOE_OK) return s;
  e = mapped ? moe::launch_copy_out(y_dev, static_cast<float*>(ym), n, st)
             : cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail("y device-to-host copy", e);
  return MOE_OK;
}

moe_status moe_layer_forward_timed(const float* x, int32_t T, const float* router_w,
                                   const float* router_bias, const moe_expert_blob* experts,
                                   const moe_expert_blob* shared, const moe_route_cfg* cfg,
                                   float* y, void* workspace, size_t ws_bytes, void* stream,
                                   const moe_stage_events* events) {
  return forward_impl(x, T, router_w, router_bias, experts, shared, cfg, y, workspace, ws_bytes,
                      stream, events);
}

int32_t moe_layer_kernel_count(int32_t T, const moe_expert_blob* experts,
                               const moe_expert_blob* shared, const moe_route_cfg* cfg) {
  if (moe_layer_workspace_bytes(T, experts, shared, cfg) == 0) return -1;
  if (T == 0) return 0;
  if (use_decode(T, experts, cfg)) return 1;   // routing and experts in one grid
  int n = T <= kFusedRouteMaxT ? 1 : 4;        // routing (fused, or quantize/logits/top-k/grouping)
  if (use_mma(T, experts, cfg)) n += 4;                                     // tensor-core tile plan, gather, gate/up, down
  if (cfg->act == MOE_ACT_G32_F16) return n + 1;   // gate/up and down of all experts in one grid
  n += 1;                                       // gate/up, routed and shared experts in one grid
  if (cfg->act != MOE_ACT_G32_F16) n += 1 + (shared ? 1 : 0);   // h quantization
  n += 1;                                       // down, routed and shared experts in one grid
  return n;
}

moe_status moe_expert_group_dots(const moe_expert_blob* blob, int32_t which, int32_t n,
                                 const int32_t* expert, const int32_t* row, const int8_t* act,
                                 int32_t* dots, void* stream) {
  BlobOffsets o;
  const moe_status s = check_blob(blob, o);
  if (s != MOE_OK) return s;
  if ((which != 0 && which != 1) || n < 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!expert || !row || !act || !dots || !aligned(act, 16)) return MOE_ERR_INVALID_ARG;
  moe::launch_group_dots(view(blob, o), which, n, expert, row, act, dots,
                         static_cast<cudaStream_t>(stream));
  return launch_status();
}

moe_status moe_read_device_status(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < 4) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, 4, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail("status copy", e);
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail("status synchronize", e);
  e = cudaMemsetAsync(workspace, 0, 4, st);
  if (e != cudaSuccess) return cuda_fail("status clear", e);
  if (h == MOE_ERR_TIMEOUT && ws_bytes >= (size_t)kControlBytes) {
    // a wait gave up: the routing ticket (word 1) and the grid-barrier counter (bytes 16-23)
    // may be left mid-call; the wait record (words 2-3) stays readable
    e = cudaMemsetAsync(static_cast<uint8_t*>(workspace) + 4, 0, 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(static_cast<uint8_t*>(workspace) + 16, 0, kControlBytes - 16, st);
    if (e != cudaSuccess) return cuda_fail("control block reset", e);
  }
  return static_cast<moe_status>(h);
}

moe_status moe_get_device_status(void* workspace, void* stream) {
  return moe_read_device_status(workspace, (size_t)kControlBytes, stream);
}

moe_status moe_layer_forward_debug(const float* x, int32_t T, const float* router_w,
                                   const float* router_bias, const moe_expert_blob* experts,
                                   const moe_expert_blob* shared, const moe_route_cfg* cfg, float* y,
                                   void* workspace, size_t ws_bytes, void* stream, moe_debug_views* views) {
  if (!cfg || !views) return MOE_ERR_INVALID_ARG;
  moe_route_cfg c = *cfg;
  c.flags |= MOE_FLAG_DEBUG;
  const moe_status s = moe_layer_forward(x, T, router_w, router_bias, experts, shared, &c, y, workspace,
                                         ws_bytes, stream);
  if (s != MOE_OK || T == 0) return s;
  return moe_layer_debug_views(T, experts, shared, &c, views);
}

}  // extern "C"
