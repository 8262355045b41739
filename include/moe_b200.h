/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) quantized Mixture-of-Experts FFN layer.
 *
 * The layer (GLM-5.2 colibri page "Show HN: getting GLM-5.2 running on my slow
 * compute", section "What's implemented"; OLMoE page "I ran a 7B
 * Mixture-of-Experts LLM in a language I built", section "Mixture-of-Experts"):
 *
 *   logits  = x . W_r^T                                (fp32 router)
 *   idx, w  = top-k of softmax(logits)                 (optionally renormalised)
 *             or DeepSeek-V3-style sigmoid noaux_tc:   s = sigmoid(logits),
 *             select on s + bias, w = s / sum_sel(s) * routed_scaling_factor
 *   q_x     = Q8_0-style int8 activations              (group-32 fp16 scales, or
 *                                                      one fp32 scale per token)
 *   g, u    = dequant-on-use int8 / packed-int4 expert matmuls (integer dots)
 *   h       = silu(g) * u, re-quantized like q_x      (SwiGLU)
 *   y_e     = down projection of h
 *   y       = sum_j w_j * y_{e_j} + FFN_shared(x)      (shared expert optional)
 *
 * with batch-union grouping ("Batch-union MoE" on the GLM page): the (token,
 * slot) pairs are grouped by expert so every selected expert's weights are
 * streamed from HBM once per call, whatever the number of tokens routed to it.
 *
 * Conventions for every entry point:
 *   - Pointers named x, y, logits, idx, w, q, scales, workspace, blob data are
 *     DEVICE pointers owned by the caller; struct arguments themselves
 *     (moe_expert_blob, moe_route_cfg) live in host memory and are read during
 *     the call only.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream). Argument and shape checks happen on the host
 *     before anything is enqueued and return synchronously; nothing is
 *     enqueued when a call returns an error.
 *   - The library never allocates device memory and never synchronizes,
 *     except moe_read_device_status, which synchronizes `stream`.
 *   - Inputs must be finite. Results for NaN or Inf inputs are unspecified.
 *   - Supported shapes: hidden H and expert intermediate I multiples of 128;
 *     1 <= top_k <= min(E, 32); E <= 1024; T >= 0 (T = 0 is a no-op).
 *
 * Numerics. Every step that decides an integer (quantized codes, top-k
 * selection) runs a fixed fp32 operation sequence, so results are bit-exact
 * across runs and against a CPU implementation of the same sequence:
 *   - quantization: d = amax / Q (fp32 division, Q = 127 int8, 7 int4 or 1 int2),
 *     stored as fp32 (per row / per token) or rounded to fp16 (group of 32);
 *     q = clamp(round_half_away(v / stored_d), -Q, Q); q = 0 if stored_d = 0;
 *   - router logits: per 32-element chunk an fma chain from +0 in ascending
 *     index, chunk partials added in ascending chunk order;
 *   - exp: Cody-Waite reduction by ln 2 with a degree-7 Taylor polynomial,
 *     argument clamped to [-87, 88]; sigmoid s = 1 / (1 + exp(-L));
 *   - expert row value: exact int32 dot per group of 32, then
 *     acc = fma((float)I_g, c_g, acc) over ascending groups from +0, where c_g
 *     is the product of the two group scales (both group-32) or the scale that
 *     varies by group, and the per-row / per-token scale multiplies the end;
 *     per-row weights with per-token activations form one group (the row);
 *   - SwiGLU h = (g / (1 + exp(-g))) * u.
 * The down projection and the weighted combine are fp32 in an unspecified
 * order (fp32 atomic adds into y); their rounding differs from run to run by
 * a few ulp.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 4

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum value */
  MOE_ERR_UNSUPPORTED = 2,   /* shape or format combination outside the supported set */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  MOE_ERR_CUDA = 4,          /* a CUDA launch or copy failed (cudaGetLastError) */
  MOE_ERR_DEVICE_CHECK = 5,  /* a kernel found an out-of-range index at run time */
  MOE_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up */
} moe_status;

/* Expert weight code type (the GLM-5.2 colibri page, "What's implemented": int8 / packed int4 /
 * packed int2). Packed int4: two's-complement nibbles, two per byte (element 2j in the low
 * nibble of byte j), codes -7..7. Packed int2: two's-complement 2-bit fields, four per byte
 * (element 4j + i in bits 2i..2i+1 of byte j), codes -1, 0, 1 (the symmetric rule with
 * Q = 1: d = amax, -2 never produced). */
enum { MOE_W_INT8 = 0, MOE_W_INT4 = 1, MOE_W_INT2 = 2 };
/* Weight scale granularity: one fp32 per row, or one fp16 per 32 values of a row. */
enum { MOE_SCALE_ROW_F32 = 0, MOE_SCALE_G32_F16 = 1 };
/* Activation quantization: one fp32 scale per token, or Q8_0-style fp16 per 32. */
enum { MOE_ACT_TOKEN_F32 = 0, MOE_ACT_G32_F16 = 1 };
/* Router scoring. */
enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID_NOAUX_TC = 1 };

/* moe_route_cfg.flags */
#define MOE_FLAG_DEBUG 1u          /* also keep gate/up stage values, per-pair down values and
                                      the down projection's int32 group dots in the workspace
                                      (see moe_layer_debug_views) */
#define MOE_FLAG_FORCE_GEMV 2u     /* run every expert on the weight-streaming (GEMV) path */
#define MOE_FLAG_FORCE_MMA 4u      /* T > 32: run every expert (shared one included) with at least
                                      one pair on the tensor-core path (normally: >= 16 pairs) */
#define MOE_FLAG_SHORT_WAITS 8u    /* the single-token kernel's waits on other CTAs (its grid
                                      barrier) give up after about 2 ms instead of about a second
                                      (MOE_ERR_TIMEOUT): for testing the timeout path */

/* A set of E quantized experts of one layer (or the single shared expert, E = 1).
 *
 * `data` (device, 256-byte aligned, caller-owned) holds `bytes` >= moe_expert_blob_bytes().
 * Byte layout, four regions each starting at a multiple of 256 bytes from `data`:
 *   R0 gate/up codes: for each expert e, for each s in [0, I/64): a block of
 *      128 rows -- rows 0..63 are gate rows 64s..64s+63, rows 64..127 the up
 *      rows of the same intermediate indices -- stored as [KB/16][128][16]:
 *      16-byte piece p of row r at (p * 128 + r) * 16. KB = H (int8), H/2
 *      (int4) or H/4 (int2) code bytes per row. One block's K range is one
 *      contiguous run, one piece of it 2 KB.
 *   R1 down codes: the [H][I] matrix of expert e cut along I into slabs of 64
 *      intermediate indices: for each e, each u in [0, I/64), each b in
 *      [0, H/128): rows 128b..128b+127, columns 64u..64u+63, stored
 *      [SB/16][128][16] (SB = 64 bytes int8, 32 bytes int4, 16 bytes int2). One
 *      slab (all H rows of 64 columns) is one contiguous run.
 *   R2 gate/up scales: for each e, each 128-row block: fp16 [H/32][128]
 *      (group-major) or fp32 [128].
 *   R3 down scales: fp16: for each e, u, b as in R1: [2][128] (the two groups
 *      of the slab); fp32: [E][H], one per row.
 * Padding bytes between regions are zero. */
typedef struct {
  int32_t wtype;      /* MOE_W_INT8 | MOE_W_INT4 | MOE_W_INT2 */
  int32_t wscale;     /* MOE_SCALE_ROW_F32 | MOE_SCALE_G32_F16 */
  int32_t n_experts;  /* E */
  int32_t hidden;     /* H */
  int32_t inter;      /* I */
  int32_t reserved;
  void* data;         /* device */
  size_t bytes;
} moe_expert_blob;

typedef struct {
  int32_t score;                /* MOE_SCORE_* */
  int32_t top_k;
  int32_t renormalize;          /* softmax: weights over the selected experts sum to 1;
                                   sigmoid: weights = s / sum of selected s */
  float routed_scaling_factor;  /* multiplies every routing weight (1.0 for plain softmax) */
  int32_t act;                  /* MOE_ACT_* (applies to x and to h) */
  uint32_t flags;               /* MOE_FLAG_* */
  float top_p;                  /* adaptive expert top-p (the GLM-5.2 colibri page's "--topp"):
                                   0 or >= 1 = off (every token keeps its k experts). In (0, 1):
                                   per token, slot j of the top-k list (descending key) has mass
                                   v_j = exp(L_j - L_0) (softmax) or sigmoid(L_j); D = v_0 + ... +
                                   v_{k-1} and C_m = v_0 + ... + v_{m-1} are fp32 sums in slot
                                   order, and the first m slots are kept for the first m with
                                   C_m >= top_p * D. Dropped slots get idx -1 and weight 0 and
                                   their experts are not read for that token; with renormalize
                                   the kept weights are renormalized over the kept experts.
                                   Must be finite and >= 0 (else MOE_ERR_INVALID_ARG). */
  int32_t n_experts_total;      /* expert parallelism (the GLM-5.2 colibri page, "Experimental
                                   resident CUDA backend": whole experts placed on devices). 0 = the
                                   layer holds every expert (E = experts->n_experts). Otherwise the
                                   router has n_experts_total experts (router_w [n_experts_total][H],
                                   router_bias [n_experts_total]) and `experts` holds the contiguous
                                   range expert_begin .. expert_begin + experts->n_experts - 1 of
                                   them: every token is routed over all n_experts_total experts
                                   (idx and w hold global ids and weights, the same on every
                                   device), and only pairs whose expert is in the range are computed
                                   and added into y. Summing y over devices that hold disjoint ranges
                                   covering all experts (the shared expert on one of them) gives the
                                   layer. Requires expert_begin >= 0, expert_begin + n_experts <=
                                   n_experts_total <= 1024 (else MOE_ERR_UNSUPPORTED). */
  int32_t expert_begin;         /* first global expert id held by `experts` (0 without EP) */
} moe_route_cfg;

/* Version of this ABI (MOE_ABI_VERSION). */
MOE_API int32_t moe_abi_version(void);

/* Description of the last MOE_ERR_CUDA returned on the calling host thread (which call
 * failed and the CUDA error text); "" if none. Valid until the thread's next failing call. */
MOE_API const char* moe_last_error(void);

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status s);

/* Bytes a blob of this format needs; 0 if the shape or format is unsupported. */
MOE_API size_t moe_expert_blob_bytes(int32_t wtype, int32_t wscale, int32_t n_experts, int32_t hidden,
                             int32_t inter);

/* Quantize fp32 expert weights into `out` (GLM page, "Quantization kernels: int8 / packed
 * int4 ... per-row scales, dequant-on-use"; group size 32 from the mtlm-7m-base card).
 *   w_gate_up [E][2I][H] fp32: rows 0..I-1 the gate projection, I..2I-1 the up projection;
 *   w_down    [E][H][I] fp32.
 * out->wtype, wscale, n_experts, hidden, inter, data and bytes are set by the caller;
 * the blob is fully rewritten (padding zeroed). Errors: INVALID_ARG (null), UNSUPPORTED
 * (shape), WORKSPACE (out->bytes too small). */
MOE_API moe_status moe_quantize_experts(const float* w_gate_up, const float* w_down,
                                const moe_expert_blob* out, void* stream);

/* The GLM-5.2 colibri page's FP8 -> int4 converter step, on the GPU: FP8 checkpoint weights
 * (float8 E4M3 codes, "fn" variant: no infinities) with one fp32 inverse scale per 128 x 128
 * block of each expert's matrix (the DeepSeek-V3-style layout) are dequantized -- value =
 * code (exact in fp32) * its block's scale, one fp32 rounding -- and quantized into `out`
 * exactly as moe_quantize_experts quantizes fp32 weights (any wtype / wscale).
 *   w_gate_up: uint8 [E][2I][H] (gate rows then up rows per expert), s_gate_up: fp32
 *   [E][ceil(2I/128)][ceil(H/128)]; w_down: uint8 [E][H][I], s_down: fp32
 *   [E][ceil(H/128)][ceil(I/128)]. All device memory, caller-owned, read only.
 * NaN codes (0x7f, 0xff) are invalid input (the blob is then undefined). Errors as
 * moe_quantize_experts. */
MOE_API moe_status moe_quantize_experts_fp8(const uint8_t* w_gate_up, const float* s_gate_up,
                                            const uint8_t* w_down, const float* s_down,
                                            const moe_expert_blob* out, void* stream);

/* Q8_0-style activation quantization (GLM page, "Integer-dot kernels (Q8_0-style int8
 * activations ...)").  x [T][H] fp32 -> q [T][H] int8 and `scales`: fp16 [T][H/32]
 * (MOE_ACT_G32_F16) or fp32 [T] (MOE_ACT_TOKEN_F32). H multiple of 32; x 16-byte, q and
 * scales 4-byte aligned (MOE_ERR_INVALID_ARG otherwise). */
MOE_API moe_status moe_quantize_activations(const float* x, int32_t T, int32_t H, int32_t act,
                                    int8_t* q, void* scales, void* stream);

/* Router logits [T][E] = x [T][H] . router_w [E][H]^T in the fixed fp32 order above. x and
 * router_w 16-byte aligned (MOE_ERR_INVALID_ARG otherwise). */
MOE_API moe_status moe_router_logits(const float* x, const float* router_w, int32_t T, int32_t E,
                             int32_t H, float* logits, void* stream);

/* Top-k selection and routing weights from logits [T][E] (GLM page: "DeepSeek-V3-style
 * sigmoid router (noaux_tc, routed_scaling_factor)"; OLMoE page: "top-8 of 64").
 * bias [E] (sigmoid mode only, may be NULL = zeros) shifts the selection key, never the
 * weights. idx [T][k] int32 in descending key order (ties: lower expert index first),
 * w [T][k] fp32. With cfg->top_p in (0, 1) (adaptive top-p, see moe_route_cfg) the slots
 * after each token's kept prefix hold idx -1 and w 0. */
MOE_API moe_status moe_route_topk(const float* logits, const float* bias, int32_t T, int32_t E,
                          const moe_route_cfg* cfg, int32_t* idx, float* w, void* stream);

/* Workspace bytes moe_permute needs for (T, k, E). */
MOE_API size_t moe_permute_workspace_bytes(int32_t T, int32_t k, int32_t E);

/* Batch-union grouping (GLM page, "Batch-union MoE"): offsets [E+1] (offsets[e] = first
 * position of expert e) and perm [offsets[E]], the pair indices t*k+j sorted by (expert, t).
 * idx values must lie in [0, E) or be -1 (a slot dropped by adaptive top-p: left out, so
 * offsets[E] = the kept pairs); other values set MOE_ERR_DEVICE_CHECK in the workspace
 * status word and are dropped. */
MOE_API moe_status moe_permute(const int32_t* idx, int32_t T, int32_t k, int32_t E, int32_t* offsets,
                       int32_t* perm, void* workspace, size_t ws_bytes, void* stream);

/* moe_permute without a workspace argument and without allocating. (The pages have no
 * counterpart: this exists for callers that can neither allocate device memory nor pass a
 * scratch buffer -- code running during CUDA graph capture, serving loops whose memory is
 * fully owned by a framework allocator, plugin hosts that hand an operator only its tensors.)
 * Scratch is a 1 MiB array compiled into the library as a device global, so every GPU that
 * loads the library holds it until the process exits; a grouping whose scratch need,
 * moe_permute_workspace_bytes(T, k, E), exceeds 1 MiB returns MOE_ERR_WORKSPACE (for example
 * T = 4096 with E = 512 fits, T = 8192 with E = 1024 does not). The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress); make that first call before
 * any stream capture on that device. All calls share the one array: calls that may overlap
 * on the GPU (different streams without ordering, several host threads) race and corrupt
 * each other's results; order them on one stream. Out-of-range expert ids are dropped, as in
 * moe_permute; the device status word that records them is not readable through this entry
 * point. Other errors and arguments as moe_permute. */
MOE_API moe_status moe_permute_no_alloc(const int32_t* idx, int32_t T, int32_t k, int32_t E,
                                        int32_t* offsets, int32_t* perm, void* stream);

/* Workspace bytes moe_layer_forward needs; 0 if the arguments are unsupported. */
MOE_API size_t moe_layer_workspace_bytes(int32_t T, const moe_expert_blob* experts,
                                 const moe_expert_blob* shared, const moe_route_cfg* cfg);

/* The whole layer: y [T][H] fp32 (overwritten) from x [T][H] fp32 (x, y and router_w 16-byte
 * aligned, the workspace 256-byte aligned: MOE_ERR_INVALID_ARG otherwise).
 *   router_w [E][H] fp32; router_bias [E] fp32 or NULL (sigmoid mode only);
 *   experts: the routed experts; shared: NULL or one expert (n_experts = 1) with the same
 *   hidden size, wtype and wscale as `experts` and its own intermediate size.
 * workspace: device buffer of ws_bytes >= moe_layer_workspace_bytes(); it holds every
 * intermediate (quantized x, logits, routing, grouping, quantized h) and, in its first 256
 * bytes, a control block (device status word, routing ticket, wait record, and at bytes 16-23
 * the single-token grid-barrier counter). The control block must be zero before the workspace
 * is first used (allocate it zeroed, e.g. cudaMemset once); the library leaves it consistent
 * after every call. Calls that share a workspace must be ordered on one stream.
 * Launch sequence: one token with group-32 activations (decode) is ONE launch: every CTA of
 * the expert kernel quantizes the token, computes the router logits of a share of the
 * experts and zeroes a share of y; after a grid barrier (all CTAs resident: the grid is at
 * most one CTA per SM) every CTA selects the same top-k (with adaptive top-p: the same kept
 * prefix, in a separate instantiation of that kernel) and streams its work units. Other
 * calls: for T <= 32 one routing kernel (activation quantization, logits, top-k and grouping;
 * the last CTA to finish its logit does the selection), larger T four; then, with group-32
 * activations, one expert kernel that covers the routed and the shared experts: per work unit
 * (expert, 64 intermediate indices) gate/up, SwiGLU, h quantization and the unit's share of
 * the down projection, added into y. With per-token activation scales h needs all of I first:
 * gate/up, h quantization, then down as separate launches. Kernels use programmatic dependent
 * launch, so under stream capture the graph gets programmatic edges; router_w and the expert
 * blobs are model parameters, read (the single-token kernel: router rows staged) before a
 * kernel waits for its predecessor in the stream, so they must not be written by it. */
MOE_API moe_status moe_layer_forward(const float* x, int32_t T, const float* router_w,
                             const float* router_bias, const moe_expert_blob* experts,
                             const moe_expert_blob* shared, const moe_route_cfg* cfg, float* y,
                             void* workspace, size_t ws_bytes, void* stream);

/* Stages of moe_layer_forward, in launch order. */
enum {
  MOE_STAGE_QUANT_X = 0,   /* activation quantization (also zeroes y) */
  MOE_STAGE_ROUTER = 1,    /* router logits */
  MOE_STAGE_TOPK = 2,      /* top-k selection and weights (grouping too when T = 1) */
  MOE_STAGE_GROUP = 3,     /* batch-union grouping (T > 1) */
  MOE_STAGE_GATE_UP = 4,   /* gate/up + SwiGLU (group-32 activations: the whole expert kernel,
                              h quantization, down projection and combine included) */
  MOE_STAGE_QUANT_H = 5,   /* h quantization (per-token activation scales only) */
  MOE_STAGE_DOWN = 6,      /* down projection + weighted combine (per-token scales only) */
  MOE_STAGE_COUNT = 7
};

/* Caller-created CUDA events (cudaEvent_t, may be NULL) recorded on `stream` just before
 * the first and just after the last kernel of each stage; a stage that launches nothing
 * records both events back to back. Inside stream capture they are recorded as external
 * event nodes, so cudaEventElapsedTime works on them after the graph runs. */
typedef struct {
  void* begin[MOE_STAGE_COUNT];
  void* end[MOE_STAGE_COUNT];
} moe_stage_events;

/* moe_layer_forward with per-stage event records (profiling). */
MOE_API moe_status moe_layer_forward_timed(const float* x, int32_t T, const float* router_w,
                                           const float* router_bias,
                                           const moe_expert_blob* experts,
                                           const moe_expert_blob* shared,
                                           const moe_route_cfg* cfg, float* y, void* workspace,
                                           size_t ws_bytes, void* stream,
                                           const moe_stage_events* events);

/* moe_layer_forward with x and y in host memory: enqueues on `stream` the copy of x_host
 * [T][H] into x_dev, the layer (y_dev [T][H]) and the copy of y_dev into y_host, and returns
 * (synchronize `stream` before reading y_host). x_host / y_host should be page-locked
 * (cudaHostAlloc) for the copies to be asynchronous; x_dev / y_dev are device buffers of
 * T * H floats, 16-byte aligned, owned by the caller, used as this call's staging: with
 * page-locked (device-mapped) host buffers the SMs move x and y in kernels chained to the
 * layer's, and x_dev may be written before work enqueued earlier on `stream` has finished, so
 * such work must not read x_dev. Errors as moe_layer_forward, plus INVALID_ARG for a null
 * buffer and CUDA for a failed copy. */
MOE_API moe_status moe_layer_forward_host(const float* x_host, int32_t T, const float* router_w,
                                          const float* router_bias, const moe_expert_blob* experts,
                                          const moe_expert_blob* shared, const moe_route_cfg* cfg,
                                          float* x_dev, float* y_dev, float* y_host, void* workspace,
                                          size_t ws_bytes, void* stream);

/* Number of kernels one moe_layer_forward call with these arguments launches. */
MOE_API int32_t moe_layer_kernel_count(int32_t T, const moe_expert_blob* experts,
                                       const moe_expert_blob* shared, const moe_route_cfg* cfg);

/* Byte offsets, inside a moe_layer_forward workspace, of the intermediates of the last
 * call with the same (T, experts, shared, cfg). -1 = not kept for this configuration.
 * Pair rows are in grouped order: row r of q_h / s_h / gate / up / y_pair belongs to the
 * (token, slot) pair perm[r]; shared-expert rows follow as rows T*k + t. */
typedef struct {
  int64_t status;       /* int32 device status word (moe_status value) */
  int64_t q_x;          /* int8 [T][H] */
  int64_t s_x;          /* fp16 [T][H/32] or fp32 [T] */
  int64_t logits;       /* fp32 [T][E] */
  int64_t idx;          /* int32 [T][k] */
  int64_t w;            /* fp32 [T][k] */
  int64_t offsets;      /* int32 [E+1] */
  int64_t perm;         /* int32 [T*k] */
  int64_t n_active;     /* int32: number of distinct experts selected */
  int64_t act_expert;   /* int32 [n_active] distinct experts, ascending */
  int64_t q_h;          /* int8 [T*k][I] then [T][I_shared] */
  int64_t s_h;          /* fp16 [T*k][I/32] then [T][I_s/32], or fp32 [T*k] then [T] */
  int64_t gate;         /* MOE_FLAG_DEBUG: fp32 [T*k][I] then [T][I_s] */
  int64_t up;           /* MOE_FLAG_DEBUG: fp32, same shape */
  int64_t y_pair;       /* MOE_FLAG_DEBUG: fp32 [T*k][H] then [T][H]: expert outputs before
                           the combine */
  int64_t dn_dots;      /* MOE_FLAG_DEBUG: int32 [T*k][H][I/32] then [T][H][I_shared/32]: the
                           exact int32 group dots of the down projection (row n of the down
                           matrix against the pair's q_h, per group of 32), as the expert kernel
                           that ran the pair formed them; entries of dropped slots are 0. Size
                           4 * H * (T*k*I + T*I_shared) / 32 bytes. */
  int64_t total;        /* == moe_layer_workspace_bytes() */
} moe_debug_views;

MOE_API moe_status moe_layer_debug_views(int32_t T, const moe_expert_blob* experts,
                                 const moe_expert_blob* shared, const moe_route_cfg* cfg,
                                 moe_debug_views* out);

/* Per-group exact int32 dots of sampled expert rows against given int8 activation rows, read
 * through the blob layout (the integer-dot step of the GLM page's "Integer-dot kernels").
 *   which 0: gate/up rows (logical row r in [0, 2I) of [2I][H]), K = H;
 *   which 1: down rows (r in [0, H) of [H][I]), K = I.
 * expert [n], row [n]: int32; act [n][K] int8; dots [n][K/32] int32. */
MOE_API moe_status moe_expert_group_dots(const moe_expert_blob* blob, int32_t which, int32_t n,
                                 const int32_t* expert, const int32_t* row, const int8_t* act,
                                 int32_t* dots, void* stream);

/* The control block's int32 words [2] and [3] record the first bounded wait that gave up
 * during the last call (MOE_ERR_TIMEOUT): [2] = pass (1 gate/up, 2 down) | wait << 4 | ring
 * stage or buffer << 8, with wait 0 = producer waiting for a free stage, 1 = consumer waiting
 * for a chunk, 2 / 4 = producer draining chunks / activation copies before exit, 3 = producer
 * waiting for a free activation buffer, 5 = consumer waiting for activation rows, 6 = the
 * single-token kernel's grid barrier, 7 = its staged router rows, 8 = the y-zero barrier of its
 * cluster variant (logits exchanged within clusters of CTAs, y zeroed before any CTA adds);
 * [3] = the CTA index; both 0 otherwise. After MOE_ERR_TIMEOUT the routing ticket and the
 * grid-barrier counter may be mid-call: reading the status resets them (not words 2-3).
 * Reads and clears the device status word of a moe_layer_forward / moe_permute workspace.
 * Synchronizes `stream`. Returns MOE_OK, MOE_ERR_DEVICE_CHECK or MOE_ERR_TIMEOUT as
 * recorded by the kernels, or MOE_ERR_CUDA if the copy fails. */
MOE_API moe_status moe_read_device_status(void* workspace, size_t ws_bytes, void* stream);

/* moe_read_device_status for a workspace of at least its 256-byte control block (every
 * moe_layer_forward and moe_permute workspace): the status query without a size. Synchronizes
 * `stream`; same returns. */
MOE_API moe_status moe_get_device_status(void* workspace, void* stream);

/* moe_layer_forward with MOE_FLAG_DEBUG added to cfg->flags (so the workspace must hold
 * moe_layer_workspace_bytes() of that configuration), and `views` filled as
 * moe_layer_debug_views() fills it: byte offsets, inside `workspace`, of the call's
 * intermediates (quantized x, logits, idx, w, grouping, quantized h, gate/up stage values,
 * per-pair down values and the down projection's int32 group dots). Errors as
 * moe_layer_forward, plus INVALID_ARG for a null cfg or views; views is written only when the
 * call returns MOE_OK with T > 0. */
MOE_API moe_status moe_layer_forward_debug(const float* x, int32_t T, const float* router_w,
                                           const float* router_bias, const moe_expert_blob* experts,
                                           const moe_expert_blob* shared, const moe_route_cfg* cfg,
                                           float* y, void* workspace, size_t ws_bytes, void* stream,
                                           moe_debug_views* views);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
