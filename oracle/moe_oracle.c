/*
 * moe_oracle.c -- plain, slow CPU oracle of the quantized MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. It shares no code, header, table or
 * constant generator with the CUDA path, and the CUDA path never calls it.
 *
 * What the layer computes (the "Show HN: getting GLM-5.2 running on my slow
 * compute" page, "What's implemented"; the OLMoE page "I ran a 7B
 * Mixture-of-Experts LLM in a language I built", "Mixture-of-Experts"):
 *   1. router logits L = x . W_r^T, then top-k selection by softmax or by the
 *      DeepSeek-V3-style sigmoid noaux_tc rule with routed_scaling_factor
 *      (GLM page, "DeepSeek-V3-style sigmoid router (noaux_tc,
 *      routed_scaling_factor), shared expert");
 *   2. Q8_0-style int8 activations and int8 / packed-int4 expert weights with
 *      per-row or group-32 scales, dequantized on use around integer dot
 *      products (GLM page, "Integer-dot kernels" and "Quantization kernels";
 *      group size 32 from the mtlm-7m-base model card, "Files");
 *   3. SwiGLU expert FFN (mtlm-7m-base card, architecture list), down
 *      projection, weighted combine plus an optional shared expert;
 *   4. batch-union grouping: each unique expert applied to every position that
 *      routes to it (GLM page, "Batch-union MoE").
 *
 * Precision. Where a floating-point value decides an integer (a quantized
 * code, a top-k selection) the decision is taken in fp32 with the fixed
 * operation sequence written out below, because that is the precision the
 * kernel decides in; everything else (routing weights, down projection,
 * combine) is fp64. The pages fix none of these sequences; the readings are:
 *   - quantization: scale d = amax / Q in fp32 (Q = 127 int8, 7 int4), stored
 *     as fp32 (per row / per token) or rounded to fp16 (group of 32); codes
 *     q = clamp(round_half_away(w / stored_d), -Q, Q), q = 0 when stored_d = 0;
 *   - int4 packing: two's-complement nibbles, element 2j in the low nibble of
 *     byte j, element 2j+1 in the high nibble;
 *   - router logits: per 32-element chunk a sequential fmaf chain from +0 in
 *     ascending index, chunk partials added in ascending chunk order;
 *   - sigmoid: s = 1 / (1 + cexp(-L)); selection key s + bias; top-k ordered
 *     by descending key, ties to the lower expert index;
 *   - stage value of an expert row: exact int32 dot I_g per group of 32, then
 *     acc = fmaf((float)I_g, c_g, acc) for ascending g from +0, where c_g is
 *     the product of the two group scales (both group-32), or the one scale
 *     that varies by group; the scale that does not vary multiplies the end;
 *     per-row weights with per-token activations form one group (the row);
 *   - SwiGLU: h = (g / (1 + cexp(-g))) * u;
 *   - cexp: own fp32 exp (Cody-Waite two-constant reduction by ln 2, degree-7
 *     Taylor polynomial in Horner form, exponent scaling), input clamped to
 *     [-87, 88];
 *   - adaptive expert top-p (the GLM page's "--topp" knob, "adaptive expert
 *     top-p", which it credits with 30-40% less expert reading): the mass of
 *     slot j of a token's top-k list is v_j = cexp(L_j - L_0) (softmax; slot 0
 *     holds the largest logit) or sigmoid(L_j); D = v_0 + ... + v_{k-1} and
 *     C_m = v_0 + ... + v_{m-1} are fp32 sums in slot order; the kept count m is
 *     the first m with C_m >= top_p * D (fp32 product). Dropped slots get
 *     expert -1 and weight 0; with renormalisation the kept weights are
 *     renormalised over the kept experts.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- utilities */

static float f16_round(float d) { _Float16 h = (_Float16)d; return (float)h; }
static uint16_t f16_bits(float d) { _Float16 h = (_Float16)d; uint16_t b; memcpy(&b, &h, 2); return b; }

/* exp(a) in fp32. ln 2 split into a 24-bit head and the fp32-rounded tail
 * (Cody & Waite); 1/k! Taylor coefficients rounded to fp32. */
float orc_cexp(float a) {
  if (a > 88.0f) a = 88.0f;
  if (a < -87.0f) a = -87.0f;
  const float log2e = 0x1.715476p+0f;
  const float ln2_hi = 0x1.62e43p-1f;
  const float ln2_lo = -0x1.05c61p-29f;
  float kf = rintf(a * log2e);
  float r = fmaf(-kf, ln2_hi, a);
  r = fmaf(-kf, ln2_lo, r);
  float p = 0x1.a01a02p-13f;           /* 1/7! */
  p = fmaf(p, r, 0x1.6c16c2p-10f);      /* 1/6! */
  p = fmaf(p, r, 0x1.111112p-7f);       /* 1/5! */
  p = fmaf(p, r, 0x1.555556p-5f);       /* 1/4! */
  p = fmaf(p, r, 0x1.555556p-3f);       /* 1/3! */
  p = fmaf(p, r, 0.5f);                 /* 1/2! */
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int n = (int)kf;
  uint32_t bits = (uint32_t)(n + 127) << 23;
  float two;
  memcpy(&two, &bits, 4);
  return p * two;
}

float orc_sigmoid(float L) { return 1.0f / (1.0f + orc_cexp(-L)); }

float orc_swiglu(float g, float u) {
  float den = 1.0f + orc_cexp(-g);
  float sg = g / den;
  return sg * u;
}

/* Array forms of the three scalar functions above, for the tests. */
void orc_cexp_n(const float* a, int64_t n, float* out) { for (int64_t i = 0; i < n; ++i) out[i] = orc_cexp(a[i]); }
void orc_sigmoid_n(const float* a, int64_t n, float* out) { for (int64_t i = 0; i < n; ++i) out[i] = orc_sigmoid(a[i]); }
void orc_swiglu_n(const float* g, const float* u, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_swiglu(g[i], u[i]);
}

static int quant_code(float v, float s, int qmax) {
  if (s == 0.0f) return 0;
  float r = roundf(v / s);
  if (r > (float)qmax) r = (float)qmax;
  if (r < -(float)qmax) r = -(float)qmax;
  return (int)r;
}

/* ------------------------------------------------------------ quantization */

/* Symmetric quantization of N rows of K values.
 * g32 != 0: one fp16-rounded scale per 32 consecutive values, s = [N][K/32].
 * g32 == 0: one fp32 scale per row, s = [N].  q = [N][K] codes in [-qmax, qmax]. */
int orc_quantize_rows(const float* w, int64_t N, int K, int qmax, int g32, int8_t* q, float* s) {
  if (K <= 0 || (g32 && K % 32) || qmax <= 0) return 1;
  for (int64_t n = 0; n < N; ++n) {
    const float* row = w + n * (int64_t)K;
    int8_t* qr = q + n * (int64_t)K;
    if (g32) {
      int G = K / 32;
      for (int g = 0; g < G; ++g) {
        float amax = 0.0f;
        for (int k = 32 * g; k < 32 * g + 32; ++k) {
          float a = fabsf(row[k]);
          if (a > amax) amax = a;
        }
        float d = f16_round(amax / (float)qmax);
        s[n * G + g] = d;
        for (int k = 32 * g; k < 32 * g + 32; ++k) qr[k] = (int8_t)quant_code(row[k], d, qmax);
      }
    } else {
      float amax = 0.0f;
      for (int k = 0; k < K; ++k) {
        float a = fabsf(row[k]);
        if (a > amax) amax = a;
      }
      float d = amax / (float)qmax;
      s[n] = d;
      for (int k = 0; k < K; ++k) qr[k] = (int8_t)quant_code(row[k], d, qmax);
    }
  }
  return 0;
}

/* Pack int4 codes two per byte: element 2j low nibble, 2j+1 high nibble. */
int orc_pack_int4(const int8_t* q, int64_t N, int K, uint8_t* out) {
  if (K % 2) return 1;
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < K / 2; ++j) {
      uint8_t lo = (uint8_t)q[n * K + 2 * j] & 0x0F;
      uint8_t hi = (uint8_t)q[n * K + 2 * j + 1] & 0x0F;
      out[n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
    }
  return 0;
}

/* Pack int2 codes four per byte (the GLM page's "packed int2"): element 4j + i in bits
 * 2i .. 2i + 1 of byte j, two's complement (codes -1, 0, 1 under the symmetric rule). */
int orc_pack_int2(const int8_t* q, int64_t N, int K, uint8_t* out) {
  if (K % 4) return 1;
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < K / 4; ++j) {
      uint8_t b = 0;
      for (int i = 0; i < 4; ++i) b |= (uint8_t)(((uint8_t)q[n * K + 4 * j + i] & 3u) << (2 * i));
      out[n * (K / 4) + j] = b;
    }
  return 0;
}

/* Code bytes of K elements of a row. */
static uint64_t code_bytes(uint64_t K, int wbits) { return K * (uint64_t)wbits / 8; }

/* ------------------------------------------------------ expert blob layout */
/* The blob byte layout is the one the library's public header documents:
 * four regions (gate/up codes, down codes, gate/up scales, down scales), each
 * starting at a multiple of 256 bytes; codes stored in 16-byte pieces
 * [row-block][piece][row][16 bytes] with 128-row gate/up blocks (64 gate rows
 * then the 64 matching up rows), scales [row-block][group][row] (fp16) or
 * [row-block][row] (fp32); the down matrix is cut along I into slabs of 64
 * intermediate indices, each slab [128-row block][piece][row][16 bytes] with
 * fp16 scales [slab][128-row block][2 groups][row], fp32 scales [expert][row]. */

static uint64_t al256(uint64_t v) { return (v + 255) & ~(uint64_t)255; }

int orc_blob_layout(int E, int H, int I, int wbits, int g32, uint64_t* off /* [5] */) {
  if (E <= 0 || H <= 0 || I <= 0 || H % 128 || I % 128 || (wbits != 8 && wbits != 4 && wbits != 2)) return 1;
  uint64_t kb_gu = code_bytes((uint64_t)H, wbits);
  uint64_t kb_dn = code_bytes((uint64_t)I, wbits);
  uint64_t s_gu = g32 ? (uint64_t)(H / 32) * 2 : 4;
  uint64_t s_dn = g32 ? (uint64_t)(I / 32) * 2 : 4;
  off[0] = 0;
  off[1] = al256(off[0] + (uint64_t)E * 2 * I * kb_gu);
  off[2] = al256(off[1] + (uint64_t)E * H * kb_dn);
  off[3] = al256(off[2] + (uint64_t)E * 2 * I * s_gu);
  off[4] = al256(off[3] + (uint64_t)E * H * s_dn);
  return 0;
}

static void put_row(uint8_t* region, int rows_per_block, uint64_t kb, int64_t block, int r,
                    const uint8_t* rowbytes) {
  uint8_t* base = region + (uint64_t)block * rows_per_block * kb;
  for (uint64_t b = 0; b < kb; ++b)
    base[(b / 16) * rows_per_block * 16 + (uint64_t)r * 16 + (b % 16)] = rowbytes[b];
}

static void row_bytes(const int8_t* q, int K, int wbits, uint8_t* out) {
  if (wbits == 8) {
    for (int k = 0; k < K; ++k) out[k] = (uint8_t)q[k];
  } else if (wbits == 4) {
    orc_pack_int4(q, 1, K, out);
  } else {
    orc_pack_int2(q, 1, K, out);
  }
}

/* q_gu [E][2I][H], s_gu ([E][2I][H/32] | [E][2I]); q_dn [E][H][I], s_dn ([E][H][I/32] | [E][H]). */
int orc_pack_blob(int E, int H, int I, int wbits, int g32, const int8_t* q_gu, const float* s_gu,
                  const int8_t* q_dn, const float* s_dn, uint8_t* blob) {
  uint64_t off[5];
  if (orc_blob_layout(E, H, I, wbits, g32, off)) return 1;
  memset(blob, 0, off[4]);
  uint64_t kb_gu = code_bytes((uint64_t)H, wbits);
  uint64_t kb_dn = code_bytes((uint64_t)I, wbits);
  int Gg = H / 32, Gd = I / 32;
  uint8_t* rb = (uint8_t*)malloc(kb_gu > kb_dn ? kb_gu : kb_dn);
  for (int e = 0; e < E; ++e) {
    /* gate/up */
    for (int sb = 0; sb < I / 64; ++sb)
      for (int r = 0; r < 128; ++r) {
        int64_t lr = r < 64 ? 64 * sb + r : (int64_t)I + 64 * sb + (r - 64);
        int64_t grow = (int64_t)e * 2 * I + lr;
        row_bytes(q_gu + grow * H, H, wbits, rb);
        put_row(blob + off[0] + (uint64_t)e * 2 * I * kb_gu, 128, kb_gu, sb, r, rb);
        if (g32) {
          uint16_t* sr = (uint16_t*)(blob + off[2] + ((uint64_t)e * 2 * I + (uint64_t)sb * 128) * Gg * 2);
          for (int g = 0; g < Gg; ++g) sr[g * 128 + r] = f16_bits(s_gu[grow * Gg + g]);
        } else {
          float* sr = (float*)(blob + off[2] + ((uint64_t)e * 2 * I + (uint64_t)sb * 128) * 4);
          sr[r] = s_gu[grow];
        }
      }
    /* down: slab (e, u) = all H rows x intermediate indices 64u .. 64u+63, stored as
       128-row blocks [hb][piece][row][16 bytes]; g32 scales [slab][hb][2][row] */
    {
      const int U = I / 64, HB = H / 128;
      const uint64_t sbytes = kb_dn / U;     /* code bytes of 64 elements: 64, 32 or 16 */
      for (int n = 0; n < H; ++n) {
        int64_t grow = (int64_t)e * H + n;
        int hb = n / 128, r = n % 128;
        row_bytes(q_dn + grow * I, I, wbits, rb);
        for (int u = 0; u < U; ++u) {
          uint64_t slab = ((uint64_t)e * U + u) * HB + hb;
          uint8_t* base = blob + off[1] + slab * 128 * sbytes;
          for (uint64_t bb = 0; bb < sbytes; ++bb)
            base[(bb / 16) * 128 * 16 + (uint64_t)r * 16 + bb % 16] = rb[u * sbytes + bb];
          if (g32) {
            uint16_t* sr = (uint16_t*)(blob + off[3] + slab * 2 * 128 * 2);
            for (int j = 0; j < 2; ++j) sr[j * 128 + r] = f16_bits(s_dn[grow * Gd + 2 * u + j]);
          }
        }
        if (!g32) ((float*)(blob + off[3]))[grow] = s_dn[grow];
      }
    }
  }
  free(rb);
  return 0;
}

/* ------------------------------------------------------------------ routing */

void orc_router_logits(const float* x, const float* Wr, int T, int E, int H, float* L) {
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      const float* xr = x + (int64_t)t * H;
      const float* wr = Wr + (int64_t)e * H;
      float total = 0.0f;
      for (int c = 0; c < H / 32; ++c) {
        float part = 0.0f;
        for (int h = 32 * c; h < 32 * c + 32; ++h) part = fmaf(xr[h], wr[h], part);
        total = total + part;
      }
      L[(int64_t)t * E + e] = total;
    }
}

typedef struct { float key; int e; } keyed;

static int by_key_desc(const void* a, const void* b) {
  const keyed* p = (const keyed*)a;
  const keyed* q = (const keyed*)b;
  if (p->key > q->key) return -1;
  if (p->key < q->key) return 1;
  return p->e < q->e ? -1 : (p->e > q->e ? 1 : 0);
}

/* Adaptive top-p cut of one token's top-k list (slot order): the number of slots kept. */
static int topp_keep(const float* Lt, const keyed* ks, int score, int k, float top_p) {
  float v[1024];
  for (int j = 0; j < k; ++j)
    v[j] = score == 0 ? orc_cexp(Lt[ks[j].e] - Lt[ks[0].e]) : orc_sigmoid(Lt[ks[j].e]);
  float D = 0.0f;
  for (int j = 0; j < k; ++j) D = D + v[j];
  const float thr = top_p * D;
  float c = 0.0f;
  for (int j = 0; j < k; ++j) {
    c = c + v[j];
    if (c >= thr) return j + 1;
  }
  return k;
}

/* score 0 = softmax, 1 = sigmoid noaux_tc. idx [T][k], w [T][k] (fp64). top_p in (0, 1):
 * adaptive top-p (dropped slots: idx -1, w 0); other values: off. */
int orc_route(const float* L, const float* bias, int T, int E, int score, int k, int renorm,
              float rsf, float top_p, int32_t* idx, double* w) {
  if (k <= 0 || k > E) return 1;
  keyed* ks = (keyed*)malloc(sizeof(keyed) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* Lt = L + (int64_t)t * E;
    for (int e = 0; e < E; ++e) {
      ks[e].e = e;
      if (score == 0) ks[e].key = Lt[e];
      else ks[e].key = orc_sigmoid(Lt[e]) + (bias ? bias[e] : 0.0f);
    }
    qsort(ks, (size_t)E, sizeof(keyed), by_key_desc);
    /* kept slots: all k, or the adaptive top-p prefix; the renormalised weights are taken
       over the kept slots */
    const int m = (top_p > 0.0f && top_p < 1.0f) ? topp_keep(Lt, ks, score, k, top_p) : k;
    for (int j = 0; j < k; ++j) {
      idx[(int64_t)t * k + j] = j < m ? ks[j].e : -1;
      w[(int64_t)t * k + j] = 0.0;
    }
    if (score == 0) {
      double M = -INFINITY;
      for (int e = 0; e < E; ++e) if ((double)Lt[e] > M) M = (double)Lt[e];
      double den = 0.0;
      if (renorm) for (int j = 0; j < m; ++j) den += exp((double)Lt[ks[j].e] - M);
      else for (int e = 0; e < E; ++e) den += exp((double)Lt[e] - M);
      for (int j = 0; j < m; ++j)
        w[(int64_t)t * k + j] = exp((double)Lt[ks[j].e] - M) / den * (double)rsf;
    } else {
      double den = 0.0;
      for (int j = 0; j < m; ++j) den += 1.0 / (1.0 + exp(-(double)Lt[ks[j].e]));
      for (int j = 0; j < m; ++j) {
        double s = 1.0 / (1.0 + exp(-(double)Lt[ks[j].e]));
        w[(int64_t)t * k + j] = (renorm ? s / den : s) * (double)rsf;
      }
    }
  }
  free(ks);
  return 0;
}

/* Batch-union grouping: offsets [E+1], perm [offsets[E]] holds t*k+j sorted by (expert, t).
 * Slots with expert -1 (dropped by adaptive top-p) are left out. */
int orc_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* perm) {
  int32_t* fill = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
  for (int e = 0; e <= E; ++e) offsets[e] = 0;
  for (int64_t p = 0; p < (int64_t)T * k; ++p) {
    int e = idx[p];
    if (e == -1) continue;
    if (e < 0 || e >= E) { free(fill); return 1; }
    offsets[e + 1] += 1;
  }
  for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
  for (int e = 0; e < E; ++e) fill[e] = offsets[e];
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(int64_t)t * k + j];
      if (e >= 0) perm[fill[e]++] = t * k + j;
    }
  free(fill);
  return 0;
}

/* ---------------------------------------------- FP8 checkpoint conversion */

/* One float8 E4M3 ("fn": no infinities) code as fp32, from the format's
 * definition: sign bit 7, exponent bits 6-3 with bias 7, mantissa bits 2-0;
 * exponent 0 is subnormal (m * 2^-9), else (8 + m) * 2^(e - 10); exponent 15
 * with mantissa 7 is NaN. Every value is exact in fp32. */
float orc_fp8_e4m3_to_f32(uint8_t v) {
  const int s = v >> 7, e = (v >> 3) & 15, m = v & 7;
  if (e == 15 && m == 7) return NAN;
  const float mag = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
  return s ? -mag : mag;
}

/* The GLM page's FP8 -> int4 converter step, dequantizing side: an FP8 matrix
 * [N][K] with one fp32 inverse scale per 128 x 128 block ([ceil(N/128)][ceil(K/128)],
 * the DeepSeek-V3-style checkpoint layout) to fp32: w = decode(code) * scale, one
 * fp32 rounding. The codes are then quantized like any fp32 weight. */
void orc_dequant_fp8(const uint8_t* w8, const float* s_inv, int64_t N, int64_t K, float* out) {
  const int64_t KB = (K + 127) / 128;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      out[n * K + k] = orc_fp8_e4m3_to_f32(w8[n * K + k]) * s_inv[(n / 128) * KB + k / 128];
}

/* -------------------------------------------------------- expert arithmetic */

/* Canonical fp32 stage value of one weight row against one activation vector.
 * sw: the row's scales (g32: K/32 values; row: 1); sa likewise for the activation.
 * dots (optional): the exact per-group int32 dots (one entry when neither is g32). */
float orc_stage(const int8_t* qw, const float* sw, int K, int wg32, const int8_t* qa,
                const float* sa, int ag32, int32_t* dots) {
  if (!wg32 && !ag32) {
    int64_t acc = 0;
    for (int k = 0; k < K; ++k) acc += (int64_t)qw[k] * qa[k];
    if (dots) dots[0] = (int32_t)acc;
    float v = fmaf((float)(int32_t)acc, sa[0], 0.0f);
    return v * sw[0];
  }
  float acc = 0.0f;
  for (int g = 0; g < K / 32; ++g) {
    int32_t d = 0;
    for (int k = 32 * g; k < 32 * g + 32; ++k) d += (int32_t)qw[k] * (int32_t)qa[k];
    if (dots) dots[g] = d;
    float c = (wg32 && ag32) ? sw[g] * sa[g] : (wg32 ? sw[g] : sa[g]);
    acc = fmaf((float)d, c, acc);
  }
  if (wg32 && ag32) return acc;
  return acc * (wg32 ? sa[0] : sw[0]);
}

/* Exact dequantized dot in fp64. */
double orc_stage_f64(const int8_t* qw, const float* sw, int K, int wg32, const int8_t* qa,
                     const float* sa, int ag32) {
  double acc = 0.0;
  for (int k = 0; k < K; ++k) {
    double a = (double)qw[k] * (double)(wg32 ? sw[k / 32] : sw[0]);
    double b = (double)qa[k] * (double)(ag32 ? sa[k / 32] : sa[0]);
    acc += a * b;
  }
  return acc;
}

typedef struct {
  int32_t E, H, I, wbits, wg32;
  const int8_t* q_gu;   /* [E][2I][H] codes (int4 codes in [-7, 7]) */
  const float* s_gu;    /* g32: [E][2I][H/32]; row: [E][2I] */
  const int8_t* q_dn;   /* [E][H][I] */
  const float* s_dn;    /* g32: [E][H][I/32]; row: [E][H] */
} orc_experts;

/* One expert on one quantized token. Outputs: ye [H] fp64 (required);
 * gate/up [I] canonical stage values, qh [I], sh, ye32 [H] (each optional). */
int orc_expert_ffn(const orc_experts* ex, int e, const int8_t* qx, const float* sx, int ag32,
                   double* ye, float* gate, float* up, int8_t* qh, float* sh, float* ye32) {
  const int H = ex->H, I = ex->I;
  const int Gg = H / 32, Gd = I / 32;
  const int sg = ex->wg32 ? Gg : 1, sd = ex->wg32 ? Gd : 1;
  float hs[4096];
  if (Gd > 4096) return 1;
  float* g = (float*)malloc(sizeof(float) * (size_t)I);
  float* u = (float*)malloc(sizeof(float) * (size_t)I);
  float* h = (float*)malloc(sizeof(float) * (size_t)I);
  int8_t* q = (int8_t*)malloc((size_t)I);
  for (int i = 0; i < I; ++i) {
    int64_t rg = (int64_t)e * 2 * I + i, ru = rg + I;
    g[i] = orc_stage(ex->q_gu + rg * H, ex->s_gu + rg * sg, H, ex->wg32, qx, sx, ag32, NULL);
    u[i] = orc_stage(ex->q_gu + ru * H, ex->s_gu + ru * sg, H, ex->wg32, qx, sx, ag32, NULL);
    h[i] = orc_swiglu(g[i], u[i]);
  }
  orc_quantize_rows(h, 1, I, 127, ag32, q, hs);
  for (int n = 0; n < H; ++n) {
    int64_t rd = (int64_t)e * H + n;
    ye[n] = orc_stage_f64(ex->q_dn + rd * I, ex->s_dn + rd * sd, I, ex->wg32, q, hs, ag32);
    if (ye32) ye32[n] = orc_stage(ex->q_dn + rd * I, ex->s_dn + rd * sd, I, ex->wg32, q, hs, ag32, NULL);
  }
  if (gate) memcpy(gate, g, sizeof(float) * (size_t)I);
  if (up) memcpy(up, u, sizeof(float) * (size_t)I);
  if (qh) memcpy(qh, q, (size_t)I);
  if (sh) memcpy(sh, hs, sizeof(float) * (size_t)(ag32 ? Gd : 1));
  free(g); free(u); free(h); free(q);
  return 0;
}

/* ------------------------------------------------------------- whole layer */

typedef struct {
  int32_t T, score, top_k, renorm, act_g32;
  float rsf;
  const float* x;        /* [T][H] */
  const float* Wr;       /* [E][H] */
  const float* bias;     /* [E] or NULL */
  const orc_experts* ex;
  const orc_experts* sh; /* NULL = no shared expert */
  float top_p;           /* adaptive top-p in (0, 1); other values: off */
} orc_layer_in;

typedef struct {
  double* y;             /* [T][H] (required) */
  float* logits;         /* [T][E] */
  int32_t* idx;          /* [T][k] */
  double* w;             /* [T][k] */
  int8_t* qx;            /* [T][H] */
  float* sx;             /* [T][H/32] or [T] */
  float* gate;           /* [T*k][I], pair (t, j) at row t*k+j */
  float* up;             /* [T*k][I] */
  int8_t* qh;            /* [T*k][I] */
  float* sh;             /* [T*k][I/32] or [T*k] */
  double* ye;            /* [T*k][H] */
  float* ye32;           /* [T*k][H] */
  double* ysh;           /* [T][H] shared expert output */
  int32_t* offsets;      /* [E+1] (batch-union path) */
  int32_t* perm;         /* [T*k] (batch-union path) */
} orc_layer_out;

static int layer_common(const orc_layer_in* in, orc_layer_out* out, float** Lp, int32_t** idxp,
                        double** wp, int8_t** qxp, float** sxp) {
  const orc_experts* ex = in->ex;
  const int T = in->T, E = ex->E, H = ex->H, k = in->top_k;
  const int sxn = in->act_g32 ? H / 32 : 1;
  if (T < 0 || k <= 0 || k > E || H % 32 || ex->I % 32) return 1;
  if (in->sh && (in->sh->H != H || in->sh->I % 32)) return 1;
  float* L = out->logits ? out->logits : (float*)malloc(sizeof(float) * (size_t)T * E + 4);
  int32_t* idx = out->idx ? out->idx : (int32_t*)malloc(sizeof(int32_t) * (size_t)T * k + 4);
  double* w = out->w ? out->w : (double*)malloc(sizeof(double) * (size_t)T * k + 8);
  int8_t* qx = out->qx ? out->qx : (int8_t*)malloc((size_t)T * H + 1);
  float* sx = out->sx ? out->sx : (float*)malloc(sizeof(float) * (size_t)T * sxn + 4);
  orc_router_logits(in->x, in->Wr, T, E, H, L);
  if (orc_route(L, in->bias, T, E, in->score, k, in->renorm, in->rsf, in->top_p, idx, w)) return 1;
  orc_quantize_rows(in->x, T, H, 127, in->act_g32, qx, sx);
  *Lp = L; *idxp = idx; *wp = w; *qxp = qx; *sxp = sx;
  return 0;
}

static void layer_free(orc_layer_out* out, float* L, int32_t* idx, double* w, int8_t* qx, float* sx) {
  if (!out->logits) free(L);
  if (!out->idx) free(idx);
  if (!out->w) free(w);
  if (!out->qx) free(qx);
  if (!out->sx) free(sx);
}

static void pair_ffn(const orc_layer_in* in, orc_layer_out* out, int64_t row, int e,
                     const int8_t* qxt, const float* sxt, double* ye_row) {
  const orc_experts* ex = in->ex;
  const int I = ex->I, H = ex->H;
  const int shn = in->act_g32 ? I / 32 : 1;
  orc_expert_ffn(ex, e, qxt, sxt, in->act_g32, ye_row,
                 out->gate ? out->gate + row * I : NULL, out->up ? out->up + row * I : NULL,
                 out->qh ? out->qh + row * I : NULL, out->sh ? out->sh + row * shn : NULL,
                 out->ye32 ? out->ye32 + row * H : NULL);
}

static void shared_and_combine(const orc_layer_in* in, orc_layer_out* out, int t, const int8_t* qxt,
                               const float* sxt, const double* w, const double* const* ye_rows) {
  const int H = in->ex->H, k = in->top_k;
  double* yt = out->y + (int64_t)t * H;
  for (int n = 0; n < H; ++n) yt[n] = 0.0;
  for (int j = 0; j < k; ++j) {
    if (!ye_rows[j]) continue;           /* a slot dropped by adaptive top-p */
    for (int n = 0; n < H; ++n) yt[n] += w[(int64_t)t * k + j] * ye_rows[j][n];
  }
  if (in->sh) {
    double* ys = (double*)malloc(sizeof(double) * (size_t)H);
    orc_expert_ffn(in->sh, 0, qxt, sxt, in->act_g32, ys, NULL, NULL, NULL, NULL, NULL);
    for (int n = 0; n < H; ++n) yt[n] += ys[n];
    if (out->ysh) memcpy(out->ysh + (int64_t)t * H, ys, sizeof(double) * (size_t)H);
    free(ys);
  }
}

/* Per-token path: for each token, its k experts in selection order. */
int orc_layer_forward(const orc_layer_in* in, orc_layer_out* out, int nthreads) {
  float* L; int32_t* idx; double* w; int8_t* qx; float* sx;
  if (layer_common(in, out, &L, &idx, &w, &qx, &sx)) return 1;
  const int T = in->T, H = in->ex->H, k = in->top_k;
  const int sxn = in->act_g32 ? H / 32 : 1;
  (void)nthreads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
  for (int t = 0; t < T; ++t) {
    double* ye = out->ye ? NULL : (double*)malloc(sizeof(double) * (size_t)k * H);
    const double* rows[64];
    for (int j = 0; j < k && j < 64; ++j) {
      int64_t row = (int64_t)t * k + j;
      double* yr = out->ye ? out->ye + row * H : ye + (int64_t)j * H;
      rows[j] = NULL;
      if (idx[row] < 0) continue;        /* dropped by adaptive top-p */
      pair_ffn(in, out, row, idx[row], qx + (int64_t)t * H, sx + (int64_t)t * sxn, yr);
      rows[j] = yr;
    }
    shared_and_combine(in, out, t, qx + (int64_t)t * H, sx + (int64_t)t * sxn, w, rows);
    free(ye);
  }
  layer_free(out, L, idx, w, qx, sx);
  return k > 64 ? 1 : 0;
}

/* Batch-union path: group (token, slot) pairs by expert with the stable
 * counting sort, visit each unique expert once and apply it to every position
 * that routes to it; combine per token in slot order afterwards. */
int orc_layer_forward_union(const orc_layer_in* in, orc_layer_out* out) {
  float* L; int32_t* idx; double* w; int8_t* qx; float* sx;
  if (layer_common(in, out, &L, &idx, &w, &qx, &sx)) return 1;
  const int T = in->T, E = in->ex->E, H = in->ex->H, k = in->top_k;
  const int sxn = in->act_g32 ? H / 32 : 1;
  if (k > 64) return 1;
  int32_t* offsets = out->offsets ? out->offsets : (int32_t*)malloc(sizeof(int32_t) * ((size_t)E + 1));
  int32_t* perm = out->perm ? out->perm : (int32_t*)malloc(sizeof(int32_t) * (size_t)T * k + 4);
  orc_permute(idx, T, k, E, offsets, perm);
  double* ye = out->ye ? out->ye : (double*)malloc(sizeof(double) * (size_t)T * k * H + 8);
  for (int e = 0; e < E; ++e)
    for (int32_t p = offsets[e]; p < offsets[e + 1]; ++p) {
      int64_t row = perm[p];
      int t = (int)(row / k);
      pair_ffn(in, out, row, e, qx + (int64_t)t * H, sx + (int64_t)t * sxn, ye + row * H);
    }
  for (int t = 0; t < T; ++t) {
    const double* rows[64];
    for (int j = 0; j < k; ++j)
      rows[j] = idx[(int64_t)t * k + j] < 0 ? NULL : ye + ((int64_t)t * k + j) * H;
    shared_and_combine(in, out, t, qx + (int64_t)t * H, sx + (int64_t)t * sxn, w, rows);
  }
  if (!out->ye) free(ye);
  if (!out->offsets) free(offsets);
  if (!out->perm) free(perm);
  layer_free(out, L, idx, w, qx, sx);
  return 0;
}
