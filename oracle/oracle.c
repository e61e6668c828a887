/*
 * oracle.c — the CPU ORACLE of the batch-1 decode step.  TEST INFRASTRUCTURE ONLY:
 * nothing in the product links or calls it; the tests, the smoke check and the
 * CPU-baseline leg of the benchmark do.  It shares no code, header, table or constant
 * with the GPU engine.
 *
 * It is the plain definition of one decoder forward step, written out with loops in
 * the order the math states, with no blocking, fusion or reordering.  Compiled twice:
 * ORC_REAL=double (liboracle64.so, the parity reference) and ORC_REAL=float
 * (liboracle32.so, the fp32 decoder stack).  OpenMP only splits independent output rows
 * (matrix-vector rows, attention heads) across threads.
 *
 * What the pages fix and what is read into them.  The pages name the fused ops whose
 * math this is — RMSNorm + QKV projection ("rmsnorm_projx_wqkvia", Static Compilation
 * for LLM Inference §5.4; "RMSNormProjxWqkvia", TileRT code audit, fused-op list),
 * output projection ("UnProjO…"), expert select + up/gate + SiLU and expert down
 * (TileRT code audit, blog-vs-code table and MoE section), the batch-1 decode
 * attention ("FlashSparseMLA", batch == 1) — but print no formula.  The standard
 * Llama-style decoder math is taken: RMSNorm x*g/sqrt(mean(x^2)+eps), half-split RoPE
 * with theta_i = theta^(-2i/D), softmax(q.k/sqrt(D)) attention with q head h reading kv
 * head h / (Hq/Hkv), SwiGLU silu(Wg x)*(Wu x), residual adds, final RMSNorm and LM
 * head.  Storage: weights, gains, embedding and KV cache are bf16; the k and v of the
 * current token are rounded to bf16 when appended to the cache and read back from it;
 * every other value stays in `real`.
 *
 * FP8 weights (optional, the seven projection matrices of a GQA layer): E4M3 bytes with
 * one fp32 scale per 128 x 128 block, decoded from the format's definition and multiplied
 * by the block's scale; activations stay in `real`.
 *
 * FP4 experts (optional, the routed experts of a MoE layer): MXFP4 rows (OCP Microscaling,
 * E2M1 elements with one E8M0 scale per 32), decoded from the formats' definitions;
 * activations stay in `real`.
 *
 * Pins (tests/test_oracle_pins.py): bf16 rounding vs torch and vs the two neighbours;
 * E4M3 decoding of all 256 bytes vs torch and vs the format's closed values; the FP8
 * matrix-vector product vs numpy on the decoded, scaled matrix; E2M1 and E8M0 decoding vs
 * the formats' value tables, the nibble order on a hand-made row, the MXFP4 product vs
 * numpy, the FP4-expert MoE layer vs the bf16 one on the decoded weights;
 * RMSNorm unit RMS; matrix-vector vs numpy matmul; RoPE identity at pos 0, norm
 * preservation, relative-position property and the complex-rotation form; attention
 * brute force in pure Python, one position returns V, equal keys return the mean of V,
 * softmax rows sum to 1; SiLU special values; the decode step against closed forms
 * when Wo / Wdown are zero, at pos 0, and under hidden-unit / head permutations.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORC_REAL
#define ORC_REAL double
#endif
typedef ORC_REAL real;

/* ------------------------------------------------------------------ storage -------- */

/* bf16 word -> value: the word is the upper half of an IEEE binary32. */
static real bf16_val(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (real)f;
}

real orc_bf16_to_real(uint16_t h) { return bf16_val(h); }

/* value -> bf16 word, round to nearest, ties to even, directly from `real` (no
 * intermediate rounding): keep 8 significant bits of the binary significand. */
uint16_t orc_round_bf16(real v) {
  double x = (double)v;
  if (isnan(x)) return 0x7fc0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  int e;
  double m = frexp(fabs(x), &e);          /* |x| = m * 2^e, m in [0.5, 1)          */
  if (e < -125) {                          /* below binary32's normal range: the     */
    double q = ldexp(1.0, -133);           /* bf16 subnormal step is 2^-133          */
    double r = nearbyint(fabs(x) / q) * q;
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)((u >> 16) | (signbit(x) ? 0x8000 : 0));
  }
  double r = ldexp(nearbyint(ldexp(m, 8)), e - 8); /* 8 significant bits, RNE        */
  float f = (float)r;                      /* exact unless it overflows to inf       */
  uint32_t u;
  memcpy(&u, &f, 4);
  u |= signbit(x) ? 0x80000000u : 0u;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ pieces --------- */

/* RMSNorm: out = x * g / sqrt(mean(x^2) + eps). */
void orc_rmsnorm(int n, const real* x, const uint16_t* g, double eps, real* out) {
  real ss = 0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  real r = (real)(1.0 / sqrt((double)ss / n + eps));
  for (int i = 0; i < n; ++i) out[i] = x[i] * r * bf16_val(g[i]);
}

/* y = W x, W row-major [N][K] bf16. */
void orc_gemv(int N, int K, const uint16_t* W, const real* x, real* y) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint16_t* row = W + (size_t)n * K;
    real acc = 0;
    for (int k = 0; k < K; ++k) acc += bf16_val(row[k]) * x[k];
    y[n] = acc;
  }
}

/* FP8 E4M3 (the OCP 8-bit floating-point format with 4 exponent bits, bias 7, and 3
 * mantissa bits; no infinities, S.1111.111 is NaN) byte -> value.  Exponent field 0 holds
 * the subnormals m/8 * 2^-6; otherwise the value is (1 + m/8) * 2^(e - 7). */
real orc_e4m3_to_real(uint8_t b) {
  int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return (real)NAN;
  if (e == 0) v = ldexp((double)m / 8.0, -6);
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return (real)(sgn ? -v : v);
}

/* y = W x with W [N][K] stored as E4M3 bytes and block scales S[ceil(N/128)][ceil(K/128)]
 * (fp32): element W[n][k] stands for e4m3(W[n][k]) * S[n / 128][k / 128] — the block-scaled
 * FP8 weight layout (128 x 128 blocks) of DeepSeek-V3-style checkpoints, which the pages'
 * fused "RMSNorm + QKV + FP8 dequant" op consumes (TileRT code audit, fused-op list). */
void orc_gemv_fp8(int N, int K, const uint8_t* W, const float* S, const real* x, real* y) {
  int KB = (K + 127) / 128;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint8_t* row = W + (size_t)n * K;
    const float* srow = S + (size_t)(n / 128) * KB;
    real acc = 0;
    for (int k = 0; k < K; ++k) acc += orc_e4m3_to_real(row[k]) * (real)srow[k / 128] * x[k];
    y[n] = acc;
  }
}

/* FP4 E2M1 (the OCP Microscaling 4-bit float: sign, 2 exponent bits with bias 1, 1 mantissa
 * bit; no infinities, no NaN) code in the low 4 bits of c -> value.  Exponent field 0 holds
 * the subnormals m/2 (0 and 0.5); otherwise the value is (1 + m/2) * 2^(e - 1). */
real orc_e2m1_to_real(uint8_t c) {
  int sgn = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (real)(sgn ? -v : v);
}

/* E8M0 (the OCP Microscaling shared scale: an unsigned 8-bit exponent with bias 127, no
 * mantissa) -> 2^(s - 127); 255 is NaN. */
real orc_e8m0_to_real(uint8_t s) {
  if (s == 255) return (real)NAN;
  return (real)ldexp(1.0, (int)s - 127);
}

/* Bytes of one stored MXFP4 row of K elements: K/2 code bytes, K/32 scale bytes, padded to
 * a multiple of 16. */
int orc_mxfp4_pitch(int K) { return (K / 2 + K / 32 + 15) / 16 * 16; }

/* y = W x with W [N][K] stored as MXFP4 rows (OCP Microscaling MXFP4, block size 32) of
 * orc_mxfp4_pitch(K) bytes: element k of row n is the E2M1 code in the low nibble (k even)
 * or high nibble (k odd) of byte k / 2, times the E8M0 scale in byte K / 2 + k / 32.  The
 * pages quantise only the MoE experts to FP4 (Speed is intelligence talk, the MiMo
 * co-design passage) and name no layout; this is the OCP MXFP4 format. */
void orc_gemv_mxfp4(int N, int K, const uint8_t* W, const real* x, real* y) {
  const int pitch = orc_mxfp4_pitch(K);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint8_t* row = W + (size_t)n * pitch;
    real acc = 0;
    for (int k = 0; k < K; ++k) {
      const uint8_t code = (k & 1) ? (uint8_t)(row[k / 2] >> 4) : (uint8_t)(row[k / 2] & 15);
      acc += orc_e2m1_to_real(code) * orc_e8m0_to_real(row[K / 2 + k / 32]) * x[k];
    }
    y[n] = acc;
  }
}

/* Half-split rotary embedding of one head vector v[D] at position pos: the pair
 * (v[i], v[i + D/2]) is rotated by the angle pos * theta^(-2i/D). */
void orc_rope(int D, int pos, double theta, real* v) {
  int h = D / 2;
  for (int i = 0; i < h; ++i) {
    double ang = (double)pos * pow(theta, -2.0 * i / D);
    real c = (real)cos(ang), s = (real)sin(ang);
    real x0 = v[i], x1 = v[i + h];
    v[i] = x0 * c - x1 * s;
    v[i + h] = x0 * s + x1 * c;
  }
}

real orc_silu(real z) { return z / ((real)1 + (real)exp(-(double)z)); }

/* Decode attention of Hq query heads over P cached positions of Hkv kv heads.
 * Cache layout [Hkv][cap][D] bf16.  Query head h reads kv head h / (Hq / Hkv).
 * out[h*D + d] = sum_t p_t V[t][d],  p = softmax_t(q_h . K[t] / sqrt(D)).
 * probs (optional, [Hq][P]) receives p. */
void orc_attention(int Hq, int Hkv, int D, int P, int cap, const real* q,
                   const uint16_t* kc, const uint16_t* vc, real* out, real* probs) {
  int G = Hq / Hkv;
  real scale = (real)(1.0 / sqrt((double)D));
#pragma omp parallel for schedule(static)
  for (int h = 0; h < Hq; ++h) {
    int g = h / G;
    real* s = (real*)malloc(sizeof(real) * (size_t)(P > 0 ? P : 1));
    real m = -INFINITY;
    for (int t = 0; t < P; ++t) {
      const uint16_t* krow = kc + ((size_t)g * cap + t) * D;
      real acc = 0;
      for (int d = 0; d < D; ++d) acc += q[(size_t)h * D + d] * bf16_val(krow[d]);
      s[t] = acc * scale;
      if (s[t] > m) m = s[t];
    }
    real l = 0;
    for (int t = 0; t < P; ++t) {
      s[t] = (real)exp((double)(s[t] - m));
      l += s[t];
    }
    for (int t = 0; t < P; ++t) s[t] /= l;
    for (int d = 0; d < D; ++d) {
      real acc = 0;
      for (int t = 0; t < P; ++t) acc += s[t] * bf16_val(vc[((size_t)g * cap + t) * D + d]);
      out[(size_t)h * D + d] = acc;
    }
    if (probs)
      for (int t = 0; t < P; ++t) probs[(size_t)h * P + t] = s[t];
    free(s);
  }
}

int orc_argmax(int n, const real* v) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  return best;
}

/* ------------------------------------------------------------------ the stack ------ */

typedef struct {
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, kv_capacity;
  double rope_theta, norm_eps;
  int32_t weight_fp8;  /* 1: the seven projection matrices are E4M3 with block scales */
} orc_gqa_config;

typedef struct {
  const uint16_t *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *wgate, *wup, *wdown;
  uint16_t *k_cache, *v_cache; /* [Hkv][cap][D] bf16, written at pos */
  /* weight_fp8: the block scales of wq, wk, wv, wo, wgate, wup, wdown (whose pointers then
   * address E4M3 bytes) */
  const float *sq, *sk, *sv, *so, *sgate, *sup, *sdown;
} orc_gqa_layer;

/* A projection of the stack: bf16 weights, or E4M3 bytes with block scales. */
static void layer_gemv(const orc_gqa_config* c, int N, int K, const uint16_t* W, const float* S,
                       const real* x, real* y) {
  if (c->weight_fp8) orc_gemv_fp8(N, K, (const uint8_t*)W, S, x, y);
  else orc_gemv(N, K, W, x, y);
}

/* The attention block of a pre-norm GQA layer at position pos:
 *   xn = RMSNorm(x); q,k,v = Wq xn, Wk xn, Wv xn; RoPE(q, k at pos);
 *   cache[pos] = bf16(k), bf16(v); o = attention over positions [0, pos];
 *   h1 = x + Wo o. */
void orc_gqa_attn_block(const orc_gqa_config* c, const orc_gqa_layer* L, int pos, const real* x,
                        real* h1) {
  int d = c->hidden, Hq = c->n_q_heads, Hkv = c->n_kv_heads, D = c->head_dim;
  int cap = c->kv_capacity;
  real* xn = (real*)malloc(sizeof(real) * d);
  real* q = (real*)malloc(sizeof(real) * (size_t)Hq * D);
  real* k = (real*)malloc(sizeof(real) * (size_t)Hkv * D);
  real* v = (real*)malloc(sizeof(real) * (size_t)Hkv * D);
  real* o = (real*)malloc(sizeof(real) * (size_t)Hq * D);
  real* y = (real*)malloc(sizeof(real) * d);
  orc_rmsnorm(d, x, L->attn_norm, c->norm_eps, xn);
  layer_gemv(c, Hq * D, d, L->wq, L->sq, xn, q);
  layer_gemv(c, Hkv * D, d, L->wk, L->sk, xn, k);
  layer_gemv(c, Hkv * D, d, L->wv, L->sv, xn, v);
  for (int h = 0; h < Hq; ++h) orc_rope(D, pos, c->rope_theta, q + (size_t)h * D);
  for (int h = 0; h < Hkv; ++h) orc_rope(D, pos, c->rope_theta, k + (size_t)h * D);
  for (int h = 0; h < Hkv; ++h)
    for (int i = 0; i < D; ++i) {
      L->k_cache[((size_t)h * cap + pos) * D + i] = orc_round_bf16(k[(size_t)h * D + i]);
      L->v_cache[((size_t)h * cap + pos) * D + i] = orc_round_bf16(v[(size_t)h * D + i]);
    }
  orc_attention(Hq, Hkv, D, pos + 1, cap, q, L->k_cache, L->v_cache, o, NULL);
  layer_gemv(c, d, Hq * D, L->wo, L->so, o, y);
  for (int i = 0; i < d; ++i) h1[i] = x[i] + y[i];
  free(xn); free(q); free(k); free(v); free(o); free(y);
}

/* A SwiGLU MLP on an already-normalised input: y = Wd (silu(Wg hn) * (Wu hn)), F hidden
 * units.  Serves the dense MLP, every routed expert and the shared expert. */
void orc_swiglu_mlp(int d, int F, const uint16_t* wgate, const uint16_t* wup,
                    const uint16_t* wdown, const real* hn, real* y) {
  real* g = (real*)malloc(sizeof(real) * F);
  real* u = (real*)malloc(sizeof(real) * F);
  orc_gemv(F, d, wgate, hn, g);
  orc_gemv(F, d, wup, hn, u);
  for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
  orc_gemv(d, F, wdown, g, y);
  free(g);
  free(u);
}

/* SwiGLU MLP of one FP4 expert: gate and up rows [F] of d elements, down rows [d] of F
 * elements, all MXFP4 (orc_gemv_mxfp4). */
void orc_swiglu_mlp_mxfp4(int d, int F, const uint8_t* wgate, const uint8_t* wup,
                          const uint8_t* wdown, const real* hn, real* y) {
  real* g = (real*)malloc(sizeof(real) * F);
  real* u = (real*)malloc(sizeof(real) * F);
  orc_gemv_mxfp4(F, d, wgate, hn, g);
  orc_gemv_mxfp4(F, d, wup, hn, u);
  for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
  orc_gemv_mxfp4(d, F, wdown, g, y);
  free(g);
  free(u);
}

/* One pre-norm GQA decoder layer at position pos, residual x[d] updated in place:
 * h1 = attention block; x = h1 + SwiGLU(RMSNorm(h1)). */
void orc_gqa_layer_step(const orc_gqa_config* c, const orc_gqa_layer* L, int pos, real* x) {
  int d = c->hidden;
  real* h1 = (real*)malloc(sizeof(real) * d);
  real* hn = (real*)malloc(sizeof(real) * d);
  real* y = (real*)malloc(sizeof(real) * d);
  orc_gqa_attn_block(c, L, pos, x, h1);
  orc_rmsnorm(d, h1, L->ffn_norm, c->norm_eps, hn);
  if (c->weight_fp8) {
    int F = c->ffn;
    real* g = (real*)malloc(sizeof(real) * F);
    real* u = (real*)malloc(sizeof(real) * F);
    orc_gemv_fp8(F, d, (const uint8_t*)L->wgate, L->sgate, hn, g);
    orc_gemv_fp8(F, d, (const uint8_t*)L->wup, L->sup, hn, u);
    for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
    orc_gemv_fp8(d, F, (const uint8_t*)L->wdown, L->sdown, g, y);
    free(g);
    free(u);
  } else {
    orc_swiglu_mlp(d, c->ffn, L->wgate, L->wup, L->wdown, hn, y);
  }
  for (int i = 0; i < d; ++i) x[i] = h1[i] + y[i];
  free(h1); free(hn); free(y);
}

/* Layers only: x[d] in, x[d] out, hidden[l*d] (optional) after every layer. */
void orc_gqa_layers_step(const orc_gqa_config* c, const orc_gqa_layer* layers, int pos,
                         real* x, real* hidden) {
  for (int l = 0; l < c->n_layers; ++l) {
    orc_gqa_layer_step(c, &layers[l], pos, x);
    if (hidden) memcpy(hidden + (size_t)l * c->hidden, x, sizeof(real) * c->hidden);
  }
}

/* One batch-1 decode step of the whole stack: x = E[token]; the layers; logits =
 * W_lm RMSNorm(x).  hidden (optional) receives the residual after every layer. */
void orc_decode_step(const orc_gqa_config* c, const uint16_t* embed, const uint16_t* final_norm,
                     const uint16_t* lm_head, const orc_gqa_layer* layers, int token, int pos,
                     real* logits, real* hidden) {
  int d = c->hidden;
  real* x = (real*)malloc(sizeof(real) * d);
  real* xn = (real*)malloc(sizeof(real) * d);
  for (int i = 0; i < d; ++i) x[i] = bf16_val(embed[(size_t)token * d + i]);
  orc_gqa_layers_step(c, layers, pos, x, hidden);
  orc_rmsnorm(d, x, final_norm, c->norm_eps, xn);
  orc_gemv(c->vocab, d, lm_head, xn, logits);
  free(x);
  free(xn);
}

/* ------------------------------------------------------------------ MoE ------------ */

/* Router of a mixture-of-experts MLP (the pages name the fused op ExpertSelectUpGateSiLU,
 * TileRT code audit, MoE paragraph, but print no formula; read as DeepSeek-style
 * sigmoid routing): s_e = sigmoid(W_r[e] . hn) for e < E; the top_k experts by s, ties
 * to the lower index; w_i = s_i / sum of the selected s.  idx[top_k], w[top_k] in
 * descending score order; scores (optional) receives all E scores. */
void orc_router_topk(int E, int top_k, int d, const uint16_t* wr, const real* hn, int* idx,
                     real* w, real* scores) {
  real* s = (real*)malloc(sizeof(real) * E);
  orc_gemv(E, d, wr, hn, s);
  for (int e = 0; e < E; ++e) s[e] = (real)(1.0 / (1.0 + exp(-(double)s[e])));
  char* taken = (char*)calloc((size_t)E, 1);
  real tot = 0;
  for (int i = 0; i < top_k; ++i) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (best < 0 || s[e] > s[best])) best = e;
    taken[best] = 1;
    idx[i] = best;
    w[i] = s[best];
    tot += s[best];
  }
  for (int i = 0; i < top_k; ++i) w[i] /= tot;
  if (scores) memcpy(scores, s, sizeof(real) * E);
  free(taken);
  free(s);
}

/* ------------------------------------------------------------------ absorbed MLA ---- */

typedef struct {
  int32_t hidden, n_heads, q_lora, kv_lora, rope_dim, nope_dim, v_dim, kv_capacity;
  double rope_theta, norm_eps;
  /* sparse attention (0 = dense): index heads H_I, index dim D_I, positions kept K */
  int32_t index_heads, index_dim, index_topk;
} orc_mla_config;

typedef struct {
  const uint16_t *attn_norm; /* [d]                          */
  const uint16_t *w_dq;      /* [q_lora][d]                  */
  const uint16_t *q_norm;    /* [q_lora]                     */
  const uint16_t *w_uq;      /* [H * (nope + rope)][q_lora]  */
  const uint16_t *w_dkv;     /* [kv_lora + rope][d]          */
  const uint16_t *kv_norm;   /* [kv_lora]                    */
  const uint16_t *w_uk;      /* [H * nope][kv_lora]          */
  const uint16_t *w_uv;      /* [H * v][kv_lora]             */
  const uint16_t *w_o;       /* [d][H * v]                   */
  uint16_t *latent_cache;    /* [cap][kv_lora + rope] bf16   */
  const uint16_t *w_iq;      /* sparse: [H_I * D_I][q_lora]  (index queries)          */
  const uint16_t *w_ik;      /* sparse: [D_I + H_I][d]       (index key, head weights) */
  uint16_t *index_cache;     /* sparse: [cap][D_I] bf16                               */
} orc_mla_layer;

/* The sparse-attention indexer (the pages: 64 index heads choose the top-2048 KV positions
 * of a 160K context, TileRT code audit, sparse-index paragraph; weights named
 * self_attn.indexer.* come with the DeepSeek-V3.2 checkpoint; no formula is printed): read
 * as DeepSeek-V3.2's lightning indexer, with plain projections (no RoPE, no norm):
 *   k_I = W_ik[0:D_I] xn (this position's index key, appended to the index cache as bf16),
 *   w_I = W_ik[D_I:D_I+H_I] xn,  q_I = W_iq c_q (c_q after its RMSNorm),
 *   I[t] = sum_j (w_I[j] / sqrt(H_I)) * ReLU(q_I[j] . k_I[t] / sqrt(D_I))  for t in [0, pos];
 * the attention keeps the K positions of largest I (ties to the lower position; every
 * position when pos + 1 <= K).  sel[] receives them in increasing order; returns their count. */
static int cmp_score_desc(const void* a, const void* b) {
  const real* x = (const real*)a;
  const real* y = (const real*)b;
  if (x[0] > y[0]) return -1;
  if (x[0] < y[0]) return 1;
  return (x[1] < y[1]) ? -1 : (x[1] > y[1]);  /* lower position first */
}
static int cmp_int(const void* a, const void* b) {
  const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}
int orc_index_select(int P, int K, const real* score, int32_t* sel) {
  if (P <= K) {
    for (int t = 0; t < P; ++t) sel[t] = t;
    return P;
  }
  real* pairs = (real*)malloc(sizeof(real) * 2 * (size_t)P);
  for (int t = 0; t < P; ++t) {
    pairs[2 * t] = score[t];
    pairs[2 * t + 1] = (real)t;
  }
  qsort(pairs, (size_t)P, 2 * sizeof(real), cmp_score_desc);
  for (int i = 0; i < K; ++i) sel[i] = (int32_t)pairs[2 * i + 1];
  qsort(sel, (size_t)K, sizeof(int32_t), cmp_int);
  free(pairs);
  return K;
}

/* One absorbed multi-head latent attention layer (attention only) at position pos, residual
 * x[d] updated in place.  The pages name FlashSparseMLA (batch == 1) and TokenSpeed's
 * q-head folding (TileRT code audit) but print no formula; read as DeepSeek-V2 MLA with the
 * up-projections absorbed:
 *   xn = RMSNorm(x); c_q = RMSNorm(W_dq xn; q_norm); [q_nope_h, q_pe_h] = (W_uq c_q)_h;
 *   [c_kv, k_pe] = W_dkv xn; c_kv = RMSNorm(c_kv; kv_norm); RoPE(q_pe_h), RoPE(k_pe) at pos;
 *   cache[pos] = bf16([c_kv, k_pe]);
 *   q_lat_h = W_uk,h^T q_nope_h;  s_h[t] = (q_lat_h . c_kv[t] + q_pe_h . k_pe[t]) / sqrt(nope+rope);
 *   o_lat_h = sum_t softmax(s_h)[t] c_kv[t];  o_h = W_uv,h o_lat_h;  x = x + W_o [o_h]. */
/* The layer with the attention over a chosen set of positions.  Sparse configs compute the
 * index scores into iscore_out ([pos + 1], may be NULL) and the chosen positions into
 * sel_out ([K], may be NULL); sel_in (n_sel_in positions, increasing) overrides the choice
 * when not NULL.  Dense configs (index_topk 0) attend to every position in [0, pos]. */
void orc_mla_layer_step_ex(const orc_mla_config* c, const orc_mla_layer* L, int pos, real* x,
                           const int32_t* sel_in, int n_sel_in, real* iscore_out,
                           int32_t* sel_out);

void orc_mla_layer_step(const orc_mla_config* c, const orc_mla_layer* L, int pos, real* x) {
  orc_mla_layer_step_ex(c, L, pos, x, NULL, 0, NULL, NULL);
}

void orc_mla_layer_step_ex(const orc_mla_config* c, const orc_mla_layer* L, int pos, real* x,
                           const int32_t* sel_in, int n_sel_in, real* iscore_out,
                           int32_t* sel_out) {
  const int d = c->hidden, H = c->n_heads, QL = c->q_lora, KL = c->kv_lora, R = c->rope_dim;
  const int NP = c->nope_dim, VD = c->v_dim, QH = NP + R, C = KL + R, cap = c->kv_capacity;
  real* xn = (real*)malloc(sizeof(real) * d);
  real* cq = (real*)malloc(sizeof(real) * QL);
  real* cqn = (real*)malloc(sizeof(real) * QL);
  real* q = (real*)malloc(sizeof(real) * (size_t)H * QH);
  real* kv = (real*)malloc(sizeof(real) * C);
  real* ckv = (real*)malloc(sizeof(real) * KL);
  real* qlat = (real*)malloc(sizeof(real) * (size_t)H * KL);
  real* olat = (real*)malloc(sizeof(real) * (size_t)H * KL);
  real* o = (real*)malloc(sizeof(real) * (size_t)H * VD);
  real* y = (real*)malloc(sizeof(real) * d);
  const int P = pos + 1;
  real* sc = (real*)malloc(sizeof(real) * P);

  orc_rmsnorm(d, x, L->attn_norm, c->norm_eps, xn);
  orc_gemv(QL, d, L->w_dq, xn, cq);
  orc_rmsnorm(QL, cq, L->q_norm, c->norm_eps, cqn);
  orc_gemv(H * QH, QL, L->w_uq, cqn, q);
  orc_gemv(C, d, L->w_dkv, xn, kv);
  orc_rmsnorm(KL, kv, L->kv_norm, c->norm_eps, ckv);
  orc_rope(R, pos, c->rope_theta, kv + KL);
  for (int h = 0; h < H; ++h) orc_rope(R, pos, c->rope_theta, q + (size_t)h * QH + NP);
  uint16_t* row = L->latent_cache + (size_t)pos * C;
  for (int i = 0; i < KL; ++i) row[i] = orc_round_bf16(ckv[i]);
  for (int i = 0; i < R; ++i) row[KL + i] = orc_round_bf16(kv[KL + i]);

  /* q_lat_h[j] = sum_n W_uk[h*NP + n][j] * q_nope_h[n] */
  for (int h = 0; h < H; ++h)
    for (int j = 0; j < KL; ++j) {
      real acc = 0;
      for (int n = 0; n < NP; ++n)
        acc += bf16_val(L->w_uk[((size_t)h * NP + n) * KL + j]) * q[(size_t)h * QH + n];
      qlat[(size_t)h * KL + j] = acc;
    }
  /* the positions attended: all of [0, pos], or the indexer's choice */
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
  int NS = P;
  for (int t = 0; t < P; ++t) sel[t] = t;
  if (c->index_topk > 0) {
    const int HI = c->index_heads, DI = c->index_dim;
    real* ki = (real*)malloc(sizeof(real) * (size_t)(DI + HI));
    real* qi = (real*)malloc(sizeof(real) * (size_t)HI * DI);
    real* isc = (real*)malloc(sizeof(real) * (size_t)P);
    orc_gemv(DI + HI, d, L->w_ik, xn, ki);
    orc_gemv(HI * DI, QL, L->w_iq, cqn, qi);
    uint16_t* irow = L->index_cache + (size_t)pos * DI;
    for (int i = 0; i < DI; ++i) irow[i] = orc_round_bf16(ki[i]);
    const double sq = 1.0 / sqrt((double)DI), sw = 1.0 / sqrt((double)HI);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < P; ++t) {
      const uint16_t* kt = L->index_cache + (size_t)t * DI;
      real acc = 0;
      for (int j = 0; j < HI; ++j) {
        real dot = 0;
        for (int i = 0; i < DI; ++i) dot += qi[(size_t)j * DI + i] * bf16_val(kt[i]);
        dot *= (real)sq;
        if (dot > 0) acc += ki[DI + j] * (real)sw * dot;
      }
      isc[t] = acc;
    }
    int32_t* mine = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    const int nm = orc_index_select(P, c->index_topk, isc, mine);
    if (sel_out) memcpy(sel_out, mine, sizeof(int32_t) * (size_t)nm);
    if (iscore_out) memcpy(iscore_out, isc, sizeof(real) * (size_t)P);
    if (sel_in) {
      NS = n_sel_in;
      memcpy(sel, sel_in, sizeof(int32_t) * (size_t)n_sel_in);
    } else {
      NS = nm;
      memcpy(sel, mine, sizeof(int32_t) * (size_t)nm);
    }
    free(ki); free(qi); free(isc); free(mine);
  }

  const real scale = (real)(1.0 / sqrt((double)QH));
  for (int h = 0; h < H; ++h) {
    real m = -INFINITY;
    for (int u = 0; u < NS; ++u) {
      const int t = sel[u];
      const uint16_t* ct = L->latent_cache + (size_t)t * C;
      real a = 0;
      for (int j = 0; j < KL; ++j) a += qlat[(size_t)h * KL + j] * bf16_val(ct[j]);
      for (int j = 0; j < R; ++j) a += q[(size_t)h * QH + NP + j] * bf16_val(ct[KL + j]);
      sc[u] = a * scale;
      if (sc[u] > m) m = sc[u];
    }
    real l = 0;
    for (int u = 0; u < NS; ++u) {
      sc[u] = (real)exp((double)(sc[u] - m));
      l += sc[u];
    }
    for (int j = 0; j < KL; ++j) {
      real acc = 0;
      for (int u = 0; u < NS; ++u)
        acc += sc[u] / l * bf16_val(L->latent_cache[(size_t)sel[u] * C + j]);
      olat[(size_t)h * KL + j] = acc;
    }
  }
  free(sel);
  /* o_h = W_uv,h o_lat_h */
  for (int h = 0; h < H; ++h)
    orc_gemv(VD, KL, L->w_uv + (size_t)h * VD * KL, olat + (size_t)h * KL, o + (size_t)h * VD);
  orc_gemv(d, H * VD, L->w_o, o, y);
  for (int i = 0; i < d; ++i) x[i] += y[i];
  free(xn); free(cq); free(cqn); free(q); free(kv); free(ckv); free(qlat); free(olat);
  free(o); free(y); free(sc);
}

int orc_real_bytes(void) { return (int)sizeof(real); }
