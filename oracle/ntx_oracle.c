/*
 * ntx_oracle.c -- plain, slow, obviously-correct CPU oracle for the batch-1
 * decode hot path of a layer-streaming Llama inference engine over GGUF
 * block-quantized weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no source,
 * header, table or helper with the CUDA path (quantized_weight_gemv_dequant_b200/csrc)
 * or with the input generator (synthgen/); every definition below is written
 * out from the method's statement.
 *
 * Precision: every quantity is computed in IEEE double, sums run in index
 * order, transcendentals come from the host libm in double.  Only the two
 * places where the method itself stores a narrower type round to it:
 * the fp16 KV cache (round to nearest even on store) and nothing else.
 * Compiled -O2 -ffp-contract=off, no fast-math.
 *
 * Sources (page title -- section):
 *  [P1] "NTransformer" -- 主な機能 (features): GGUF formats Q4_0/Q8_0/Q6_K;
 *       Llama architecture: RoPE, GQA, SwiGLU, RMSNorm, KV cache.
 *  [P1a] "NTransformer" -- アーキテクチャ概要 (architecture): CUDA kernels GEMV,
 *       RMSNorm, RoPE, SwiGLU, softmax.
 *  [P2] "Show HN: NVMe経由でCPUをバイパスして単一のRTX 3090上で動作するLlama 3.1 70B"
 *       -- 量子化フォーマット対応表 (format table): Q4_0 4.5 bit/weight in blocks
 *       of 32, Q8_0 8.5 bit/weight in blocks of 32, Q6_K "6.6" bit/weight in
 *       blocks of 256.
 *  [P3] "RTX 3090 1枚でLlama 70B" -- レイヤースキップ機構 (layer skip): each
 *       layer's output is compared with its input by cosine similarity and
 *       near-identical layers are skipped (threshold 0.98).
 * The pages give no bit layout, formula or constant beyond the above; the
 * readings taken where they are silent are:
 *  - block layouts are GGUF's (Q8_0: fp16 d, int8 q[32]; Q4_0: fp16 d, 16
 *    bytes, element j in the low nibble of byte j, element j+16 in the high
 *    nibble; Q6_K: ql[128], qh[64], int8 scales[16], fp16 d);
 *  - RMSNorm y = w x / sqrt(mean(x^2) + eps);
 *  - RoPE rotates adjacent pairs (2i, 2i+1) by pos * theta^(-2i/D);
 *  - attention is causal over positions 0..pos with the current token's k, v
 *    read back from the fp16 cache; query head h uses KV head h / (Hq/Hkv);
 *  - SwiGLU silu(g) u, silu(z) = z / (1 + e^-z);
 *  - the layer is the pre-norm Llama block; the model is embed (fp16 row),
 *    layers, final RMSNorm, output head, greedy argmax (ties -> lowest id);
 *  - cosine c = <h_in, h_out> / (|h_in| |h_out|), layer skipped if c >= tau.
 * The same format table lists Q4_K_M (4.5 bit/weight, blocks of 256, "mixed"),
 * Q5_K (5.5 bit/weight, blocks of 256) and F16/F32 (16/32 bit/weight, blocks
 * of 1).  Readings (GGUF's layouts, consistent with those sizes):
 *  - Q4_K super-block, 144 B: fp16 d, fp16 dmin, 12 bytes of packed 6-bit
 *    sub-block scales sc[8] and mins m[8], 128 bytes of 4-bit codes;
 *    element 64c + l (c < 4, l < 32) is the low nibble of qs[32c + l] and
 *    element 64c + 32 + l its high nibble; w = d sc[n/32] q - dmin m[n/32];
 *  - Q5_K super-block, 176 B: the same d, dmin and scales, then qh[32] and
 *    qs[128]; the fifth bit of element 64c + l is bit 2c of qh[l], of element
 *    64c + 32 + l bit 2c + 1; q in 0..31, same formula;
 *  - "M" (mixed) means some matrices of the model use another block type; the
 *    oracle's layer takes one type per matrix;
 *  - F16: IEEE binary16 per weight; F32: IEEE binary32 per weight.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* GGUF type ids */
#define ORC_F32 0
#define ORC_F16 1
#define ORC_Q4_0 2
#define ORC_Q8_0 8
#define ORC_Q4_K 12
#define ORC_Q5_K 13
#define ORC_Q6_K 14

/* ------------------------------------------------------------ binary16 */
/* IEEE binary16 -> double (exact). */
double orc_half(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);                    /* subnormal or zero */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(1024 + m), e - 25);                /* (1 + m/1024) 2^(e-15) */
  return sign ? -v : v;
}

/* double -> IEEE binary16, round to nearest, ties to even. */
uint16_t orc_to_half(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isnan(v)) return 0x7E00;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);          /* a = f 2^e2, f in [0.5, 1)  ->  a in [2^(e2-1), 2^e2) */
  int e = e2 - 1;         /* a = (1.x) 2^e */
  if (e < -14) {          /* subnormal range: units of 2^-24 */
    double q = nearbyint(ldexp(a, 24)); /* default rounding mode: to nearest even */
    if (q >= 1024.0) return (uint16_t)(sign | 0x0400); /* rounded up to the smallest normal */
    return (uint16_t)(sign | (uint16_t)q);
  }
  double q = nearbyint(ldexp(a, 10 - e)); /* significand in units of 2^(e-10), in [1024, 2048] */
  if (q == 2048.0) { q = 1024.0; e += 1; }
  if (e > 15) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)q - 1024));
}

/* ------------------------------------------------------------ dequant */
int orc_block_elems(int qtype) {
  switch (qtype) {
    case ORC_F32: case ORC_F16: return 1;
    case ORC_Q4_0: case ORC_Q8_0: return 32;
    case ORC_Q4_K: case ORC_Q5_K: case ORC_Q6_K: return 256;
    default: return 0;
  }
}
int orc_block_bytes(int qtype) {
  switch (qtype) {
    case ORC_F32: return 4;
    case ORC_F16: return 2;
    case ORC_Q4_0: return 18;
    case ORC_Q8_0: return 34;
    case ORC_Q4_K: return 144;
    case ORC_Q5_K: return 176;
    case ORC_Q6_K: return 210;
    default: return 0;
  }
}

static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Q8_0 block (34 B): d = fp16 at bytes 0-1, q_i = int8 at byte 2+i;  w_i = d q_i. */
static void dq_q8_0(const uint8_t* blk, double* w) {
  double d = orc_half(rd16(blk));
  for (int i = 0; i < 32; ++i) w[i] = d * (double)(int8_t)blk[2 + i];
}

/* Q4_0 block (18 B): d = fp16 at bytes 0-1; byte 2+j holds q_j (low nibble)
 * and q_(j+16) (high nibble);  w_i = d (q_i - 8). */
static void dq_q4_0(const uint8_t* blk, double* w) {
  double d = orc_half(rd16(blk));
  for (int j = 0; j < 16; ++j) {
    int lo = blk[2 + j] & 0x0F, hi = blk[2 + j] >> 4;
    w[j] = d * (double)(lo - 8);
    w[j + 16] = d * (double)(hi - 8);
  }
}

/* Q6_K super-block (210 B): ql[128] at 0, qh[64] at 128, int8 scales[16] at
 * 192, fp16 d at 208.  Element n: h = n/128, r = n%128, g = r/32, l = r%32;
 * low 4 bits from ql[64h + 32(g%2) + l] (low nibble if g < 2, else high),
 * high 2 bits = (qh[32h + l] >> 2g) & 3;  w_n = d scales[n/16] (q_n - 32). */
static void dq_q6_k(const uint8_t* blk, double* w) {
  const uint8_t* ql = blk;
  const uint8_t* qh = blk + 128;
  const int8_t* sc = (const int8_t*)(blk + 192);
  double d = orc_half(rd16(blk + 208));
  for (int n = 0; n < 256; ++n) {
    int h = n / 128, r = n % 128, g = r / 32, l = r % 32;
    int byte = ql[64 * h + 32 * (g % 2) + l];
    int low = (g < 2) ? (byte & 0x0F) : (byte >> 4);
    int high = (qh[32 * h + l] >> (2 * g)) & 3;
    int q = low | (high << 4);
    w[n] = d * (double)sc[n / 16] * (double)(q - 32);
  }
}

/* The 6-bit scale and min of sub-block j (0..7) of a Q4_K / Q5_K super-block
 * from its 12 packed bytes p: sub-blocks 0-3 keep their scale in the low six
 * bits of p[j] and their min in the low six bits of p[j + 4]; sub-blocks 4-7
 * keep the low four bits of the scale in the low nibble of p[j + 4] and of the
 * min in its high nibble, and the top two bits of each in the top two bits of
 * p[j - 4] (scale) and p[j] (min). */
static void k_scale_min(const uint8_t* p, int j, int* sc, int* m) {
  if (j < 4) {
    *sc = p[j] & 63;
    *m = p[j + 4] & 63;
  } else {
    *sc = (p[j + 4] & 0x0F) | ((p[j - 4] >> 6) << 4);
    *m = (p[j + 4] >> 4) | ((p[j] >> 6) << 4);
  }
}

/* Q4_K super-block (144 B): d at 0, dmin at 2, scales at 4..15, qs at 16..143.
 * Element n = 64c + 32h + l takes nibble h of qs[32c + l];
 * w_n = d sc_j q_n - dmin m_j with j = n / 32. */
static void dq_q4_k(const uint8_t* blk, double* w) {
  double d = orc_half(rd16(blk)), dmin = orc_half(rd16(blk + 2));
  const uint8_t* qs = blk + 16;
  for (int n = 0; n < 256; ++n) {
    int c = n / 64, h = (n % 64) / 32, l = n % 32;
    int q = (qs[32 * c + l] >> (4 * h)) & 0x0F;
    int sc, m;
    k_scale_min(blk + 4, n / 32, &sc, &m);
    w[n] = d * (double)sc * (double)q - dmin * (double)m;
  }
}

/* Q5_K super-block (176 B): d at 0, dmin at 2, scales at 4..15, qh at
 * 16..47, qs at 48..175.  Element n = 64c + 32h + l: low four bits from
 * nibble h of qs[32c + l], fifth bit = bit (2c + h) of qh[l];
 * w_n = d sc_j q_n - dmin m_j with j = n / 32. */
static void dq_q5_k(const uint8_t* blk, double* w) {
  double d = orc_half(rd16(blk)), dmin = orc_half(rd16(blk + 2));
  const uint8_t* qh = blk + 16;
  const uint8_t* qs = blk + 48;
  for (int n = 0; n < 256; ++n) {
    int c = n / 64, h = (n % 64) / 32, l = n % 32;
    int q = ((qs[32 * c + l] >> (4 * h)) & 0x0F) | (((qh[l] >> (2 * c + h)) & 1) << 4);
    int sc, m;
    k_scale_min(blk + 4, n / 32, &sc, &m);
    w[n] = d * (double)sc * (double)q - dmin * (double)m;
  }
}

/* F16: one IEEE binary16 per weight; F32: one IEEE binary32 per weight. */
static void dq_f16(const uint8_t* blk, double* w) { w[0] = orc_half(rd16(blk)); }
static void dq_f32(const uint8_t* blk, double* w) {
  float f;
  memcpy(&f, blk, 4);
  w[0] = (double)f;
}

static void dq_block(int qtype, const uint8_t* blk, double* w) {
  switch (qtype) {
    case ORC_Q8_0: dq_q8_0(blk, w); break;
    case ORC_Q4_0: dq_q4_0(blk, w); break;
    case ORC_Q4_K: dq_q4_k(blk, w); break;
    case ORC_Q5_K: dq_q5_k(blk, w); break;
    case ORC_F16: dq_f16(blk, w); break;
    case ORC_F32: dq_f32(blk, w); break;
    default: dq_q6_k(blk, w); break;
  }
}

/* n values (n a multiple of the block size) from consecutive blocks. */
int orc_dequant(int qtype, const uint8_t* blocks, int64_t n, double* out) {
  int be = orc_block_elems(qtype), bb = orc_block_bytes(qtype);
  if (!be || n % be) return -1;
  for (int64_t b = 0; b < n / be; ++b) dq_block(qtype, blocks + b * bb, out + b * be);
  return 0;
}

/* ------------------------------------------------------------ GEMV */
/* y_i = sum_j w_ij x_j and b_i = sum_j |w_ij x_j|, j ascending, for rows of a
 * row-major M x K matrix of blocks.  Rows are independent; threads split rows
 * only, so the result does not depend on the thread count. */
typedef struct {
  int qtype;
  const uint8_t* W;
  int64_t K, r0, r1;
  const double* x;
  double *y, *b;
} gemv_job;

static void* gemv_rows(void* p) {
  gemv_job* j = (gemv_job*)p;
  int be = orc_block_elems(j->qtype), bb = orc_block_bytes(j->qtype);
  int64_t nb = j->K / be;
  double w[256];
  for (int64_t i = j->r0; i < j->r1; ++i) {
    double acc = 0.0, absacc = 0.0;
    for (int64_t blk = 0; blk < nb; ++blk) {
      dq_block(j->qtype, j->W + (i * nb + blk) * bb, w);
      for (int t = 0; t < be; ++t) {
        double p = w[t] * j->x[blk * be + t];
        acc += p;
        absacc += fabs(p);
      }
    }
    j->y[i] = acc;
    if (j->b) j->b[i] = absacc;
  }
  return NULL;
}

int orc_gemv(int qtype, const uint8_t* W, int64_t M, int64_t K, const double* x, double* y, double* b, int nthreads) {
  int be = orc_block_elems(qtype);
  if (!be || K % be || M < 0) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 128) nthreads = 128;
  if (M < nthreads) nthreads = M > 0 ? (int)M : 1;
  gemv_job jobs[128];
  pthread_t th[128];
  int ok[128];
  for (int t = 0; t < nthreads; ++t) {
    gemv_job g = {qtype, W, K, M * t / nthreads, M * (t + 1) / nthreads, x, y, b};
    jobs[t] = g;
    ok[t] = nthreads > 1 && pthread_create(&th[t], NULL, gemv_rows, &jobs[t]) == 0;
    if (!ok[t]) gemv_rows(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (ok[t]) pthread_join(th[t], NULL);
  return 0;
}

/* ------------------------------------------------------------ small ops */
/* RMSNorm: y_i = w_i x_i / sqrt(mean_j x_j^2 + eps). */
void orc_rmsnorm(const double* x, const double* w, int64_t n, double eps, double* y) {
  double ss = 0.0;
  for (int64_t i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int64_t i = 0; i < n; ++i) y[i] = w[i] * (x[i] * inv);
}

/* RoPE on n_heads consecutive heads of head_dim values, in place: the pair
 * (v[2i], v[2i+1]) of every head turns by angle pos * theta^(-2i/head_dim). */
void orc_rope(double* v, int n_heads, int head_dim, int pos, double theta) {
  for (int h = 0; h < n_heads; ++h)
    for (int i = 0; i < head_dim / 2; ++i) {
      double inv_freq = pow(theta, -2.0 * (double)i / (double)head_dim);
      double ang = (double)pos * inv_freq;
      double c = cos(ang), s = sin(ang);
      double* p = v + (int64_t)h * head_dim + 2 * i;
      double a = p[0], b = p[1];
      p[0] = a * c - b * s;
      p[1] = a * s + b * c;
    }
}

/* GQA decode attention.  q: n_q_heads x D.  Caches: fp16, [n_kv_heads][max_ctx][D].
 * out_h = sum_p softmax_p(q_h . k_p / sqrt(D)) v_p over p = 0 .. n_ctx-1, where
 * query head h reads KV head h / (n_q_heads / n_kv_heads).  bound (nullable)
 * receives sum_p p_p |v_p| per output element, the scale of its rounding error. */
int orc_attention(const double* q, const uint16_t* kc, const uint16_t* vc, int n_q_heads, int n_kv_heads, int D,
                  int n_ctx, int max_ctx, double* out, double* bound) {
  if (n_kv_heads <= 0 || n_q_heads % n_kv_heads || n_ctx < 1 || n_ctx > max_ctx) return -1;
  int group = n_q_heads / n_kv_heads;
  double* s = (double*)malloc(sizeof(double) * (size_t)n_ctx);
  if (!s) return -1;
  for (int h = 0; h < n_q_heads; ++h) {
    int kvh = h / group;
    const double* qh = q + (int64_t)h * D;
    double smax = -INFINITY;
    for (int p = 0; p < n_ctx; ++p) {
      const uint16_t* kp = kc + ((int64_t)kvh * max_ctx + p) * D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qh[d] * orc_half(kp[d]);
      s[p] = dot / sqrt((double)D);
      if (s[p] > smax) smax = s[p];
    }
    double sum = 0.0;
    for (int p = 0; p < n_ctx; ++p) { s[p] = exp(s[p] - smax); sum += s[p]; }
    for (int d = 0; d < D; ++d) {
      double o = 0.0, ob = 0.0;
      for (int p = 0; p < n_ctx; ++p) {
        double vv = orc_half(vc[((int64_t)kvh * max_ctx + p) * D + d]);
        o += (s[p] / sum) * vv;
        ob += (s[p] / sum) * fabs(vv);
      }
      out[(int64_t)h * D + d] = o;
      if (bound) bound[(int64_t)h * D + d] = ob;
    }
  }
  free(s);
  return 0;
}

/* SwiGLU: out_i = silu(g_i) u_i, silu(z) = z / (1 + exp(-z)). */
void orc_swiglu(const double* g, const double* u, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (g[i] / (1.0 + exp(-g[i]))) * u[i];
}

/* Cosine similarity <a,b> / (|a| |b|). */
double orc_cosine(const double* a, const double* b, int64_t n) {
  double ab = 0.0, aa = 0.0, bb = 0.0;
  for (int64_t i = 0; i < n; ++i) { ab += a[i] * b[i]; aa += a[i] * a[i]; bb += b[i] * b[i]; }
  return ab / (sqrt(aa) * sqrt(bb));
}

/* Greedy token: index of the largest value, lowest index on ties. */
int64_t orc_argmax(const double* v, int64_t n) {
  int64_t best = 0;
  for (int64_t i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  return best;
}

/* ------------------------------------------------------------ layer */
typedef struct {
  int32_t hidden, n_heads, n_kv_heads, head_dim, ffn, vocab, n_layers;
  double eps, theta;
  int32_t max_ctx;
} orc_config;

typedef struct {
  int32_t qt[7];                                   /* block type of wq, wk, wv, wo, wg, wu, wd */
  const uint8_t *wq, *wk, *wv, *wo, *wg, *wu, *wd; /* row-major out x in block matrices */
  const float *attn_norm, *ffn_norm;               /* hidden fp32 each */
} orc_layer_weights;

static double* dalloc(int64_t n) { return (double*)calloc((size_t)(n > 0 ? n : 1), sizeof(double)); }

/* One pre-norm Llama block for one token at position pos:
 *   n1 = RMSNorm(h) w_attn;  q = Wq n1, k = Wk n1, v = Wv n1;  RoPE(q), RoPE(k);
 *   k, v -> fp16 cache row pos;  a = Attention(q, cache[0..pos]);
 *   h1 = h + Wo a;  n2 = RMSNorm(h1) w_ffn;  h2 = h1 + Wd (silu(Wg n2) (Wu n2)).
 * h_out may alias h_in.  cos_out (nullable) receives cosine(h_in, h_out). */
int orc_layer(const orc_config* c, const orc_layer_weights* L, uint16_t* k_cache, uint16_t* v_cache,
              const double* h_in, int pos, double* h_out, double* cos_out, int nthreads) {
  const int64_t H = c->hidden, D = c->head_dim, F = c->ffn;
  const int64_t Q = (int64_t)c->n_heads * D, KV = (int64_t)c->n_kv_heads * D;
  if (pos < 0 || pos >= c->max_ctx) return -1;
  double *h = dalloc(H), *wn = dalloc(H), *n1 = dalloc(H), *q = dalloc(Q), *k = dalloc(KV), *v = dalloc(KV);
  double *a = dalloc(Q), *t = dalloc(H), *h1 = dalloc(H), *n2 = dalloc(H), *g = dalloc(F), *u = dalloc(F);
  double *s = dalloc(F), *h2 = dalloc(H);
  int rc = -1;
  if (!h || !wn || !n1 || !q || !k || !v || !a || !t || !h1 || !n2 || !g || !u || !s || !h2) goto done;
  memcpy(h, h_in, sizeof(double) * (size_t)H);

  for (int64_t i = 0; i < H; ++i) wn[i] = (double)L->attn_norm[i];
  orc_rmsnorm(h, wn, H, c->eps, n1);
  if (orc_gemv(L->qt[0], L->wq, Q, H, n1, q, NULL, nthreads)) goto done;
  if (orc_gemv(L->qt[1], L->wk, KV, H, n1, k, NULL, nthreads)) goto done;
  if (orc_gemv(L->qt[2], L->wv, KV, H, n1, v, NULL, nthreads)) goto done;
  orc_rope(q, c->n_heads, (int)D, pos, c->theta);
  orc_rope(k, c->n_kv_heads, (int)D, pos, c->theta);
  for (int kh = 0; kh < c->n_kv_heads; ++kh)
    for (int64_t d = 0; d < D; ++d) {
      k_cache[((int64_t)kh * c->max_ctx + pos) * D + d] = orc_to_half(k[kh * D + d]);
      v_cache[((int64_t)kh * c->max_ctx + pos) * D + d] = orc_to_half(v[kh * D + d]);
    }
  if (orc_attention(q, k_cache, v_cache, c->n_heads, c->n_kv_heads, (int)D, pos + 1, c->max_ctx, a, NULL)) goto done;
  if (orc_gemv(L->qt[3], L->wo, H, Q, a, t, NULL, nthreads)) goto done;
  for (int64_t i = 0; i < H; ++i) h1[i] = h[i] + t[i];

  for (int64_t i = 0; i < H; ++i) wn[i] = (double)L->ffn_norm[i];
  orc_rmsnorm(h1, wn, H, c->eps, n2);
  if (orc_gemv(L->qt[4], L->wg, F, H, n2, g, NULL, nthreads)) goto done;
  if (orc_gemv(L->qt[5], L->wu, F, H, n2, u, NULL, nthreads)) goto done;
  orc_swiglu(g, u, F, s);
  if (orc_gemv(L->qt[6], L->wd, H, F, s, t, NULL, nthreads)) goto done;
  for (int64_t i = 0; i < H; ++i) h2[i] = h1[i] + t[i];

  if (cos_out) *cos_out = orc_cosine(h, h2, H);
  memcpy(h_out, h2, sizeof(double) * (size_t)H);
  rc = 0;
done:
  free(h); free(wn); free(n1); free(q); free(k); free(v); free(a); free(t); free(h1); free(n2); free(g); free(u);
  free(s); free(h2);
  return rc;
}

/* Embedding lookup: fp16 row `token` of a [vocab][hidden] table. */
void orc_embed(const uint16_t* table, int64_t hidden, int64_t token, double* out) {
  for (int64_t i = 0; i < hidden; ++i) out[i] = orc_half(table[token * hidden + i]);
}

/* Output head: logits = W_head (RMSNorm(h) w_final). */
int orc_head(const orc_config* c, int head_qtype, const uint8_t* head, const float* final_norm, const double* h,
             double* logits, int nthreads) {
  const int64_t H = c->hidden;
  double *wn = dalloc(H), *n = dalloc(H);
  int rc = -1;
  if (wn && n) {
    for (int64_t i = 0; i < H; ++i) wn[i] = (double)final_norm[i];
    orc_rmsnorm(h, wn, H, c->eps, n);
    rc = orc_gemv(head_qtype, head, c->vocab, H, n, logits, NULL, nthreads);
  }
  free(wn); free(n);
  return rc;
}
