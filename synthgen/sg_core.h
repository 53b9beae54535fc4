/*
 * sg_core.h -- seeded, counter-based synthetic-input generator (shared by the
 * host C build and its CUDA twin; nothing else includes it).
 *
 * This module only MAKES inputs: random fp32/fp16 tensors, random token ids and
 * GGUF-style block-quantized weight matrices built from random fp32 weights.
 * It holds none of the arithmetic that is being tested (no dequantisation, no
 * GEMV, no normalisation, no attention).  Both the CPU oracle and the CUDA path
 * consume its output bytes; neither links the other.
 *
 * Every value is a pure function of (seed, tensor id, element index), so the
 * host and the device produce identical bytes regardless of threading or
 * launch shape.  To make that hold bit for bit, only IEEE-754 basic operations
 * (+ - * / sqrt, conversions) are used, each rounded to nearest-even, with no
 * fused multiply-add: the host file is compiled with -ffp-contract=off and the
 * device side spells each operation as an explicit _rn intrinsic.
 *
 *  - Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *    easy as 1, 2, 3", SC'11 (the published round function, multipliers and
 *    Weyl key increments).
 *  - Normal deviates: Marsaglia & Bray's polar method (SIAM Review 6, 1964),
 *    with the natural log evaluated by the atanh series
 *    ln m = 2 atanh((m-1)/(m+1)) after splitting off the binary exponent.
 *  - Quantisers: the recipes stated for the synthetic workloads (Q8_0: d =
 *    max|w|/127, q = round(w/d); Q4_0: d = (signed max-|w| element)/-8,
 *    q = clamp(round(w/d)+8, 0, 15); Q6_K: 16-element sub-block scales stored
 *    as int8 relative to one fp16 super-scale, q = clamp(round(w/(d*sc))+32,
 *    0, 63); Q4_K / Q5_K: per 32-element sub-block a scale (max - min')/n_max
 *    and a min -min' with min' = min(0, smallest element), both stored as 6-bit
 *    codes relative to fp16 super-scales d = (largest scale)/63 and dmin =
 *    (largest min)/63, q = clamp(round((w + dmin m)/(d sc)), 0, n_max) with
 *    n_max 15 / 31; F16 / F32: the value itself), rounding half away from
 *    zero, block byte layouts as GGUF stores them (per-format layout in the
 *    functions below).
 */
#ifndef SG_CORE_H
#define SG_CORE_H

#include <stdint.h>

#ifdef __CUDACC__
#define SG_HD static __host__ __device__ __forceinline__
#else
#define SG_HD static inline
#endif

/* Explicitly rounded IEEE basic operations. */
#if defined(__CUDA_ARCH__)
#define SG_DADD(a, b) __dadd_rn((a), (b))
#define SG_DSUB(a, b) __dsub_rn((a), (b))
#define SG_DMUL(a, b) __dmul_rn((a), (b))
#define SG_DDIV(a, b) __ddiv_rn((a), (b))
#define SG_DSQRT(a) __dsqrt_rn((a))
#define SG_D2F(a) __double2float_rn((a))
#define SG_FMUL(a, b) __fmul_rn((a), (b))
#define SG_FDIV(a, b) __fdiv_rn((a), (b))
#define SG_FADD(a, b) __fadd_rn((a), (b))
#define SG_FSUB(a, b) __fsub_rn((a), (b))
#define SG_AS_U64(d) ((uint64_t)__double_as_longlong(d))
#define SG_AS_DBL(u) (__longlong_as_double((long long)(u)))
#define SG_AS_U32(f) ((uint32_t)__float_as_uint(f))
#define SG_AS_FLT(u) (__uint_as_float(u))
#else
#include <string.h>
#define SG_DADD(a, b) ((a) + (b))
#define SG_DSUB(a, b) ((a) - (b))
#define SG_DMUL(a, b) ((a) * (b))
#define SG_DDIV(a, b) ((a) / (b))
#define SG_DSQRT(a) __builtin_sqrt((a))
#define SG_D2F(a) ((float)(a))
#define SG_FMUL(a, b) ((a) * (b))
#define SG_FDIV(a, b) ((a) / (b))
#define SG_FADD(a, b) ((a) + (b))
#define SG_FSUB(a, b) ((a) - (b))
SG_HD uint64_t sg_as_u64_(double d) { uint64_t u; memcpy(&u, &d, 8); return u; }
SG_HD double sg_as_dbl_(uint64_t u) { double d; memcpy(&d, &u, 8); return d; }
SG_HD uint32_t sg_as_u32_(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
SG_HD float sg_as_flt_(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
#define SG_AS_U64(d) sg_as_u64_(d)
#define SG_AS_DBL(u) sg_as_dbl_(u)
#define SG_AS_U32(f) sg_as_u32_(f)
#define SG_AS_FLT(u) sg_as_flt_(u)
#endif

/* GGUF type ids of the formats produced here. */
#define SG_F32 0
#define SG_F16 1
#define SG_Q4_0 2
#define SG_Q8_0 8
#define SG_Q4_K 12
#define SG_Q5_K 13
#define SG_Q6_K 14

/* Counter word 3 tags the use of a draw so streams never overlap. */
#define SG_TAG_NORMAL 0x4E4F524Du /* "NORM" */
#define SG_TAG_TOKEN 0x544F4B4Eu  /* "TOKN" */

/* ---------------------------------------------------------------- Philox */
SG_HD void sg_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += W0; k1 += W1; }
    uint64_t p0 = (uint64_t)M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* FNV-1a, 32 bit: maps a tensor name to its Philox key word. */
SG_HD uint32_t sg_fnv1a(const char* s) {
  uint32_t h = 2166136261u;
  while (*s) { h ^= (uint8_t)(*s++); h *= 16777619u; }
  return h;
}

/* --------------------------------------------------------- normal deviate */
/* u in [0, 2^32) -> (u + 1/2) 2^-31 - 1 in (-1, 1); every step is exact. */
SG_HD double sg_u32_to_pm1(uint32_t u) {
  return SG_DSUB(SG_DMUL(SG_DADD((double)u, 0.5), 4.656612873077392578125e-10), 1.0);
}

/* Natural log of s in (0, 1): s = 2^e m, m folded into [1/sqrt2, sqrt2),
 * ln m = 2 t (1 + t^2/3 + t^4/5 + ...), t = (m-1)/(m+1), |t| < 0.1716. */
SG_HD double sg_ln_unit(double s) {
  uint64_t bits = SG_AS_U64(s);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;
  double m = SG_AS_DBL((bits & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull);
  if (m > 1.4142135623730951) { m = SG_DMUL(m, 0.5); e += 1; }
  double t = SG_DDIV(SG_DSUB(m, 1.0), SG_DADD(m, 1.0));
  double t2 = SG_DMUL(t, t);
  /* 1/(2k+1), k = 0..12 */
  const double c[13] = {1.0,
                        0.33333333333333331,
                        0.20000000000000001,
                        0.14285714285714285,
                        0.1111111111111111,
                        0.090909090909090912,
                        0.076923076923076927,
                        0.066666666666666666,
                        0.058823529411764705,
                        0.052631578947368418,
                        0.047619047619047616,
                        0.043478260869565216,
                        0.040000000000000001};
  double p = c[12];
  for (int k = 11; k >= 0; --k) p = SG_DADD(SG_DMUL(p, t2), c[k]);
  const double LN2 = 0.69314718055994529;
  return SG_DADD(SG_DMUL((double)e, LN2), SG_DMUL(SG_DMUL(2.0, t), p));
}

/* Standard normal deviate number `idx` of stream (seed, tid): polar method,
 * up to 8 Philox draws of two candidate pairs each; 0 if all 16 are rejected
 * (probability ~2e-11). */
SG_HD double sg_normal(uint32_t seed, uint32_t tid, uint64_t idx) {
  const uint32_t key[2] = {seed, tid};
  for (uint32_t a = 0; a < 8; ++a) {
    const uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), a, SG_TAG_NORMAL};
    uint32_t r[4];
    sg_philox4x32_10(ctr, key, r);
    for (int p = 0; p < 4; p += 2) {
      double va = sg_u32_to_pm1(r[p]);
      double vb = sg_u32_to_pm1(r[p + 1]);
      double s = SG_DADD(SG_DMUL(va, va), SG_DMUL(vb, vb));
      if (s > 0.0 && s < 1.0) {
        double l = sg_ln_unit(s);
        double q = SG_DDIV(SG_DMUL(-2.0, l), s);
        return SG_DMUL(va, SG_DSQRT(q));
      }
    }
  }
  return 0.0;
}

/* mean + sigma * z, rounded once to fp32. */
SG_HD float sg_normal_f32(uint32_t seed, uint32_t tid, uint64_t idx, double mean, double sigma) {
  return SG_D2F(SG_DADD(mean, SG_DMUL(sigma, sg_normal(seed, tid, idx))));
}

/* Uniform token id in [0, V): high word of u * V (exact integer arithmetic). */
SG_HD int32_t sg_token(uint32_t seed, uint32_t tid, uint64_t idx, uint32_t V) {
  const uint32_t key[2] = {seed, tid};
  const uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), 0u, SG_TAG_TOKEN};
  uint32_t r[4];
  sg_philox4x32_10(ctr, key, r);
  return (int32_t)(((uint64_t)r[0] * (uint64_t)V) >> 32);
}

/* ------------------------------------------------------- fp16 conversion */
/* IEEE binary32 -> binary16, round to nearest even (bit manipulation). */
SG_HD uint16_t sg_f32_to_f16(float f) {
  uint32_t x = SG_AS_U32(f);
  uint32_t sign = (x >> 16) & 0x8000u;
  uint32_t ax = x & 0x7FFFFFFFu;
  if (ax >= 0x7F800000u) return (uint16_t)(sign | (ax > 0x7F800000u ? 0x7E00u : 0x7C00u));
  if (ax >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u); /* rounds to >= 65520: inf */
  if (ax < 0x38800000u) {                                     /* below 2^-14: subnormal half */
    if (ax < 0x33000000u) return (uint16_t)sign;             /* < 2^-25: rounds to 0 */
    uint32_t e = ax >> 23;
    uint32_t m = (ax & 0x7FFFFFu) | 0x800000u;
    uint32_t shift = 126u - e; /* value = m * 2^(e-150); half ulp = 2^-24 */
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
    return (uint16_t)(sign | q);
  }
  uint32_t e = (ax >> 23) - 112u; /* rebias 127 -> 15 */
  uint32_t m = ax & 0x7FFFFFu;
  uint32_t q = (e << 10) | (m >> 13);
  uint32_t rem = m & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (q & 1u))) q += 1u;
  return (uint16_t)(sign | q);
}

/* binary16 -> binary32 (exact). */
SG_HD float sg_f16_to_f32(uint16_t h) {
  uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
  uint32_t e = ((uint32_t)h >> 10) & 0x1Fu;
  uint32_t m = (uint32_t)h & 0x3FFu;
  if (e == 0x1Fu) return SG_AS_FLT(sign | 0x7F800000u | (m << 13));
  if (e == 0) {
    if (m == 0) return SG_AS_FLT(sign);
    int k = 0;
    while (!(m & 0x400u)) { m <<= 1; ++k; }
    m &= 0x3FFu;
    return SG_AS_FLT(sign | ((uint32_t)(113 - k) << 23) | (m << 13));
  }
  return SG_AS_FLT(sign | ((e + 112u) << 23) | (m << 13));
}

/* ------------------------------------------------------------ quantisers */
SG_HD float sg_fabs(float v) { return SG_AS_FLT(SG_AS_U32(v) & 0x7FFFFFFFu); }

/* Round half away from zero of a finite float to int (the float is already an
 * exact quotient; truncation + compare keeps it exact). */
SG_HD int sg_round_away(float v) {
  float a = sg_fabs(v);
  if (a >= 8388608.0f) return (int)v;
  int t = (int)a; /* floor of |v| */
  float fr = a - (float)t; /* exact */
  if (fr >= 0.5f) t += 1;
  return (SG_AS_U32(v) & 0x80000000u) ? -t : t;
}

SG_HD int sg_clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Q8_0: 34 bytes = fp16 d | int8 q[32]; w = d * q. */
SG_HD void sg_quant_q8_0(const float* w, uint8_t* blk) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) { float a = sg_fabs(w[i]); if (a > amax) amax = a; }
  float d = SG_FDIV(amax, 127.0f);
  uint16_t dh = sg_f32_to_f16(d);
  blk[0] = (uint8_t)(dh & 0xFF); blk[1] = (uint8_t)(dh >> 8);
  for (int i = 0; i < 32; ++i) {
    int q = (amax == 0.0f) ? 0 : sg_clampi(sg_round_away(SG_FDIV(w[i], d)), -127, 127);
    blk[2 + i] = (uint8_t)(int8_t)q;
  }
}

/* Q4_0: 18 bytes = fp16 d | 16 bytes; byte j holds element j in its low
 * nibble and element j+16 in its high nibble; w = d * (q - 8). */
SG_HD void sg_quant_q4_0(const float* w, uint8_t* blk) {
  float amax = 0.0f, m = 0.0f;
  for (int i = 0; i < 32; ++i) { float a = sg_fabs(w[i]); if (a > amax) { amax = a; m = w[i]; } }
  float d = SG_FDIV(m, -8.0f);
  uint16_t dh = sg_f32_to_f16(d);
  blk[0] = (uint8_t)(dh & 0xFF); blk[1] = (uint8_t)(dh >> 8);
  uint8_t q[32];
  for (int i = 0; i < 32; ++i)
    q[i] = (uint8_t)((amax == 0.0f) ? 8 : sg_clampi(sg_round_away(SG_FDIV(w[i], d)) + 8, 0, 15));
  for (int j = 0; j < 16; ++j) blk[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));
}

/* Q6_K: 210 bytes = ql[128] | qh[64] | int8 scales[16] | fp16 d.
 * Element n of the 256: h = n/128, r = n%128, g = r/32, l = r%32;
 *   low 4 bits  in ql[64h + 32(g&1) + l] (low nibble for g<2, high for g>=2),
 *   high 2 bits in qh[32h + l] at bit 2g,
 *   sub-block scale scales[n/16];  w = d * scale * (q - 32). */
SG_HD void sg_quant_q6_k(const float* w, uint8_t* blk) {
  float s[16];
  float smax = 0.0f, S = 0.0f;
  for (int j = 0; j < 16; ++j) {
    float amax = 0.0f, m = 0.0f;
    for (int i = 0; i < 16; ++i) { float a = sg_fabs(w[16 * j + i]); if (a > amax) { amax = a; m = w[16 * j + i]; } }
    s[j] = SG_FDIV(m, -32.0f);
    float as = sg_fabs(s[j]);
    if (as > smax) { smax = as; S = s[j]; }
  }
  uint16_t dh = sg_f32_to_f16(SG_FDIV(S, -128.0f));
  float df = sg_f16_to_f32(dh);
  int8_t sc[16];
  for (int j = 0; j < 16; ++j)
    sc[j] = (int8_t)((df == 0.0f) ? 0 : sg_clampi(sg_round_away(SG_FDIV(s[j], df)), -128, 127));
  uint8_t q[256];
  for (int n = 0; n < 256; ++n) {
    float step = SG_FMUL(df, (float)sc[n / 16]);
    q[n] = (uint8_t)((step == 0.0f) ? 32 : sg_clampi(sg_round_away(SG_FDIV(w[n], step)) + 32, 0, 63));
  }
  uint8_t* ql = blk;
  uint8_t* qh = blk + 128;
  for (int i = 0; i < 128; ++i) ql[i] = 0;
  for (int i = 0; i < 64; ++i) qh[i] = 0;
  for (int n = 0; n < 256; ++n) {
    int h = n / 128, r = n % 128, g = r / 32, l = r % 32;
    int qi = 64 * h + 32 * (g & 1) + l;
    ql[qi] |= (uint8_t)((q[n] & 0xF) << (g >= 2 ? 4 : 0));
    qh[32 * h + l] |= (uint8_t)(((q[n] >> 4) & 0x3) << (2 * g));
  }
  for (int j = 0; j < 16; ++j) blk[192 + j] = (uint8_t)sc[j];
  blk[208] = (uint8_t)(dh & 0xFF); blk[209] = (uint8_t)(dh >> 8);
}

/* Q4_K (144 bytes) / Q5_K (176 bytes) super-blocks of 256:
 *   fp16 d | fp16 dmin | scales[12] | (Q5_K: qh[32]) | qs[128];
 * sub-block j (32 elements) has a 6-bit scale sc_j and min m_j:
 *   j < 4:  sc_j = scales[j] & 63, m_j = scales[j+4] & 63;
 *   j >= 4: sc_j = (scales[j+4] & 15) | (scales[j-4] >> 6) << 4,
 *           m_j  = (scales[j+4] >> 4) | (scales[j] >> 6) << 4;
 * element n = 64c + 32h + l takes nibble h of qs[32c + l] (and, for Q5_K,
 * bit 2c + h of qh[l] as its fifth bit);  w = d sc_j q - dmin m_j. */
SG_HD void sg_quant_kq(const float* w, uint8_t* blk, int five) {
  const int nmax = five ? 31 : 15;
  float s[8], mm[8], smax = 0.0f, mmax = 0.0f;
  for (int j = 0; j < 8; ++j) {
    float mn = 0.0f, mx = w[32 * j];
    for (int i = 0; i < 32; ++i) {
      float v = w[32 * j + i];
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    s[j] = SG_FDIV(SG_FSUB(mx, mn), (float)nmax);
    mm[j] = SG_FSUB(0.0f, mn);
    if (s[j] > smax) smax = s[j];
    if (mm[j] > mmax) mmax = mm[j];
  }
  uint16_t dh = sg_f32_to_f16(SG_FDIV(smax, 63.0f)), mh = sg_f32_to_f16(SG_FDIV(mmax, 63.0f));
  float df = sg_f16_to_f32(dh), mf = sg_f16_to_f32(mh);
  int sc[8], mi[8];
  for (int j = 0; j < 8; ++j) {
    sc[j] = (df == 0.0f) ? 0 : sg_clampi(sg_round_away(SG_FDIV(s[j], df)), 0, 63);
    mi[j] = (mf == 0.0f) ? 0 : sg_clampi(sg_round_away(SG_FDIV(mm[j], mf)), 0, 63);
  }
  blk[0] = (uint8_t)(dh & 0xFF); blk[1] = (uint8_t)(dh >> 8);
  blk[2] = (uint8_t)(mh & 0xFF); blk[3] = (uint8_t)(mh >> 8);
  uint8_t* p = blk + 4;
  for (int j = 0; j < 4; ++j) {
    p[j] = (uint8_t)((sc[j] & 63) | ((sc[j + 4] >> 4) << 6));
    p[j + 4] = (uint8_t)((mi[j] & 63) | ((mi[j + 4] >> 4) << 6));
    p[j + 8] = (uint8_t)((sc[j + 4] & 15) | ((mi[j + 4] & 15) << 4));
  }
  uint8_t* qh = blk + 16;
  uint8_t* qs = blk + (five ? 48 : 16);
  for (int i = 0; i < 128; ++i) qs[i] = 0;
  if (five)
    for (int i = 0; i < 32; ++i) qh[i] = 0;
  for (int n = 0; n < 256; ++n) {
    const int j = n / 32, c = n / 64, h = (n % 64) / 32, l = n % 32;
    float step = SG_FMUL(df, (float)sc[j]);
    float off = SG_FMUL(mf, (float)mi[j]);
    int q = (step == 0.0f) ? 0 : sg_clampi(sg_round_away(SG_FDIV(SG_FADD(w[n], off), step)), 0, nmax);
    qs[32 * c + l] |= (uint8_t)((q & 15) << (4 * h));
    if (five) qh[l] |= (uint8_t)(((q >> 4) & 1) << (2 * c + h));
  }
}

/* F16: one binary16 per weight (little-endian); F32: the binary32 itself. */
SG_HD void sg_quant_f16(const float* w, uint8_t* blk) {
  uint16_t h = sg_f32_to_f16(w[0]);
  blk[0] = (uint8_t)(h & 0xFF); blk[1] = (uint8_t)(h >> 8);
}
SG_HD void sg_quant_f32(const float* w, uint8_t* blk) {
  uint32_t u = SG_AS_U32(w[0]);
  for (int i = 0; i < 4; ++i) blk[i] = (uint8_t)(u >> (8 * i));
}

SG_HD int sg_block_elems(int qtype) {
  switch (qtype) {
    case SG_F32: case SG_F16: return 1;
    case SG_Q4_0: case SG_Q8_0: return 32;
    case SG_Q4_K: case SG_Q5_K: case SG_Q6_K: return 256;
    default: return 0;
  }
}
SG_HD int sg_block_bytes(int qtype) {
  switch (qtype) {
    case SG_F32: return 4;
    case SG_F16: return 2;
    case SG_Q4_0: return 18;
    case SG_Q8_0: return 34;
    case SG_Q4_K: return 144;
    case SG_Q5_K: return 176;
    case SG_Q6_K: return 210;
    default: return 0;
  }
}

SG_HD void sg_quant_block(int qtype, const float* w, uint8_t* blk) {
  switch (qtype) {
    case SG_Q8_0: sg_quant_q8_0(w, blk); break;
    case SG_Q4_0: sg_quant_q4_0(w, blk); break;
    case SG_Q6_K: sg_quant_q6_k(w, blk); break;
    case SG_Q4_K: sg_quant_kq(w, blk, 0); break;
    case SG_Q5_K: sg_quant_kq(w, blk, 1); break;
    case SG_F16: sg_quant_f16(w, blk); break;
    case SG_F32: sg_quant_f32(w, blk); break;
    default: break;
  }
}

#endif /* SG_CORE_H */
