// gemv.cuh -- fused dequantize + GEMV for GGUF Q8_0 / Q4_0 / Q6_K on sm_100a.
//
// y = W_deq x with fp32 accumulation ("NTransformer" -- アーキテクチャ概要: the
// GEMV kernel; decode time is weight bytes over memory bandwidth, "RTX 3090
// 1枚でLlama 70B" -- VRAMの壁).  Batch-1 GEMV is not a dense contraction: it is
// bound by HBM bandwidth, so the design is about moving the packed blocks at
// full bandwidth and decoding them with few instructions, not tensor cores.
//
// Work decomposition (one persistent CTA per SM)
//  * Output rows are split evenly over the CTAs (in units of 1 or 2 rows so
//    that paired epilogues see both rows of a pair).  A CTA streams its rows in
//    stages of TR whole rows: one 1-D bulk copy (TMA, cp.async.bulk) per row
//    into a ring of S shared-memory stages guarded by full/empty mbarriers.
//  * K is split into slices of 2048 columns.  Consumer warp (c, g) owns slice
//    c and row group g: its lanes hold their 64 columns of x (fp32, or
//    RMSNorm(h) w formed on the fly) in registers for the whole kernel, so the
//    only shared-memory traffic is the weight bytes themselves.  Each warp
//    reduces a row's partial with shuffles and leaves it in shared memory.
//  * The producer warp issues the copies (weights never depend on the previous
//    kernel, so the first S stages go out before the programmatic-launch wait),
//    sums the slice partials of each finished stage in a fixed order, runs the
//    epilogue (store, + residual, RoPE + KV append, SwiGLU pairs, residual +
//    cosine statistics, argmax) and refills the stage.
//  * Dot products are exact integer sums: x is held as 22-bit fixed point in
//    byte limbs and each block's (Q6_K: each 16-column run's) sum of code x
//    limb products is formed with dp4a in int32; block scales and the
//    fixed-point scale are applied once per block (Q6_K: once per row slice).
#pragma once

#include "common.cuh"

namespace ntx {

constexpr int QT_F32 = 0, QT_F16 = 1, QT_Q4_0 = 2, QT_Q8_0 = 8, QT_Q4_K = 12, QT_Q5_K = 13, QT_Q6_K = 14;

// Formats whose lanes hold x as fp32 in registers (no fixed-point staging).
__host__ __device__ constexpr bool qt_float(int qt) { return qt == QT_F16 || qt == QT_F32; }
// Formats with Q4_K-style super-blocks (fp16 d, dmin, packed 6-bit scales and mins).
__host__ __device__ constexpr bool qt_kmin(int qt) { return qt == QT_Q4_K || qt == QT_Q5_K; }

#ifndef NTX_GEMV_MAX_CONSUMERS
#define NTX_GEMV_MAX_CONSUMERS 15
#endif
#ifndef NTX_GEMV_STAGE_BYTES
#define NTX_GEMV_STAGE_BYTES 34816
#endif
constexpr int kSliceCols = 2048;                         // columns per K slice (64 per lane)
constexpr int kMaxConsumers = NTX_GEMV_MAX_CONSUMERS;    // consumer warps per CTA
constexpr int kMaxTR = 32;                               // rows per stage
constexpr int kStageTarget = NTX_GEMV_STAGE_BYTES;       // bytes a stage aims at
constexpr int kGemvThreads = (kMaxConsumers + 1) * 32;
constexpr int kEpiTable = 128;        // float2 entries of the epilogue table (RoPE: head_dim/2)
#ifndef NTX_GEMV_PF_BYTES
#define NTX_GEMV_PF_BYTES 0
#endif
constexpr int kGemvPrefetchBytes = NTX_GEMV_PF_BYTES;  // weight bytes per CTA requested into L2 ahead of the ring

template <int QT>
struct QTraits;
template <>
struct QTraits<QT_Q8_0> {
  static constexpr int BE = 32, BB = 34, SEG = kSliceCols / 32 * 34;
};
template <>
struct QTraits<QT_Q4_0> {
  static constexpr int BE = 32, BB = 18, SEG = kSliceCols / 32 * 18;
};
template <>
struct QTraits<QT_Q6_K> {
  static constexpr int BE = 256, BB = 210, SEG = kSliceCols / 256 * 210;
};
template <>
struct QTraits<QT_Q4_K> {
  static constexpr int BE = 256, BB = 144, SEG = kSliceCols / 256 * 144;
};
template <>
struct QTraits<QT_Q5_K> {
  static constexpr int BE = 256, BB = 176, SEG = kSliceCols / 256 * 176;
};
template <>
struct QTraits<QT_F16> {
  static constexpr int BE = 1, BB = 2, SEG = kSliceCols * 2;
};
template <>
struct QTraits<QT_F32> {
  static constexpr int BE = 1, BB = 4, SEG = kSliceCols * 4;
};

__host__ __device__ constexpr int qt_block_elems(int qt) {
  return qt == QT_Q6_K || qt == QT_Q4_K || qt == QT_Q5_K ? 256 : qt_float(qt) ? 1 : 32;
}
__host__ __device__ constexpr int qt_block_bytes(int qt) {
  return qt == QT_Q6_K ? 210 : qt == QT_Q4_K ? 144 : qt == QT_Q5_K ? 176 : qt == QT_Q8_0 ? 34 : qt == QT_Q4_0 ? 18
       : qt == QT_F16 ? 2 : 4;
}

// Launch plan, computed on the host.
struct GemvPlan {
  int TR;        // rows per stage
  int S;         // stages in the ring
  int n_slices;  // ceil(K / 2048)
  int n_rg;      // row groups (consumer warps per slice)
  int NW;        // consumer warps = n_slices * n_rg
  int row_bytes;
  int stage_bytes;
  int xstage_bytes;  // shared memory holding x for the lanes (16-byte multiple)
  int pf_stages;     // stages kept requested into L2 ahead of the ring (0: none)
};

// ------------------------------------------------------------- row maps
struct MapSingle {
  const uint8_t* W;
  int64_t row_bytes;
  __device__ __forceinline__ const uint8_t* row(int64_t r) const { return W + r * row_bytes; }
};

// Rows [0, nq) from Wq, [nq, nq+nkv) from Wk, [nq+nkv, nq+2nkv) from Wv.
struct MapQKV {
  const uint8_t *Wq, *Wk, *Wv;
  int64_t row_bytes, nq, nkv;
  __device__ __forceinline__ const uint8_t* row(int64_t r) const {
    if (r < nq) return Wq + r * row_bytes;
    if (r < nq + nkv) return Wk + (r - nq) * row_bytes;
    return Wv + (r - nq - nkv) * row_bytes;
  }
};

// Logical row 2i is row i of Wa, 2i+1 is row i of Wb (gate/up pairs).
struct MapPair {
  const uint8_t *Wa, *Wb;
  int64_t row_bytes;
  __device__ __forceinline__ const uint8_t* row(int64_t r) const { return ((r & 1) ? Wb : Wa) + (r >> 1) * row_bytes; }
};

// ------------------------------------------------------------- x loaders
struct ProPlain {
  const float* x;
  __device__ __forceinline__ void setup(int) {}
  __device__ __forceinline__ float4 ld(int64_t j) const { return ldg4(x + j); }
};

// x_j = w_j * (h_j * r),  r = 1 / sqrt(sum(h^2)/n + eps), sum(h^2) from the
// producer's per-CTA partials (slot 0 of 4 floats per CTA).
struct ProRms {
  const float* h;
  const float* w;
  const float* parts;
  int nparts;
  int n;
  float eps;
  float r;
  __device__ __forceinline__ void setup(int lane) {
    const float ss = warp_sum_array(parts, nparts, 4, lane);
    r = 1.0f / sqrtf(ss / (float)n + eps);
  }
  __device__ __forceinline__ float4 ld(int64_t j) const {
    const float4 a = ldg4(h + j), b = ldg4(w + j);
    return make_float4(b.x * (a.x * r), b.y * (a.y * r), b.z * (a.z * r), b.w * (a.w * r));
  }
};

// ---------------------------------------------------------------------------
// Q8_0 / Q4_0: exact integer block dot products.
//
// A lane owns two whole 32-column blocks of x.  Once per kernel it stores each
// block in 22-bit block fixed point: X_i = rint(x_i * 2^(22-e)) with 2^e >
// max|x| over the block (|X_i| <= 2^22; the representation error of each x_i
// is at most 2^-23 of the block's largest |x|), split into byte limbs
// X = L0 + 2^8 L1 + 2^16 L2 (L0, L1 unsigned, L2 signed), four columns per
// 32-bit register.  A block's sum_i q_i X_i is then three sums of 4-way byte
// dot products (dp4a), exact in int32, combined and scaled once in fp32:
// d * 2^(e-22) * (2^16 A2 + 2^8 A1 + A0).  Q8_0 codes are int8 as stored;
// Q4_0 nibbles are unsigned and the -8 offset is folded into the starting
// value of each limb's accumulator (-8 times the block's limb sum).
struct XFix {
  uint32_t l0[16], l1[16], l2[16];  // block b, word k (columns 4k..4k+3) at [8b + k]
  float xs[2];                      // 2^(e_b - 22)
  int c0[2], c1[2], c2[2];          // -8 * sum of the block's limb bytes (Q4_0)
  float sx[2];                      // sum of the block's x values (Q4_K / Q5_K: the min term)
};

__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  uint32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return (int)d;
}
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ float limbs_to_f(int a0, int a1, int a2) {
  return fmaf((float)a2, 65536.0f, (float)a1 * 256.0f) + (float)a0;
}

// Q8_0 rows: lane l owns blocks 2l, 2l+1 (68 bytes = 17 words at offset 68 l).
// Block 0: scale = low half of word 0, codes at bytes 2..33 (re-aligned by a
// funnel shift); block 1: scale = high half of word 8, codes = words 9..16.
__device__ __forceinline__ float rowfix_q8_0(const uint8_t* seg, int lane, const XFix& x) {
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(seg + lane * 68);
  uint32_t w[17];
#pragma unroll
  for (int i = 0; i < 17; ++i) w[i] = wp[i];
  float r = 0.f;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    int a0 = 0, a1 = 0, a2 = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t q = b == 0 ? __funnelshift_r(w[k], w[k + 1], 16) : w[9 + k];
      a0 = dp4a_su(q, x.l0[8 * b + k], a0);
      a1 = dp4a_su(q, x.l1[8 * b + k], a1);
      a2 = dp4a_ss(q, x.l2[8 * b + k], a2);
    }
    const float d = half_bits_to_float(b == 0 ? w[0] : (w[8] >> 16));
    r = fmaf(d * x.xs[b], limbs_to_f(a0, a1, a2), r);
  }
  return r;
}

// Q4_0 rows: lane l owns blocks 2l, 2l+1 (36 bytes = 9 words at offset 36 l).
// Block 0: scale = low half of word 0, nibble bytes 2..17 (re-aligned);
// block 1: scale = high half of word 4, nibble bytes = words 5..8.  Nibble
// word k: low nibbles are elements 4k..4k+3, high nibbles 16+4k..16+4k+3.
__device__ __forceinline__ float rowfix_q4_0(const uint8_t* seg, int lane, const XFix& x) {
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(seg + lane * 36);
  uint32_t w[9];
#pragma unroll
  for (int i = 0; i < 9; ++i) w[i] = wp[i];
  float r = 0.f;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    int a0 = x.c0[b], a1 = x.c1[b], a2 = x.c2[b];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t n = b == 0 ? __funnelshift_r(w[k], w[k + 1], 16) : w[5 + k];
      const uint32_t lo = n & 0x0F0F0F0Fu, hi = (n >> 4) & 0x0F0F0F0Fu;
      a0 = dp4a_uu(lo, x.l0[8 * b + k], a0);
      a0 = dp4a_uu(hi, x.l0[8 * b + 4 + k], a0);
      a1 = dp4a_uu(lo, x.l1[8 * b + k], a1);
      a1 = dp4a_uu(hi, x.l1[8 * b + 4 + k], a1);
      a2 = dp4a_us(lo, x.l2[8 * b + k], a2);
      a2 = dp4a_us(hi, x.l2[8 * b + 4 + k], a2);
    }
    const float d = half_bits_to_float(b == 0 ? w[0] : (w[4] >> 16));
    r = fmaf(d * x.xs[b], limbs_to_f(a0, a1, a2), r);
  }
  return r;
}

// Q4_K / Q5_K rows: a slice is 8 super-blocks; lane l owns super-block
// sb = l / 4 and its 64-element chunk c = l % 4, i.e. the slice columns
// 64 l .. 64 l + 63 as for Q8_0: sub-block 2c (low nibbles of the chunk's 32
// code bytes, x words 0..7) and sub-block 2c + 1 (high nibbles, x words
// 8..15).  Every super-block starts 16-byte aligned (144 / 176 bytes), so the
// header (d, dmin, 12 scale bytes) and the codes come in as 16-byte loads.
// With A_b the exact integer sum of code x limb products of sub-block b and
// X_b the sum of its fixed-point x, the lane's share of the row is
//   sum_b 2^(e_b-22) (d sc_b A_b - dmin m_b X_b).
// The 6-bit scale and min of sub-block j: j < 4 from the low six bits of
// scale bytes j and j + 4; j >= 4 from the nibbles of byte j + 4 and the top
// two bits of bytes j - 4 (scale) and j (min) -- chosen without branches
// since c varies across the warp.
__device__ __forceinline__ void kq_scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int c, int t, float& sc,
                                             float& mn) {
  const uint32_t sh = 8u * (uint32_t)((2 * c + t) & 3);
  const uint32_t b0 = (s0 >> sh) & 0xFFu, b1 = (s1 >> sh) & 0xFFu, b2 = (s2 >> sh) & 0xFFu;
  const uint32_t lo_sc = b0 & 63u, lo_m = b1 & 63u;
  const uint32_t hi_sc = (b2 & 15u) | ((b0 >> 6) << 4), hi_m = (b2 >> 4) | ((b1 >> 6) << 4);
  sc = (float)(c < 2 ? lo_sc : hi_sc);
  mn = (float)(c < 2 ? lo_m : hi_m);
}

template <bool FIVE>
__device__ __forceinline__ float rowfix_kq(const uint8_t* seg, int lane, const XFix& x) {
  const int sb = lane >> 2, c = lane & 3;
  const uint8_t* blk = seg + (FIVE ? 176 : 144) * sb;
  const uint4 hdr = *reinterpret_cast<const uint4*>(blk);
  const uint4* qp = reinterpret_cast<const uint4*>(blk + (FIVE ? 48 : 16) + 32 * c);
  const uint4 qa = qp[0], qb = qp[1];
  const uint32_t qs[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
  uint32_t qh[8];
  if constexpr (FIVE) {
    const uint4* hp = reinterpret_cast<const uint4*>(blk + 16);
    const uint4 ha = hp[0], hb = hp[1];
    qh[0] = ha.x; qh[1] = ha.y; qh[2] = ha.z; qh[3] = ha.w;
    qh[4] = hb.x; qh[5] = hb.y; qh[6] = hb.z; qh[7] = hb.w;
  }
  int a0 = 0, a1 = 0, a2 = 0, b0 = 0, b1 = 0, b2 = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t lo = qs[k] & 0x0F0F0F0Fu, hi = (qs[k] >> 4) & 0x0F0F0F0Fu;
    if constexpr (FIVE) {
      lo |= ((qh[k] >> (2 * c)) & 0x01010101u) << 4;
      hi |= ((qh[k] >> (2 * c + 1)) & 0x01010101u) << 4;
    }
    a0 = dp4a_uu(lo, x.l0[k], a0);
    a1 = dp4a_uu(lo, x.l1[k], a1);
    a2 = dp4a_us(lo, x.l2[k], a2);
    b0 = dp4a_uu(hi, x.l0[8 + k], b0);
    b1 = dp4a_uu(hi, x.l1[8 + k], b1);
    b2 = dp4a_us(hi, x.l2[8 + k], b2);
  }
  const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
  float sca, mna, scb, mnb;
  kq_scale_min(hdr.y, hdr.z, hdr.w, c, 0, sca, mna);
  kq_scale_min(hdr.y, hdr.z, hdr.w, c, 1, scb, mnb);
  const float ta = (d * sca) * x.xs[0], tb = (d * scb) * x.xs[1];
  float r = fmaf(ta, limbs_to_f(a0, a1, a2), tb * limbs_to_f(b0, b1, b2));
  return fmaf(-dmin, fmaf(mna, x.sx[0], mnb * x.sx[1]), r);
}

// F16 / F32 rows: x stays fp32 in the lane's registers.  F16: lane l owns the
// slice columns 8 l + 256 i + t (i < 8, t < 8), one 16-byte load per i;
// F32: columns 4 l + 128 i + t (i < 16, t < 4).  Consecutive lanes read
// consecutive 16 bytes, so the loads are free of bank conflicts.  ni = the
// slice's valid 16-byte groups per lane (K a multiple of 256).
template <int QT>
struct XFloat {
  float v[64];
  int ni;
  template <class Pro>
  __device__ __forceinline__ void load_direct(const Pro& pro, int64_t c0, int ucols, int lane) {
    constexpr int W = QT == QT_F16 ? 8 : 4;   // columns per 16-byte group
    constexpr int STEP = 32 * W;              // columns between a lane's groups
    ni = ucols / STEP;
#pragma unroll
    for (int i = 0; i < 64 / W; ++i) {
      if (i < ni) {
#pragma unroll
        for (int q = 0; q < W / 4; ++q) {
          const float4 f = pro.ld(c0 + (int64_t)STEP * i + W * lane + 4 * q);
          v[W * i + 4 * q + 0] = f.x;
          v[W * i + 4 * q + 1] = f.y;
          v[W * i + 4 * q + 2] = f.z;
          v[W * i + 4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int t = 0; t < W; ++t) v[W * i + t] = 0.f;
      }
    }
  }
  __device__ __forceinline__ float dot(const uint8_t* seg, int lane) const {
    float r0 = 0.f, r1 = 0.f;
    if constexpr (QT == QT_F16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < ni) {
          const uint4 w = *reinterpret_cast<const uint4*>(seg + 512 * i + 16 * lane);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            r0 = fmaf(half_bits_to_float(ww[k]), v[8 * i + 2 * k], r0);
            r1 = fmaf(half_bits_to_float(ww[k] >> 16), v[8 * i + 2 * k + 1], r1);
          }
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < ni) {
          const float4 w = *reinterpret_cast<const float4*>(seg + 512 * i + 16 * lane);
          r0 = fmaf(w.x, v[4 * i + 0], r0);
          r1 = fmaf(w.y, v[4 * i + 1], r1);
          r0 = fmaf(w.z, v[4 * i + 2], r0);
          r1 = fmaf(w.w, v[4 * i + 3], r1);
        }
      }
    }
    return r0 + r1;
  }
};

// Q6_K: a slice is 8 super-blocks (1680 bytes).  Lane l owns super-block
// sb = l >> 2, half h = (l >> 1) & 1 and run r16 = l & 1: the elements
// 128h + 32g + 16 r16 + i (g < 4, i < 16) -- four runs of 16 that each lie in
// one 16-element sub-block (scale index 8h + r16 + 2g).  Their low nibbles are
// 16 consecutive ql bytes at 64h + 32(g & 1) + 16 r16 (low nibble for g < 2,
// high for g >= 2), their top bits the 2-bit field 2g of the 16 qh bytes at
// 128 + 32h + 16 r16: 12 words of quant bytes and 2 of scales serve 64
// elements.  Super-blocks sit 210 bytes apart, so an odd one starts 2 bytes
// past a word boundary; its words are re-aligned with a funnel shift (shift 0
// for the even ones, so every lane runs the same code).
//
// The dot product is the integer one of Q8_0 / Q4_0: x in 22-bit block fixed
// point (32-column blocks; run g of a lane is half of block 8 sb + 4h + g of
// the slice, the other half belongs to lane l ^ 1), byte limbs, dp4a sums of
// the unsigned 6-bit codes q in int32; the -32 offset is folded into the
// starting value of each limb's sum (-32 times the run's limb sum), and each
// run's sum is scaled by its sub-block scale, the block scale of x and d.
struct XFix6 {
  uint32_t l0[16], l1[16], l2[16];  // word 4g + w = columns 4w..4w+3 of run g
  float xs;                         // 2^(e - 22) of the lane's 128-column group (all four runs)
  int c[4][3];                      // -32 * sum of run g's limb-j bytes
};

// Four words at byte offset o of a super-block (o a multiple of 4), given the
// aligned word pointer below the super-block and the re-alignment shift.
__device__ __forceinline__ void q6k_run4(const uint32_t* wb, int o, uint32_t sh, uint32_t* w) {
  const uint32_t* p = wb + (o >> 2);
  uint32_t a[5];
#pragma unroll
  for (int k = 0; k < 5; ++k) a[k] = p[k];
#pragma unroll
  for (int k = 0; k < 4; ++k) w[k] = __funnelshift_r(a[k], a[k + 1], sh);
}


__device__ __forceinline__ float rowfix_q6_k(const uint8_t* seg, int lane, const XFix6& x) {
  const int sb = lane >> 2, h = (lane >> 1) & 1, r16 = lane & 1;
  const uint32_t boff = 210u * (uint32_t)sb;
  const uint32_t* wb = reinterpret_cast<const uint32_t*>(seg + (boff & ~3u));
  const uint32_t sh = (boff & 3u) * 8u;  // 0 or 16
  const uint32_t* sp = wb + ((192 + 8 * h) >> 2);
  // the lane's sub-scales (bytes r16 + 2g of scales[8h .. 8h+7]) moved to bytes 0 and 2
  const uint32_t s0 = __funnelshift_r(sp[0], sp[1], sh) >> (8 * r16);
  const uint32_t s1 = __funnelshift_r(sp[1], sp[2], sh) >> (8 * r16);
  const float d = half_bits_to_float((wb[208 >> 2] >> sh) & 0xFFFFu);
  uint32_t ql[4], qh[4];
  q6k_run4(wb, 128 + 32 * h + 16 * r16, sh, qh);
  // The four runs share one fixed-point scale, so each run's exact limb sums
  // are weighted by its int8 sub-scale in int32 (at most 2^26 in magnitude)
  // and the row's total is converted once.
  int A0 = 0, A1 = 0, A2 = 0;
  // runs g = 0, 2 share one ql run (low / high nibbles), then g = 1, 3 the other
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    q6k_run4(wb, 64 * h + 32 * half + 16 * r16, sh, ql);
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      const int g = half + 2 * gg;
      int a0 = x.c[g][0], a1 = x.c[g][1], a2 = x.c[g][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = (gg ? (ql[k] >> 4) : ql[k]) & 0x0F0F0F0Fu;
        const uint32_t hi = (g == 3) ? (qh[k] >> 2) : (qh[k] << (4 - 2 * g));
        const uint32_t q = lo | (hi & 0x30303030u);
        a0 = dp4a_uu(q, x.l0[4 * g + k], a0);
        a1 = dp4a_uu(q, x.l1[4 * g + k], a1);
        a2 = dp4a_us(q, x.l2[4 * g + k], a2);
      }
      const int sc = (int)(int8_t)(((g < 2) ? s0 : s1) >> (16 * (g & 1)));
      A0 += sc * a0;
      A1 += sc * a1;
      A2 += sc * a2;
    }
  }
  return (d * x.xs) * limbs_to_f(A0, A1, A2);
}

// A Q6_K lane's x straight from global memory (no shared staging): the lane
// converts its four runs itself.  The scale is shared by the four 32-column
// blocks the runs lie in (128 columns): the max over the lane's 64 columns and
// the partner lane's (lane ^ 1), found in a first pass over the values.
template <class Pro>
__device__ __forceinline__ void fix6_direct(const Pro& pro, int64_t c0, int lane, XFix6& x) {
  const int sb = lane >> 2, h = (lane >> 1) & 1, r16 = lane & 1;
  const int64_t base = c0 + 256 * sb + 128 * h + 16 * r16;
  float m = 0.f;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = pro.ld(base + 32 * g + 4 * q);
#pragma unroll
    for (int q = 0; q < 4; ++q) m = fmaxf(m, fmaxf(fmaxf(fabsf(v[q].x), fabsf(v[q].y)), fmaxf(fabsf(v[q].z), fabsf(v[q].w))));
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 126;
  if (e < -100) e = -100;
  const float up = __uint_as_float((uint32_t)(127 + 22 - e) << 23);
  x.xs = __uint_as_float((uint32_t)(127 + e - 22) << 23);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = pro.ld(base + 32 * g + 4 * q);
    int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float f[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
      uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int X = __float2int_rn(f[t] * up);
        const uint32_t b0 = (uint32_t)X & 0xFFu, b1 = ((uint32_t)X >> 8) & 0xFFu;
        const int hi = X >> 16;
        w0 |= b0 << (8 * t);
        w1 |= b1 << (8 * t);
        w2 |= ((uint32_t)hi & 0xFFu) << (8 * t);
        s0 += (int)b0;
        s1 += (int)b1;
        s2 += hi;
      }
      x.l0[4 * g + q] = w0;
      x.l1[4 * g + q] = w1;
      x.l2[4 * g + q] = w2;
    }
    x.c[g][0] = -32 * s0;
    x.c[g][1] = -32 * s1;
    x.c[g][2] = -32 * s2;
  }
}

// Columns of x a lane owns within its slice (relative to the slice start):
// Q8_0/Q4_0: 64 l + i;  Q6_K: 512 P + 256 odd + 128 h + 32 g + 4 j + t.
template <int QT>
__device__ __forceinline__ bool lane_active(int lane, int ucols) {
  if constexpr (QT == QT_Q6_K) return ucols == kSliceCols;  // Q6_K slices are always whole
  else if constexpr (qt_float(QT)) return ucols > 0;        // per-group bounds inside the lane
  else return 2 * lane < ucols / 32;
}

// ---------------------------------------------------------------------------
// x staging: once per CTA, the consumer warps read x (coalesced) and leave it
// in shared memory in the form the lanes need; after a named barrier among
// the consumer warps each lane copies its own part into registers.  All
// formats keep x as 22-bit block fixed point (see XFix): one warp per 128
// columns, the 8 lanes holding a 32-column block take its max|x| with
// shuffles, each lane turns its 4 columns into one 32-bit word per limb,
// stored at wd[(j*16 + k) * NP + c*32 + l] (limb j, word k of lane l of slice
// c; NP = 32 * slices + 2, the pad making the stores of a warp hit 32
// distinct banks); the block scale 2^(e-22) goes to sc[B]; cr holds the
// offset corrections (Q4_0: -8 * sum(limb j) per block; Q6_K: -32 * sum(limb
// j) per 16-column run).
struct XStage {
  uint32_t* wd;
  float* sc;
  int* cr;
  int np;
};

// Q6_K keeps one correction triple per 16-column run (K / 16 of them), Q4_0
// and the K-quants one per 32-column block; Q8_0 codes carry no offset, so it
// keeps none (the persistent kernel's plan gives the space to its weight ring).
__host__ __device__ inline size_t xstage_bytes(int qtype, int64_t K) {
  const int64_t nslices = (K + kSliceCols - 1) / kSliceCols;
  const int64_t ncorr = qtype == QT_Q6_K ? K / 16 : qtype == QT_Q8_0 ? 0 : K / 32;
  return (size_t)3 * 16 * (32 * nslices + 2) * 4 + (size_t)(K / 32) * 4 + (size_t)ncorr * 12;
}

__device__ __forceinline__ XStage xstage_at(uint8_t* base, int64_t K) {
  XStage x;
  const int64_t nslices = (K + kSliceCols - 1) / kSliceCols;
  x.np = (int)(32 * nslices + 2);
  x.wd = reinterpret_cast<uint32_t*>(base);
  x.sc = reinterpret_cast<float*>(base + (size_t)3 * 16 * x.np * 4);
  x.cr = reinterpret_cast<int*>(x.sc + K / 32);
  return x;
}

__device__ __forceinline__ float group8_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
}
__device__ __forceinline__ int group8_sum(int v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v + __shfl_xor_sync(0xffffffffu, v, 4);
}

// One 128-column chunk of x (4 columns per lane, starting at col = chunk
// start + 4 lane) into the staged form: 22-bit block fixed point, byte limbs
// packed four columns to a word, stored where the owning lane will read them.
template <int QT>
__device__ __forceinline__ void stage_chunk(const float4 v, int64_t col, const XStage& xs, int lane) {
  // Block max: per 32 columns, except Q6_K, whose lanes' four runs lie in four
  // blocks of one 128-column chunk and share one scale (this warp's chunk).
  const float am = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  const float m = QT == QT_Q6_K ? warp_max(am) : group8_max(am);
  // e with 2^(e-1) <= m < 2^e from the exponent field (m = 0 or subnormal: the
  // clamp at -100 makes every X round to 0, as it must); both scales are
  // normal powers of two built from their exponent fields.
  int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 126;
  if (e < -100) e = -100;
  const float up = __uint_as_float((uint32_t)(127 + 22 - e) << 23);
  const int X[4] = {__float2int_rn(v.x * up), __float2int_rn(v.y * up), __float2int_rn(v.z * up),
                    __float2int_rn(v.w * up)};
  uint32_t w0 = 0, w1 = 0, w2 = 0;
  int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t b0 = (uint32_t)X[t] & 0xFFu, b1 = ((uint32_t)X[t] >> 8) & 0xFFu;
    const int hi = X[t] >> 16;  // arithmetic: in [-64, 64]
    w0 |= b0 << (8 * t);
    w1 |= b1 << (8 * t);
    w2 |= ((uint32_t)hi & 0xFFu) << (8 * t);
    s0 += (int)b0;
    s1 += (int)b1;
    s2 += hi;
  }
  const int c = (int)(col / kSliceCols), u = (int)(col % kSliceCols);
  // owning lane l and word k (Q8_0/Q4_0: lane l has columns 64 l .. 64 l + 63;
  // Q6_K: see rowfix_q6_k)
  int l, k;
  if constexpr (QT == QT_Q6_K) {
    const int g = (u % 128) / 32;
    l = 4 * (u / 256) + 2 * ((u % 256) / 128) + (u % 32) / 16;
    k = 4 * g + (u % 16) / 4;
  } else {
    l = u / 64;
    k = (u % 64) / 4;
  }
  const int wi = k * xs.np + c * 32 + l;
  xs.wd[wi] = w0;
  xs.wd[16 * xs.np + wi] = w1;
  xs.wd[32 * xs.np + wi] = w2;
  const int64_t B = col / 32;
  if constexpr (qt_kmin(QT)) {
    // the block's sum of fixed-point x (|sum| < 2^27): the min term's weight
    s0 = group8_sum(s0);
    s1 = group8_sum(s1);
    s2 = group8_sum(s2);
    if ((lane & 7) == 0) xs.cr[3 * B] = s0 + 256 * s1 + 65536 * s2;
  }
  if constexpr (QT == QT_Q4_0) {
    s0 = group8_sum(s0);
    s1 = group8_sum(s1);
    s2 = group8_sum(s2);
    if ((lane & 7) == 0) {
      xs.cr[3 * B + 0] = -8 * s0;
      xs.cr[3 * B + 1] = -8 * s1;
      xs.cr[3 * B + 2] = -8 * s2;
    }
  }
  if constexpr (QT == QT_Q6_K) {
    // per 16-column run (4 lanes): -32 times the limb sums
    s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
    s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
    if ((lane & 3) == 0) {
      int* cc = xs.cr + ((int64_t)(c * 32 + l) * 4 + (u % 128) / 32) * 3;
      cc[0] = -32 * s0;
      cc[1] = -32 * s1;
      cc[2] = -32 * s2;
    }
  }
  if ((lane & 7) == 0) xs.sc[B] = __uint_as_float((uint32_t)(127 + e - 22) << 23);
}

// K is a multiple of 256 on every path that stages x.
template <int QT, class Pro>
__device__ __forceinline__ void stage_x(const Pro& pro, int64_t K, const XStage& xs, int cw, int NW, int lane) {
  constexpr int kBatch = 8;
  const int nchunk = (int)(K / 128);
  for (int ch0 = cw; ch0 < nchunk; ch0 += kBatch * NW) {
    float4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int ch = ch0 + b * NW;
      v[b] = ch < nchunk ? pro.ld((int64_t)ch * 128 + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int ch = ch0 + b * NW;
      if (ch >= nchunk) break;  // uniform across the warp
      stage_chunk<QT>(v[b], (int64_t)ch * 128 + 4 * lane, xs, lane);
    }
  }
}

// The x registers a consumer lane keeps for the whole kernel, per format.
template <int QT>
struct XRegs {
  XFix x;
  __device__ __forceinline__ void load(const XStage& xs, int c, int lane) {
    const int idx = c * 32 + lane;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      x.l0[k] = xs.wd[(0 * 16 + k) * xs.np + idx];
      x.l1[k] = xs.wd[(1 * 16 + k) * xs.np + idx];
      x.l2[k] = xs.wd[(2 * 16 + k) * xs.np + idx];
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int B = c * 64 + 2 * lane + b;
      x.xs[b] = xs.sc[B];
      if constexpr (QT == QT_Q4_0) {
        x.c0[b] = xs.cr[3 * B + 0];
        x.c1[b] = xs.cr[3 * B + 1];
        x.c2[b] = xs.cr[3 * B + 2];
      }
      if constexpr (qt_kmin(QT)) x.sx[b] = (float)xs.cr[3 * B] * x.xs[b];
    }
  }
  __device__ __forceinline__ float dot(const uint8_t* seg, int lane) const {
    if constexpr (QT == QT_Q8_0) return rowfix_q8_0(seg, lane, x);
    else if constexpr (QT == QT_Q4_K) return rowfix_kq<false>(seg, lane, x);
    else if constexpr (QT == QT_Q5_K) return rowfix_kq<true>(seg, lane, x);
    else return rowfix_q4_0(seg, lane, x);
  }
};
template <>
struct XRegs<QT_F16> {
  XFloat<QT_F16> x;
  template <class Pro>
  __device__ __forceinline__ void load_direct(const Pro& pro, int64_t c0, int ucols, int lane) {
    x.load_direct(pro, c0, ucols, lane);
  }
  __device__ __forceinline__ float dot(const uint8_t* seg, int lane) const { return x.dot(seg, lane); }
};
template <>
struct XRegs<QT_F32> {
  XFloat<QT_F32> x;
  template <class Pro>
  __device__ __forceinline__ void load_direct(const Pro& pro, int64_t c0, int ucols, int lane) {
    x.load_direct(pro, c0, ucols, lane);
  }
  __device__ __forceinline__ float dot(const uint8_t* seg, int lane) const { return x.dot(seg, lane); }
};
template <>
struct XRegs<QT_Q6_K> {
  XFix6 x;
  __device__ __forceinline__ void load(const XStage& xs, int c, int lane) {
    const int idx = c * 32 + lane;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      x.l0[k] = xs.wd[(0 * 16 + k) * xs.np + idx];
      x.l1[k] = xs.wd[(1 * 16 + k) * xs.np + idx];
      x.l2[k] = xs.wd[(2 * 16 + k) * xs.np + idx];
    }
    const int B0 = c * 64 + 8 * (lane >> 2) + 4 * ((lane >> 1) & 1);  // block of run 0
    x.xs = xs.sc[B0];  // the same for the four runs' blocks
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int* cc = xs.cr + ((int64_t)idx * 4 + g) * 3;
      x.c[g][0] = cc[0];
      x.c[g][1] = cc[1];
      x.c[g][2] = cc[2];
    }
  }
  template <class Pro>
  __device__ __forceinline__ void load_direct(const Pro& pro, int c, int lane) {
    fix6_direct(pro, (int64_t)c * kSliceCols, lane, x);
  }
  __device__ __forceinline__ float dot(const uint8_t* seg, int lane) const { return rowfix_q6_k(seg, lane, x); }
};

// ------------------------------------------------------------- epilogues
// Run by the producer warp, off the ring-refill path:
//   init(esm, lane)        once, after the programmatic-launch wait (tables);
//   preload(rs, nr, lane)  loads the global inputs of the next stage's rows
//                          into registers (latency hidden by the next wait);
//   rotate()               makes the preloaded values current;
//   apply(r, a, b)         kAlign == 1: row r has value a; kAlign == 2: rows r
//                          (even) and r + 1 have values a and b;  lane k of
//                          the producer handles row (pair) k of the stage;
//   finish(lane)           per-lane statistics reduced over the warp into
//                          parts[blockIdx.x * 4 + k].
struct EpiStore {
  float* y;
  const float* resid;
  float nres, cres;
  static constexpr int kAlign = 1;
  __device__ __forceinline__ void init(float2*, int) {}
  __device__ __forceinline__ void preload(int64_t rs, int nr, int lane) {
    if (resid && lane < nr) nres = resid[rs + lane];
  }
  __device__ __forceinline__ void rotate() { cres = nres; }
  __device__ __forceinline__ void apply(int64_t r, float a, float) { y[r] = resid ? a + cres : a; }
  __device__ __forceinline__ void finish(int) {}
};

// QKV with RoPE (adjacent pairs, angle pos * theta^(-2i/D), cos and sin formed
// in fp64 once per kernel into a shared table) and the k, v store into the
// fp16 caches at row pos.
struct EpiQKV {
  float* q_out;
  uint16_t* k_cache;
  uint16_t* v_cache;
  const int* pos_dev;  // if non-null, pos = *pos_dev
  int pos;
  int64_t nq, nkv;
  int head_dim, max_ctx;
  float theta;
  const float2* cs;  // shared: (cos, sin) of pair i
  int* status = nullptr;  // bounds-check record (debug build)
  static constexpr int kAlign = 2;
  __device__ __forceinline__ void init(float2* esm, int lane) {
    if (pos_dev) pos = *pos_dev;
    for (int i = lane; i < head_dim / 2; i += 32) {
      const double inv_freq = pow((double)theta, -2.0 * (double)i / (double)head_dim);
      double sn, cn;
      sincos((double)pos * inv_freq, &sn, &cn);
      esm[i] = make_float2((float)cn, (float)sn);
    }
    cs = esm;
    __syncwarp();
  }
  __device__ __forceinline__ void preload(int64_t, int, int) {}
  __device__ __forceinline__ void rotate() {}
  __device__ __forceinline__ void apply(int64_t r, float a, float b) {
    const int64_t i2 = r % head_dim;  // even index within the head
    if (r < nq + nkv) {
      const float2 t = cs[i2 >> 1];
      const float ra = a * t.x - b * t.y, rb = a * t.y + b * t.x;
      a = ra;
      b = rb;
    }
    if (r < nq) {
      *reinterpret_cast<float2*>(q_out + r) = make_float2(a, b);
    } else {
      const bool is_k = r < nq + nkv;
      const int64_t kr = is_k ? r - nq : r - nq - nkv;
      const int64_t head = kr / head_dim;
      if (!chk(status, kChkKvAppendOp, pos, max_ctx)) return;  // (debug build) no append past the cache
      uint16_t* cache = is_k ? k_cache : v_cache;
      const uint32_t packed = (uint32_t)float_to_half_bits(a) | ((uint32_t)float_to_half_bits(b) << 16);
      *reinterpret_cast<uint32_t*>(cache + (head * max_ctx + pos) * head_dim + i2) = packed;
    }
  }
  __device__ __forceinline__ void finish(int) {}
};

// SwiGLU over interleaved (gate, up) rows: out[i] = silu(g_i) u_i.
struct EpiSwiGLU {
  float* out;
  static constexpr int kAlign = 2;
  __device__ __forceinline__ void init(float2*, int) {}
  __device__ __forceinline__ void preload(int64_t, int, int) {}
  __device__ __forceinline__ void rotate() {}
  __device__ __forceinline__ void apply(int64_t r, float g, float u) { out[r >> 1] = (g / (1.0f + expf(-g))) * u; }
  __device__ __forceinline__ void finish(int) {}
};

// out = v + resid; statistics sum(out^2), sum(hc out), sum(hc^2) where hc is
// the layer input.  hc is read one stage ahead of the store to out, so `out`
// may alias hc (each row is read before it is overwritten).
struct EpiResid {
  float* out;
  const float* resid;
  const float* hc;  // nullable
  float* parts;     // [gridDim.x][4]
  float st0, st1, st2;
  float nres, nhc, cres, chc;
  static constexpr int kAlign = 1;
  __device__ __forceinline__ void init(float2*, int) { st0 = st1 = st2 = 0.f; }
  // L2 loads: inside the persistent decode kernel these rows were written by
  // an earlier phase of the same launch.
  __device__ __forceinline__ void preload(int64_t rs, int nr, int lane) {
    if (lane < nr) {
      nres = __ldcg(resid + rs + lane);
      nhc = hc ? __ldcg(hc + rs + lane) : 0.f;
    }
  }
  __device__ __forceinline__ void rotate() {
    cres = nres;
    chc = nhc;
  }
  __device__ __forceinline__ void apply(int64_t r, float a, float) {
    const float o = a + cres;
    if (hc) {
      st1 = fmaf(chc, o, st1);
      st2 = fmaf(chc, chc, st2);
    }
    st0 = fmaf(o, o, st0);
    out[r] = o;
  }
  __device__ __forceinline__ void finish(int lane) {
    const float a = warp_sum(st0), b = warp_sum(st1), c = warp_sum(st2);
    if (lane == 0) {
      parts[blockIdx.x * 4 + 0] = a;
      parts[blockIdx.x * 4 + 1] = b;
      parts[blockIdx.x * 4 + 2] = c;
    }
  }
};

// Logits store + argmax (ties -> lowest index) into parts[cta*4] (value) and
// parts[cta*4 + 1] (index bits, -1 if the CTA had no rows).
struct EpiArgmax {
  float* y;
  float* parts;
  float best;
  int64_t besti;
  static constexpr int kAlign = 1;
  __device__ __forceinline__ void init(float2*, int) {
    best = -INFINITY;
    besti = INT64_MAX;
  }
  __device__ __forceinline__ void preload(int64_t, int, int) {}
  __device__ __forceinline__ void rotate() {}
  __device__ __forceinline__ void apply(int64_t r, float a, float) {
    if (y) y[r] = a;
    if (a > best || (a == best && r < besti)) { best = a; besti = r; }
  }
  __device__ __forceinline__ void finish(int lane) {
    float b = best;
    int64_t bi = besti;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, b, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > b || (ob == b && oi < bi)) { b = ob; bi = oi; }
    }
    if (lane == 0) {
      parts[blockIdx.x * 4] = b;
      reinterpret_cast<int*>(parts)[blockIdx.x * 4 + 1] = (int)(bi == INT64_MAX ? -1 : bi);
    }
  }
};

// ------------------------------------------------------------- kernel
// Warp-uniform bounded wait on an mbarrier phase: each lane sleeps in the
// hardware try_wait; the warp agrees on the outcome.  False on timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  bool done = mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  const uint64_t t0 = global_ns();
  while (!__all_sync(0xffffffffu, done)) {
    if (!done) done = mbar_try_wait_sleep(bar, parity);
    if (__any_sync(0xffffffffu, !done && global_ns() - t0 > kWaitLimitNs)) break;
  }
  return __all_sync(0xffffffffu, done);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// MAXC: consumer warps the CTA is built for.  With MAXC <= 8 two CTAs fit on
// one SM (registers and shared memory), so the next kernel of a
// programmatic-launch chain can start streaming its weights while this one
// drains.
template <int QT, class Map, class Pro, class Epi, int MAXC>
__global__ void __launch_bounds__((MAXC + 1) * 32, MAXC <= 8 ? 2 : 1)
    gemv_tma_kernel(Map map, Pro pro, Epi epi, int64_t M, int64_t K, GemvPlan p, int* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem;
  uint8_t* xstage_base = smem + (size_t)p.S * p.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(xstage_base + p.xstage_bytes);
  uint64_t* empty = full + p.S;
  float* red = reinterpret_cast<float*>(empty + p.S);  // [S][TR][n_slices]
  float2* esm = reinterpret_cast<float2*>(red + p.S * p.TR * p.n_slices);  // epilogue table, 128 entries
  int* abort_flag = reinterpret_cast<int*>(esm + kEpiTable);

  // rows of this CTA, in units of Epi::kAlign rows
  const int64_t A = Epi::kAlign;
  const int64_t units = (M + A - 1) / A;
  const int64_t r0 = units * blockIdx.x / gridDim.x * A;
  const int64_t r1 = min64(M, units * (blockIdx.x + 1) / gridDim.x * A);
  const int64_t nrows = r1 > r0 ? r1 - r0 : 0;
  const int n_stages = (int)((nrows + p.TR - 1) / p.TR);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], p.NW);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == p.NW) {
    // ---------------------------------------------------------- producer
    const uint64_t policy = l2_evict_first_policy();
    auto issue = [&](int i, int s) {
      const int64_t rs = r0 + (int64_t)i * p.TR;
      const int nr = (int)min64(p.TR, r1 - rs);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(nr * p.row_bytes));
      __syncwarp();
      for (int r = lane; r < nr; r += 32)
        bulk_g2s(ring + (size_t)s * p.stage_bytes + (size_t)r * p.row_bytes, map.row(rs + r), (uint32_t)p.row_bytes,
                 &full[s], policy);
    };
    // Weights do not depend on the previous kernel: start streaming them first,
    // the ring's stages by bulk copy and a window of further stages into L2
    // (so a kernel that became resident while its predecessor drains has its
    // weights on the way before it may read x).
    auto prefetch = [&](int i) {
      const int64_t rs = r0 + (int64_t)i * p.TR;
      const int nr = (int)min64(p.TR, r1 - rs);
      for (int r = lane; r < nr; r += 32) l2_prefetch(map.row(rs + r), (uint32_t)p.row_bytes);
    };
    const int pre = min(p.S, n_stages);
    for (int i = 0; i < pre; ++i) issue(i, i);
    int pf_next = pre;
    for (const int pf_end = min(n_stages, pre + p.pf_stages); pf_next < pf_end; ++pf_next) prefetch(pf_next);
    pdl_launch_dependents();
    pdl_wait();
    epi.init(esm, lane);
    if (n_stages > 0) epi.preload(r0, (int)min64(p.TR, r1 - r0), lane);
    int i = 0, s = 0;
    uint32_t ph = 0;
    for (; i < n_stages; ++i) {
      if (!warp_wait(&empty[s], ph)) break;
      const int64_t rs = r0 + (int64_t)i * p.TR;
      const int nr = (int)min64(p.TR, r1 - rs);
      // 1. this stage's row totals (fixed slice order) into registers
      const float* rd = red + (size_t)s * p.TR * p.n_slices;
      float a = 0.f, b = 0.f;
      const int row_a = Epi::kAlign == 1 ? lane : 2 * lane;
      const bool mine = row_a < nr;
      if (mine) {
        for (int c = 0; c < p.n_slices; ++c) {
          a += rd[row_a * p.n_slices + c];
          if (Epi::kAlign == 2) b += rd[(row_a + 1) * p.n_slices + c];
        }
      }
      __syncwarp();
      // 2. refill the slot before any global-memory epilogue work
      if (i + p.S < n_stages) issue(i + p.S, s);
      if (pf_next < n_stages) prefetch(pf_next++);
      if (++s == p.S) { s = 0; ph ^= 1u; }
      // 3. epilogue; the next stage's inputs are requested first
      epi.rotate();
      if (i + 1 < n_stages) epi.preload(rs + p.TR, (int)min64(p.TR, r1 - rs - p.TR), lane);
      if (mine) epi.apply(rs + row_a, a, b);
    }
    if (i < n_stages) {
      // A wait ran out: record it, stop the consumers, and let the copies
      // already issued land before the CTA's shared memory is released.
      if (lane == 0) {
        atomicExch(status, (int)kStatusTmaTimeout);
        atomicExch(abort_flag, 1);
        const uint64_t t0 = global_ns();
        for (int k = i; k < min(i + p.S, n_stages); ++k)
          while (!mbar_try_wait(&full[k % p.S], (uint32_t)((k / p.S) & 1)))
            if (global_ns() - t0 > kWaitLimitNs) { atomicExch(status, (int)kStatusDrainTimeout); break; }
      }
      __syncwarp();
    }
    epi.finish(lane);
  } else {
    // ---------------------------------------------------------- consumers
    pdl_launch_dependents();
    pdl_wait();
    const int c = warp % p.n_slices, g = warp / p.n_slices;
    const int64_t c0 = (int64_t)c * kSliceCols;
    const int ucols = (int)min64(kSliceCols, K - c0);
    const bool active = lane_active<QT>(lane, ucols);
    pro.setup(lane);
    XRegs<QT> xr;
    if constexpr (qt_float(QT)) {
      if (active) xr.load_direct(pro, c0, ucols, lane);  // fp32 x straight into registers
    } else {
      const XStage xs = xstage_at(xstage_base, K);
      stage_x<QT>(pro, K, xs, warp, p.NW, lane);
      asm volatile("bar.sync 1, %0;" ::"r"(p.NW * 32) : "memory");  // consumer warps only
      if (active) xr.load(xs, c, lane);
    }
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < n_stages; ++i) {
      if (!warp_wait(&full[s], ph)) {
        if (lane == 0) atomicExch(abort_flag, 1);
        break;
      }
      const int64_t rs = r0 + (int64_t)i * p.TR;
      const int nr = (int)min64(p.TR, r1 - rs);
      const uint8_t* st = ring + (size_t)s * p.stage_bytes + (size_t)c * QTraits<QT>::SEG;
      float* rd = red + (size_t)s * p.TR * p.n_slices;
      for (int r = g; r < nr; r += p.n_rg) {
        const bool in = chk(status, kChkGemvRing, (int64_t)(r + 1) * p.row_bytes - 1, p.stage_bytes);
        float v = active && in ? xr.dot(st + (size_t)r * p.row_bytes, lane) : 0.f;
        v = warp_sum(v);
        if (lane == 0 && chk(status, kChkGemvPartial, r * p.n_slices + c, (int64_t)p.TR * p.n_slices))
          rd[r * p.n_slices + c] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == p.S) { s = 0; ph ^= 1u; }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
    }
  }
}

// Host-side plan for a GEMV over rows of row_bytes bytes.  smem budget in
// bytes for the ring; align: 1 or 2 (rows per epilogue unit).
inline GemvPlan make_gemv_plan(int qtype, int64_t K, int align, int smem_budget, int max_consumers) {
  GemvPlan p;
  const int be = qt_block_elems(qtype), bb = qt_block_bytes(qtype);
  p.row_bytes = (int)(K / be * bb);
  p.n_slices = (int)((K + kSliceCols - 1) / kSliceCols);
  int trmax = kStageTarget / p.row_bytes;
  if (trmax < 1) trmax = 1;
  if (trmax > kMaxTR) trmax = kMaxTR;
  int n_rg = max_consumers / p.n_slices;
  if (n_rg < 1) n_rg = 1;
  if (n_rg > trmax) n_rg = trmax;
  int tr = trmax / n_rg * n_rg;
  if (align == 2 && (tr & 1)) {
    if (tr > 1) tr -= 1;
    else tr = 2;
    if (n_rg > tr) n_rg = tr;
    tr = tr / n_rg * n_rg;
    if (tr & 1) { tr = 2; n_rg = n_rg > 2 ? 2 : n_rg; }
  }
  p.TR = tr;
  p.n_rg = n_rg;
  p.NW = p.n_slices * n_rg;
  p.stage_bytes = p.TR * p.row_bytes;
  p.xstage_bytes = qt_float(qtype) ? 0 : (int)((xstage_bytes(qtype, K) + 15) / 16 * 16);
  int S = smem_budget / p.stage_bytes;
  if (S > 8) S = 8;
  if (S < 2) S = 2;
  p.S = S;
  p.pf_stages = kGemvPrefetchBytes / p.stage_bytes;
  return p;
}

inline size_t gemv_smem_bytes(const GemvPlan& p) {
  return (size_t)p.S * p.stage_bytes + p.xstage_bytes + (size_t)p.S * 16 + (size_t)p.S * p.TR * p.n_slices * 4 +
         kEpiTable * 8 + 16;
}

// ------------------------------------------------------------- generic path
// Any K that is a multiple of the block length, any alignment >= 2 bytes:
// one warp per row, lanes stride over blocks, byte loads.  Used only for shapes
// the bulk-copy path cannot take.
template <int QT>
__device__ __forceinline__ float block_dot_generic(const uint8_t* blk, const float* x) {
  if constexpr (qt_kmin(QT)) {
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8)), dmin = half_bits_to_float(blk[2] | (blk[3] << 8));
    const uint8_t* p = blk + 4;
    float s = 0.f;
    for (int j = 0; j < 8; ++j) {
      const int sc = j < 4 ? (p[j] & 63) : ((p[j + 4] & 15) | ((p[j - 4] >> 6) << 4));
      const int mn = j < 4 ? (p[j + 4] & 63) : ((p[j + 4] >> 4) | ((p[j] >> 6) << 4));
      float t = 0.f, sx = 0.f;
      for (int i = 0; i < 32; ++i) {
        const int n = 32 * j + i, c = n >> 6, h = (n >> 5) & 1, l = n & 31;
        int q = (blk[(QT == QT_Q5_K ? 48 : 16) + 32 * c + l] >> (4 * h)) & 15;
        if constexpr (QT == QT_Q5_K) q |= ((blk[16 + l] >> (2 * c + h)) & 1) << 4;
        t = fmaf((float)q, x[n], t);
        sx += x[n];
      }
      s = fmaf(d * (float)sc, t, s);
      s = fmaf(-dmin * (float)mn, sx, s);
    }
    return s;
  } else if constexpr (QT == QT_F16) {
    return half_bits_to_float(blk[0] | (blk[1] << 8)) * x[0];
  } else if constexpr (QT == QT_F32) {
    return __uint_as_float(blk[0] | (blk[1] << 8) | (blk[2] << 16) | ((uint32_t)blk[3] << 24)) * x[0];
  } else if constexpr (QT == QT_Q8_0) {
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    float s = 0.f;
    for (int i = 0; i < 32; ++i) s = fmaf((float)(int8_t)blk[2 + i], x[i], s);
    return d * s;
  } else if constexpr (QT == QT_Q4_0) {
    const float d = half_bits_to_float(blk[0] | (blk[1] << 8));
    float s = 0.f;
    for (int j = 0; j < 16; ++j) {
      s = fmaf((float)((blk[2 + j] & 15) - 8), x[j], s);
      s = fmaf((float)((blk[2 + j] >> 4) - 8), x[j + 16], s);
    }
    return d * s;
  } else {
    const float d = half_bits_to_float(blk[208] | (blk[209] << 8));
    float s = 0.f;
    for (int sub = 0; sub < 16; ++sub) {
      float t = 0.f;
      for (int e = 0; e < 16; ++e) {
        const int n = 16 * sub + e, h = n >> 7, rr = n & 127, g = rr >> 5, l = rr & 31;
        const int byte = blk[64 * h + 32 * (g & 1) + l];
        const int lo = (g < 2) ? (byte & 15) : (byte >> 4);
        const int hi = (blk[128 + 32 * h + l] >> (2 * g)) & 3;
        t = fmaf((float)((lo | (hi << 4)) - 32), x[n], t);
      }
      s = fmaf((float)(int8_t)blk[192 + sub], t, s);
    }
    return d * s;
  }
}

template <int QT>
__global__ void gemv_generic_kernel(const uint8_t* W, int64_t M, int64_t K, const float* x, float* y,
                                    const float* resid) {
  using T = QTraits<QT>;
  const int lane = threadIdx.x & 31;
  const int64_t nb = K / T::BE;
  const int64_t row_bytes = nb * T::BB;
  for (int64_t r = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5); r < M;
       r += (int64_t)gridDim.x * (blockDim.x / 32)) {
    float s = 0.f;
    for (int64_t b = lane; b < nb; b += 32) s += block_dot_generic<QT>(W + r * row_bytes + b * T::BB, x + b * T::BE);
    s = warp_sum(s);
    if (lane == 0) y[r] = resid ? s + resid[r] : s;
  }
}

}  // namespace ntx
