// attn.cuh -- split-KV grouped-query decode attention over an fp16 KV cache.
//
// ("NTransformer" -- 主な機能: GQA, KV cache; アーキテクチャ概要: softmax.)
// For query head h, KV head g = h / G (G = Hq / Hkv):
//   out_h = sum_{p < n_ctx} softmax_p(q_h . k_p / sqrt(D)) v_p.
// Decode reads each KV head once for its G query heads.  Positions are split
// over `n_split` CTAs per KV head (so n_split * Hkv CTAs cover the SMs even at
// batch 1); each CTA writes (max score m, sum of exp l, unnormalised output o)
// per query head, and a combine kernel merges the splits with the log-sum-exp
// rule out = sum_s o_s e^(m_s - M) / sum_s l_s e^(m_s - M), M = max_s m_s.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace ntx {

constexpr int kAttnD = 128;      // head_dim
constexpr int kAttnWarps = 4;    // warps per split CTA
constexpr int kAttnMaxChunk = 256;  // positions per split CTA at most

__host__ __device__ inline int attn_part_stride() { return kAttnD + 2; }

template <int G>
__global__ void __launch_bounds__(kAttnWarps * 32)
    attn_split_kernel(const float* __restrict__ q, const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
                      float* __restrict__ part, int n_ctx_host, const int* pos_dev, int max_ctx, int n_split,
                      int* status) {
  __shared__ float s_sc[G][kAttnMaxChunk];
  __shared__ float s_o[kAttnWarps][G][kAttnD];
  __shared__ float s_ml[G][2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, kvh = blockIdx.y;

  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = pos_dev ? *pos_dev + 1 : n_ctx_host;
  if (!chk(status, kChkAttnCtx, n_ctx - 1, max_ctx)) n_ctx = 0;  // (debug build) read nothing past the cache
  const int chunk = (n_ctx + n_split - 1) / n_split;
  const int p0 = split * chunk;
  const int p1 = min(p0 + chunk, n_ctx);
  const int np = p1 > p0 ? p1 - p0 : 0;

  // q of the G heads: lane holds elements 4 lane .. 4 lane + 3
  float qr[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float4 t = ldg4(q + (int64_t)(kvh * G + h) * kAttnD + 4 * lane);
    qr[h][0] = t.x; qr[h][1] = t.y; qr[h][2] = t.z; qr[h][3] = t.w;
  }
  const float scale = 0.08838834764831845f;  // 1 / sqrt(128)
  const uint16_t* kbase = kc + (int64_t)kvh * max_ctx * kAttnD;
  const uint16_t* vbase = vc + (int64_t)kvh * max_ctx * kAttnD;

  // scores: one warp per position, lanes split the head dimension
  for (int i = warp; i < np; i += kAttnWarps) {
    const uint2 kr = __ldg(reinterpret_cast<const uint2*>(kbase + (int64_t)(p0 + i) * kAttnD + 4 * lane));
    const float k0 = half_bits_to_float(kr.x), k1 = half_bits_to_float(kr.x >> 16);
    const float k2 = half_bits_to_float(kr.y), k3 = half_bits_to_float(kr.y >> 16);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float s = qr[h][0] * k0;
      s = fmaf(qr[h][1], k1, s);
      s = fmaf(qr[h][2], k2, s);
      s = fmaf(qr[h][3], k3, s);
      s = warp_sum(s);
      if (lane == 0) s_sc[h][i] = s * scale;
    }
  }
  __syncthreads();

  // per head: max, exp, sum (warp h % kAttnWarps owns head h)
  for (int h = warp; h < G; h += kAttnWarps) {
    float m = -INFINITY;
    for (int i = lane; i < np; i += 32) m = fmaxf(m, s_sc[h][i]);
    m = warp_max(m);
    float l = 0.f;
    for (int i = lane; i < np; i += 32) {
      const float e = expf(s_sc[h][i] - m);
      s_sc[h][i] = e;
      l += e;
    }
    l = warp_sum(l);
    if (lane == 0) { s_ml[h][0] = m; s_ml[h][1] = l; }
  }
  __syncthreads();

  // P V: lanes split the head dimension, warps split positions
  float o[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
  for (int i = warp; i < np; i += kAttnWarps) {
    const uint2 vr = __ldg(reinterpret_cast<const uint2*>(vbase + (int64_t)(p0 + i) * kAttnD + 4 * lane));
    const float v0 = half_bits_to_float(vr.x), v1 = half_bits_to_float(vr.x >> 16);
    const float v2 = half_bits_to_float(vr.y), v3 = half_bits_to_float(vr.y >> 16);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float e = s_sc[h][i];
      o[h][0] = fmaf(e, v0, o[h][0]);
      o[h][1] = fmaf(e, v1, o[h][1]);
      o[h][2] = fmaf(e, v2, o[h][2]);
      o[h][3] = fmaf(e, v3, o[h][3]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int t = 0; t < 4; ++t) s_o[warp][h][4 * lane + t] = o[h][t];
  __syncthreads();

  const int S = attn_part_stride();
  for (int idx = threadIdx.x; idx < G * kAttnD; idx += blockDim.x) {
    const int h = idx / kAttnD, d = idx % kAttnD;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) s += s_o[w][h][d];
    float* dst = part + ((int64_t)(kvh * G + h) * n_split + split) * S;
    dst[2 + d] = s;
    if (d == 0) {
      dst[0] = np > 0 ? s_ml[h][0] : -INFINITY;
      dst[1] = np > 0 ? s_ml[h][1] : 0.f;
    }
  }
}

// One CTA of 128 threads per query head.
__global__ void __launch_bounds__(kAttnD) attn_combine_kernel(const float* __restrict__ part, float* __restrict__ out,
                                                              int n_split) {
  pdl_launch_dependents();
  pdl_wait();
  const int h = blockIdx.x, d = threadIdx.x;
  const int S = attn_part_stride();
  const float* ph = part + (int64_t)h * n_split * S;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, ph[s * S]);
  float L = 0.f, O = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float m = ph[s * S];
    if (m == -INFINITY) continue;
    const float w = expf(m - M);
    L = fmaf(ph[s * S + 1], w, L);
    O = fmaf(ph[s * S + 2 + d], w, O);
  }
  out[(int64_t)h * kAttnD + d] = O / L;
}

// Fused variant for clusters: grid (CS, Hkv) with a cluster of CS CTAs per KV
// head.  Each CTA computes its chunk's (m, l, o) for the G query heads into
// its own shared memory; after a cluster barrier, CTA r combines query head
// h = r, r + CS, ... by reading every peer's partial through distributed
// shared memory, and writes out_h.  A second cluster barrier keeps every
// CTA's shared memory alive until all reads are done.  Every CTA reaches both
// barriers on every path.
template <int G>
__global__ void __launch_bounds__(kAttnWarps * 32)
    attn_cluster_kernel(const float* __restrict__ q, const uint16_t* __restrict__ kc,
                        const uint16_t* __restrict__ vc, float* __restrict__ out, int n_ctx_host, const int* pos_dev,
                        int max_ctx, int* status) {
  namespace cg = cooperative_groups;
  __shared__ float s_sc[G][kAttnMaxChunk];
  __shared__ float s_o[kAttnWarps][G][kAttnD];
  __shared__ float s_part[G][kAttnD + 2];  // this CTA's (o[128], m, l) per head
  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int kvh = blockIdx.y;

  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = pos_dev ? *pos_dev + 1 : n_ctx_host;
  if (!chk(status, kChkAttnCtx, n_ctx - 1, max_ctx)) n_ctx = 0;  // (debug build) read nothing past the cache
  const int chunk = (n_ctx + CS - 1) / CS;
  const int p0 = rank * chunk;
  const int p1 = min(p0 + chunk, n_ctx);
  const int np = p1 > p0 ? p1 - p0 : 0;

  float qr[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float4 t = ldg4(q + (int64_t)(kvh * G + h) * kAttnD + 4 * lane);
    qr[h][0] = t.x; qr[h][1] = t.y; qr[h][2] = t.z; qr[h][3] = t.w;
  }
  const float scale = 0.08838834764831845f;  // 1 / sqrt(128)
  const uint16_t* kbase = kc + (int64_t)kvh * max_ctx * kAttnD;
  const uint16_t* vbase = vc + (int64_t)kvh * max_ctx * kAttnD;

  // scores: one warp per position (two positions in flight), lanes split the head dimension
  int i = warp;
  for (; i + kAttnWarps < np; i += 2 * kAttnWarps) {
    const uint2 ka = __ldg(reinterpret_cast<const uint2*>(kbase + (int64_t)(p0 + i) * kAttnD + 4 * lane));
    const uint2 kb = __ldg(reinterpret_cast<const uint2*>(kbase + (int64_t)(p0 + i + kAttnWarps) * kAttnD + 4 * lane));
    const float a0 = half_bits_to_float(ka.x), a1 = half_bits_to_float(ka.x >> 16);
    const float a2 = half_bits_to_float(ka.y), a3 = half_bits_to_float(ka.y >> 16);
    const float b0 = half_bits_to_float(kb.x), b1 = half_bits_to_float(kb.x >> 16);
    const float b2 = half_bits_to_float(kb.y), b3 = half_bits_to_float(kb.y >> 16);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float sa = qr[h][0] * a0, sb = qr[h][0] * b0;
      sa = fmaf(qr[h][1], a1, sa); sb = fmaf(qr[h][1], b1, sb);
      sa = fmaf(qr[h][2], a2, sa); sb = fmaf(qr[h][2], b2, sb);
      sa = fmaf(qr[h][3], a3, sa); sb = fmaf(qr[h][3], b3, sb);
      sa = warp_sum(sa);
      sb = warp_sum(sb);
      if (lane == 0) { s_sc[h][i] = sa * scale; s_sc[h][i + kAttnWarps] = sb * scale; }
    }
  }
  for (; i < np; i += kAttnWarps) {
    const uint2 kr = __ldg(reinterpret_cast<const uint2*>(kbase + (int64_t)(p0 + i) * kAttnD + 4 * lane));
    const float k0 = half_bits_to_float(kr.x), k1 = half_bits_to_float(kr.x >> 16);
    const float k2 = half_bits_to_float(kr.y), k3 = half_bits_to_float(kr.y >> 16);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float sc = qr[h][0] * k0;
      sc = fmaf(qr[h][1], k1, sc);
      sc = fmaf(qr[h][2], k2, sc);
      sc = fmaf(qr[h][3], k3, sc);
      sc = warp_sum(sc);
      if (lane == 0) s_sc[h][i] = sc * scale;
    }
  }
  __syncthreads();

  for (int h = warp; h < G; h += kAttnWarps) {
    float m = -INFINITY;
    for (int j = lane; j < np; j += 32) m = fmaxf(m, s_sc[h][j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < np; j += 32) {
      const float e = expf(s_sc[h][j] - m);
      s_sc[h][j] = e;
      l += e;
    }
    l = warp_sum(l);
    if (lane == 0) { s_part[h][kAttnD] = np > 0 ? m : -INFINITY; s_part[h][kAttnD + 1] = np > 0 ? l : 0.f; }
  }
  __syncthreads();

  float o[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
  for (int j = warp; j < np; j += kAttnWarps) {
    const uint2 vr = __ldg(reinterpret_cast<const uint2*>(vbase + (int64_t)(p0 + j) * kAttnD + 4 * lane));
    const float v0 = half_bits_to_float(vr.x), v1 = half_bits_to_float(vr.x >> 16);
    const float v2 = half_bits_to_float(vr.y), v3 = half_bits_to_float(vr.y >> 16);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float e = s_sc[h][j];
      o[h][0] = fmaf(e, v0, o[h][0]);
      o[h][1] = fmaf(e, v1, o[h][1]);
      o[h][2] = fmaf(e, v2, o[h][2]);
      o[h][3] = fmaf(e, v3, o[h][3]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int t = 0; t < 4; ++t) s_o[warp][h][4 * lane + t] = o[h][t];
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * kAttnD; idx += blockDim.x) {
    const int h = idx / kAttnD, d = idx % kAttnD;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) sum += s_o[w][h][d];
    s_part[h][d] = sum;
  }
  cluster.sync();  // every CTA's partial is complete and visible cluster-wide

  for (int h = rank; h < G; h += CS) {
    const int d = threadIdx.x;  // blockDim.x == kAttnD
    float M = -INFINITY;
    for (int r = 0; r < CS; ++r) M = fmaxf(M, cluster.map_shared_rank(&s_part[h][kAttnD], r)[0]);
    float L = 0.f, O = 0.f;
    for (int r = 0; r < CS; ++r) {
      const float* pr = cluster.map_shared_rank(&s_part[h][0], r);
      const float m = pr[kAttnD];
      if (m == -INFINITY) continue;
      const float w = expf(m - M);
      L = fmaf(pr[kAttnD + 1], w, L);
      O = fmaf(pr[d], w, O);
    }
    out[(int64_t)(kvh * G + h) * kAttnD + d] = O / L;
  }
  cluster.sync();  // peers' shared memory stays alive until every read is done
}

}  // namespace ntx
