// ops.cuh -- the small kernels around the GEMVs: dequantisation, RMSNorm,
// RoPE, SwiGLU, embedding lookup, residual statistics, greedy argmax and the
// cosine layer-skip test.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace ntx {

// ------------------------------------------------------------- dequant
// One thread per block.  Q8_0, Q4_0, Q6_K: exact (d * sc * (q - off) fits
// fp32).  Q4_K / Q5_K: d sc q and dmin m are each exact, their difference is
// rounded once (fp32 round to nearest) -- the exact value when it fits fp32.
// F16 / F32: the value.
template <int QT>
__global__ void dequant_kernel(const uint8_t* __restrict__ blocks, float* __restrict__ out, int64_t nblocks) {
  using T = QTraits<QT>;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks; b += (int64_t)gridDim.x * blockDim.x) {
    const uint8_t* p = blocks + b * T::BB;
    float* o = out + b * T::BE;
    if constexpr (qt_kmin(QT)) {
      const float d = half_bits_to_float(p[0] | (p[1] << 8)), dmin = half_bits_to_float(p[2] | (p[3] << 8));
      const uint8_t* sc = p + 4;
      for (int j = 0; j < 8; ++j) {
        const int s = j < 4 ? (sc[j] & 63) : ((sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4));
        const int m = j < 4 ? (sc[j + 4] & 63) : ((sc[j + 4] >> 4) | ((sc[j] >> 6) << 4));
        const float ds = d * (float)s, dm = dmin * (float)m;  // both exact
        for (int i = 0; i < 32; ++i) {
          const int n = 32 * j + i, c = n >> 6, h = (n >> 5) & 1, l = n & 31;
          int q = (p[(QT == QT_Q5_K ? 48 : 16) + 32 * c + l] >> (4 * h)) & 15;
          if constexpr (QT == QT_Q5_K) q |= ((p[16 + l] >> (2 * c + h)) & 1) << 4;
          o[n] = __fmaf_rn(ds, (float)q, -dm);  // one rounding of the exact d sc q - dmin m
        }
      }
    } else if constexpr (QT == QT_F16) {
      o[0] = half_bits_to_float(p[0] | (p[1] << 8));
    } else if constexpr (QT == QT_F32) {
      o[0] = __uint_as_float(p[0] | (p[1] << 8) | (p[2] << 16) | ((uint32_t)p[3] << 24));
    } else if constexpr (QT == QT_Q8_0) {
      const float d = half_bits_to_float(p[0] | (p[1] << 8));
      for (int i = 0; i < 32; ++i) o[i] = d * (float)(int8_t)p[2 + i];
    } else if constexpr (QT == QT_Q4_0) {
      const float d = half_bits_to_float(p[0] | (p[1] << 8));
      for (int j = 0; j < 16; ++j) {
        o[j] = d * (float)((p[2 + j] & 15) - 8);
        o[j + 16] = d * (float)((p[2 + j] >> 4) - 8);
      }
    } else {
      const float d = half_bits_to_float(p[208] | (p[209] << 8));
      for (int n = 0; n < 256; ++n) {
        const int h = n >> 7, r = n & 127, g = r >> 5, l = r & 31;
        const int byte = p[64 * h + 32 * (g & 1) + l];
        const int lo = (g < 2) ? (byte & 15) : (byte >> 4);
        const int hi = (p[128 + 32 * h + l] >> (2 * g)) & 3;
        // d * sc is exact (11 x 8 bits); the product with (q - 32) is exact too
        o[n] = (d * (float)(int8_t)p[192 + n / 16]) * (float)((lo | (hi << 4)) - 32);
      }
    }
  }
}

// ------------------------------------------------------------- RMSNorm
// One CTA: deterministic block reduction of sum(x^2), then y = w (x r).
__global__ void __launch_bounds__(1024) rmsnorm_kernel(const float* x, const float* w, float* y, int64_t n,
                                                       float eps) {
  __shared__ float red[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s = fmaf(x[i], x[i], s);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float r = 1.0f / sqrtf(red[0] / (float)n + eps);
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) y[i] = w[i] * (x[i] * r);
}

// ------------------------------------------------------------- RoPE
// One thread per (head, pair); angle in fp64, rotation in fp32.
__global__ void rope_kernel(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int pos, float theta) {
  const int half = head_dim / 2;
  const int64_t total = (int64_t)(n_q_heads + n_kv_heads) * half;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t head = t / half;
    const int i = (int)(t % half);
    float* v = head < n_q_heads ? q + head * head_dim : k + (head - n_q_heads) * head_dim;
    const double inv_freq = pow((double)theta, -2.0 * i / (double)head_dim);
    double s, c;
    sincos((double)pos * inv_freq, &s, &c);
    const float cf = (float)c, sf = (float)s;
    const float a = v[2 * i], b = v[2 * i + 1];
    v[2 * i] = a * cf - b * sf;
    v[2 * i + 1] = a * sf + b * cf;
  }
}

// ------------------------------------------------------------- SwiGLU
__global__ void swiglu_kernel(const float* g, const float* u, float* out, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float a = g[i];
    out[i] = (a / (1.0f + expf(-a))) * u[i];
  }
}

// ------------------------------------------------------------- statistics
// Per-CTA partial sum(h^2) into parts[cta * 4].
__global__ void __launch_bounds__(256) sumsq_kernel(const float* h, int64_t n, float* parts) {
  __shared__ float red[8];
  pdl_launch_dependents();
  pdl_wait();
  const int64_t per = (n + gridDim.x - 1) / gridDim.x;
  const int64_t i0 = blockIdx.x * per, i1 = min(n, i0 + per);
  float s = 0.f;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += blockDim.x) s = fmaf(h[i], h[i], s);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    parts[blockIdx.x * 4] = t;
  }
}

// Embedding lookup of one token (fp16 row -> fp32) plus sum(h^2) partials.
// token = *tok_param if >= 0, else *tok_state (the previous step's argmax).
// An id outside [0, V) (possible only if the logits were not finite) is
// replaced by 0 and recorded in the status word.
__global__ void __launch_bounds__(256) embed_kernel(const uint16_t* table, int64_t H, int64_t V, const int* tok_param,
                                                    const int* tok_state, float* h, float* parts, int* status) {
  __shared__ float red[8];
  pdl_launch_dependents();
  pdl_wait();
  const int tp = *tok_param;
  int64_t tok = tp >= 0 ? tp : *tok_state;
  if (tok < 0 || tok >= V) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(status, (int)kStatusBadToken);
    tok = 0;
  }
  const int64_t per = (H + gridDim.x - 1) / gridDim.x;
  const int64_t i0 = blockIdx.x * per, i1 = min(H, i0 + per);
  float s = 0.f;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const float v = half_bits_to_float(table[tok * H + i]);
    h[i] = v;
    s = fmaf(v, v, s);
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    parts[blockIdx.x * 4] = t;
  }
}

// Greedy token from per-CTA (value, index) partials; ties -> lowest index.
__global__ void argmax_finalize_kernel(const float* parts, int nparts, int* token_state, int* next_token) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x;
  float b = -INFINITY;
  int bi = 0x7fffffff;
  for (int i = lane; i < nparts; i += 32) {
    const float v = parts[i * 4];
    const int vi = reinterpret_cast<const int*>(parts)[i * 4 + 1];
    if (vi < 0) continue;
    if (v > b || (v == b && vi < bi)) { b = v; bi = vi; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, b, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > b || (ob == b && oi < bi)) { b = ob; bi = oi; }
  }
  if (lane == 0) {
    if (token_state) *token_state = bi;
    if (next_token) *next_token = bi;
  }
}

// Cosine of each listed layer from the down-projection statistics
// (sum h_out^2, sum h_in h_out, sum h_in^2 per CTA):
// cos = <h_in, h_out> / (|h_in| |h_out|).
__global__ void cos_finalize_kernel(const float* stats, int nparts, const int* layers, int nlayers,
                                    int64_t layer_stride, float* cos_out) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  for (int k = threadIdx.x >> 5; k < nlayers; k += blockDim.x >> 5) {
    const int l = layers ? layers[k] : k;
    const float* p = stats + l * layer_stride;
    const float yy = warp_sum_array(p + 0, nparts, 4, lane);
    const float hy = warp_sum_array(p + 1, nparts, 4, lane);
    const float hh = warp_sum_array(p + 2, nparts, 4, lane);
    if (lane == 0) cos_out[l] = hy / (sqrtf(hh) * sqrtf(yy));
  }
}

}  // namespace ntx
