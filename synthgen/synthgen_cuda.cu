/*
 * synthgen_cuda.cu -- device twin of the seeded synthetic-input generator.
 *
 * Benchmark and test infrastructure only.  It writes the same bytes as the
 * host build (synthgen.c) straight into device memory, so multi-gigabyte
 * synthetic models can be made in seconds; tests compare sampled rows of its
 * output with the host build bit for bit.  Every function is a thin grid-stride
 * loop around the shared per-element definitions in sg_core.h.
 */
#include <cuda_runtime.h>

#include "sg_core.h"

namespace {

__global__ void k_fill_f32(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, float* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = sg_normal_f32(seed, tid, (uint64_t)i, mean, sigma);
}

__global__ void k_fill_f16(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = sg_f32_to_f16(sg_normal_f32(seed, tid, (uint64_t)i, mean, sigma));
}

__global__ void k_tokens(uint32_t seed, uint32_t tid, int64_t n, uint32_t V, int32_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = sg_token(seed, tid, (uint64_t)i, V);
}

/* One thread per quantization block. */
template <int QT>
__global__ void k_quant_rows(uint32_t seed, uint32_t tid, int64_t row0, int64_t nrows, int64_t K, double mean,
                             double sigma, uint8_t* out) {
  constexpr int BE = (QT == SG_Q6_K || QT == SG_Q4_K || QT == SG_Q5_K) ? 256 : (QT == SG_F16 || QT == SG_F32) ? 1 : 32;
  constexpr int BB = QT == SG_Q6_K ? 210 : QT == SG_Q4_K ? 144 : QT == SG_Q5_K ? 176 : QT == SG_Q8_0 ? 34
                   : QT == SG_Q4_0 ? 18 : QT == SG_F16 ? 2 : 4;
  const int64_t nb = K / BE;
  const int64_t total = nrows * nb;
  float w[BE];
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = row0 + g / nb, b = g % nb;
    const uint64_t base = (uint64_t)r * (uint64_t)K + (uint64_t)(b * BE);
    for (int i = 0; i < BE; ++i) w[i] = sg_normal_f32(seed, tid, base + (uint64_t)i, mean, sigma);
    sg_quant_block(QT, w, out + g * BB);
  }
}

int grid_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  if (g > 148 * 64) g = 148 * 64;
  return g < 1 ? 1 : (int)g;
}

}  // namespace

extern "C" {

int sgc_fill_f32(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, float* out, void* stream) {
  if (n <= 0) return 0;
  k_fill_f32<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(seed, tid, n, mean, sigma, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

int sgc_fill_f16(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, uint16_t* out, void* stream) {
  if (n <= 0) return 0;
  k_fill_f16<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(seed, tid, n, mean, sigma, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

int sgc_fill_tokens(uint32_t seed, uint32_t tid, int64_t n, uint32_t V, int32_t* out, void* stream) {
  if (n <= 0) return 0;
  k_tokens<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(seed, tid, n, V, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

/* Same contract as the host sg_quant_rows; `out` is device memory. */
int sgc_quant_rows(int qtype, uint32_t seed, uint32_t tid, int64_t row0, int64_t nrows, int64_t K, double mean,
                   double sigma, uint8_t* out, void* stream) {
  const int be = sg_block_elems(qtype);
  if (be == 0 || K <= 0 || K % be) return -1;
  const int64_t total = nrows * (K / be);
  if (total <= 0) return 0;
  cudaStream_t s = (cudaStream_t)stream;
  switch (qtype) {
    case SG_Q8_0:
      k_quant_rows<SG_Q8_0><<<grid_for(total, 128), 128, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    case SG_Q4_0:
      k_quant_rows<SG_Q4_0><<<grid_for(total, 128), 128, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    case SG_Q6_K:
      k_quant_rows<SG_Q6_K><<<grid_for(total, 64), 64, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    case SG_Q4_K:
      k_quant_rows<SG_Q4_K><<<grid_for(total, 64), 64, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    case SG_Q5_K:
      k_quant_rows<SG_Q5_K><<<grid_for(total, 64), 64, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    case SG_F16:
      k_quant_rows<SG_F16><<<grid_for(total, 256), 256, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
    default:
      k_quant_rows<SG_F32><<<grid_for(total, 256), 256, 0, s>>>(seed, tid, row0, nrows, K, mean, sigma, out);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // extern "C"
