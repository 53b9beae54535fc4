// kernels.cu -- instantiation and launch of every libntx kernel (sm_100a).
#include <mutex>
#include <type_traits>
#include <utility>

#include "attn.cuh"
#include "common.cuh"
#include "gemv.cuh"
#include "launch.h"
#include "ops.cuh"

namespace ntx {

// [0] the device status word; [1..3] the bounds-check record of a build with
// NTX_CHECK defined (site, index low and high words), 0 otherwise.
__device__ int g_status[4] = {0, 0, 0, 0};

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
int g_cps = 1;
bool g_gemv_pdl = false;
std::mutex g_mu;

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int* status_ptr() {
  static int* ptrs[kMaxDevices];
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  if (!ptrs[d]) {
    std::lock_guard<std::mutex> g(g_mu);
    if (!ptrs[d]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_status) == cudaSuccess) ptrs[d] = static_cast<int*>(p);
    }
  }
  return ptrs[d];
}

}  // namespace

int* device_status_ptr() { return status_ptr(); }

namespace {

// Raise the dynamic shared-memory limit of a kernel once per device; `done`
// is a per-kernel bit set (one bit per device).
template <class K>
cudaError_t ensure_smem(K kern, size_t bytes, unsigned long long& done) {
  const int d = current_device();
  if (bytes <= 48 * 1024) return cudaSuccess;
  if (done & (1ull << d)) return cudaSuccess;
  std::lock_guard<std::mutex> g(g_mu);
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done |= 1ull << d;
  return e;
}

template <class... KArgs, class... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int grid_1d(int64_t n, int threads, int cap) {
  int64_t g = (n + threads - 1) / threads;
  if (g > cap) g = cap;
  return g < 1 ? 1 : (int)g;
}

#ifndef NTX_GEMV_RING_BYTES
#define NTX_GEMV_RING_BYTES (150 * 1024)
#endif
#ifndef NTX_GEMV_RING_BYTES_PAIRED
#define NTX_GEMV_RING_BYTES_PAIRED (100 * 1024)
#endif
#ifndef NTX_GEMV_PAIRED
#define NTX_GEMV_PAIRED 0
#endif
constexpr int kRingBudget = NTX_GEMV_RING_BYTES;           // one CTA per SM
constexpr int kRingBudgetPaired = NTX_GEMV_RING_BYTES_PAIRED;  // two CTAs per SM
constexpr int kPairedConsumers = 8;
constexpr int kSmemMax = 227 * 1024;  // attribute ceiling for every GEMV instantiation

template <int QT, int MAXC, class Map, class Pro, class Epi>
cudaError_t gemv_tma_v(Map map, Pro pro, Epi epi, int64_t M, int64_t K, int grid, cudaStream_t s, bool pdl,
                       int ring) {
  static unsigned long long done = 0;  // unique per instantiation
  auto kern = gemv_tma_kernel<QT, Map, Pro, Epi, MAXC>;
  // the ring gives up what x staging needs beyond the per-CTA ceiling (half the
  // SM's shared memory when two CTAs are to share an SM)
  const int xst = qt_float(QT) ? 0 : (int)((xstage_bytes(QT, K) + 15) / 16 * 16);
  const int cap = MAXC <= 8 ? 112 * 1024 : kSmemMax;
  if (ring > cap - 8192 - xst) ring = cap - 8192 - xst;
  const GemvPlan plan = make_gemv_plan(QT, K, Epi::kAlign, ring, MAXC);
  const size_t smem = gemv_smem_bytes(plan);
  cudaError_t e = ensure_smem(kern, kSmemMax, done);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(grid), dim3((plan.NW + 1) * 32), smem, s, pdl, map, pro, epi, M, K, plan, status_ptr());
}

// Two co-resident CTAs per SM when the K slices fit 8 consumer warps (Q8_0 and
// Q4_0, K <= 16384); one wide CTA per SM otherwise.
template <int QT, class Map, class Pro, class Epi>
cudaError_t gemv_tma(Map map, Pro pro, Epi epi, int64_t M, int64_t K, int grid, cudaStream_t s, bool pdl) {
  if constexpr (QT != QT_Q6_K && NTX_GEMV_PAIRED) {
    const int n_slices = (int)((K + kSliceCols - 1) / kSliceCols);
    if (n_slices <= kPairedConsumers)
      return gemv_tma_v<QT, kPairedConsumers>(map, pro, epi, M, K, grid, s, pdl, kRingBudgetPaired);
  }
  return gemv_tma_v<QT, kMaxConsumers>(map, pro, epi, M, K, grid, s, pdl, kRingBudget);
}

// Calls f(std::integral_constant<int, QT>) for the block type qt (any type the
// GEMV kernels take); cudaErrorInvalidValue for others.
template <class F>
cudaError_t with_qt(int qt, F&& f) {
  switch (qt) {
    case QT_Q8_0: return f(std::integral_constant<int, QT_Q8_0>{});
    case QT_Q4_0: return f(std::integral_constant<int, QT_Q4_0>{});
    case QT_Q6_K: return f(std::integral_constant<int, QT_Q6_K>{});
    case QT_Q4_K: return f(std::integral_constant<int, QT_Q4_K>{});
    case QT_Q5_K: return f(std::integral_constant<int, QT_Q5_K>{});
    case QT_F16: return f(std::integral_constant<int, QT_F16>{});
    case QT_F32: return f(std::integral_constant<int, QT_F32>{});
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  if (!g_sms[d]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) v = 148;
    g_sms[d] = v;
  }
  return g_sms[d];
}

void set_gemv_ctas_per_sm(int cps) { g_cps = cps < 1 ? 1 : (cps > 4 ? 4 : cps); }
int gemv_ctas_per_sm() { return g_cps; }
void set_gemv_pdl(bool on) { g_gemv_pdl = on; }
bool gemv_pdl() { return g_gemv_pdl; }

int gemv_grid(int64_t M, int align) {
  const int64_t units = (M + align - 1) / align;
  const int64_t cap = (int64_t)sm_count() * g_cps;
  return (int)(units < cap ? (units < 1 ? 1 : units) : cap);
}

int attn_splits(int n_kv_heads, int n_ctx) {
  if (n_ctx < 1) n_ctx = 1;
  int s = (2 * sm_count() + n_kv_heads - 1) / n_kv_heads;
  const int need = (n_ctx + kAttnMaxChunk - 1) / kAttnMaxChunk;
  if (s < need) s = need;
  if (s > n_ctx) s = n_ctx;
  return s < 1 ? 1 : s;
}

bool gemv_tma_ok(int qtype, const void* W, int64_t K) {
  if ((reinterpret_cast<uintptr_t>(W) & 15) != 0) return false;
  if (K > (int64_t)kMaxConsumers * kSliceCols) return false;
  if (qtype == QT_Q6_K) return K % 2048 == 0;
  if (qtype == QT_Q8_0 || qtype == QT_Q4_0 || qtype == QT_Q4_K || qtype == QT_Q5_K || qtype == QT_F16 ||
      qtype == QT_F32)
    return K % 256 == 0;
  return false;
}

cudaError_t launch_dequant(int qtype, const void* blocks, float* out, int64_t nblocks, cudaStream_t s) {
  if (nblocks <= 0) return cudaSuccess;
  const uint8_t* b = static_cast<const uint8_t*>(blocks);
  return with_qt(qtype, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    const int g = grid_1d(nblocks, 128, sm_count() * 16);
    dequant_kernel<QT><<<g, 128, 0, s>>>(b, out, nblocks);
    return cudaGetLastError();
  });
}

template <int QT>
static cudaError_t gemv_plain_qt(const void* W, int64_t M, int64_t K, const float* x, float* y, const float* resid,
                                 cudaStream_t s, bool pdl) {
  const uint8_t* w = static_cast<const uint8_t*>(W);
  const int64_t rb = K / QTraits<QT>::BE * QTraits<QT>::BB;
  if (gemv_tma_ok(QT, W, K)) {
    EpiStore epi{y, resid};
    return gemv_tma<QT>(MapSingle{w, rb}, ProPlain{x}, epi, M, K, gemv_grid(M, 1), s, pdl);
  }
  const int g = grid_1d(M, 8, sm_count() * 8);
  gemv_generic_kernel<QT><<<g, 256, 0, s>>>(w, M, K, x, y, resid);
  return cudaGetLastError();
}

cudaError_t launch_gemv(int qtype, const void* W, int64_t M, int64_t K, const float* x, float* y, const float* resid,
                        cudaStream_t s, bool pdl) {
  return with_qt(qtype, [&](auto t) {
    return gemv_plain_qt<decltype(t)::value>(W, M, K, x, y, resid, s, pdl);
  });
}

cudaError_t launch_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, cudaStream_t s) {
  rmsnorm_kernel<<<1, 1024, 0, s>>>(x, w, y, n, eps);
  return cudaGetLastError();
}

cudaError_t launch_rope(float* q, float* k, int nq, int nkv, int head_dim, int pos, float theta, cudaStream_t s) {
  const int64_t total = (int64_t)(nq + nkv) * (head_dim / 2);
  if (total <= 0) return cudaSuccess;
  rope_kernel<<<grid_1d(total, 256, 4096), 256, 0, s>>>(q, k, nq, nkv, head_dim, pos, theta);
  return cudaGetLastError();
}

cudaError_t launch_swiglu(const float* g, const float* u, float* out, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  swiglu_kernel<<<grid_1d(n, 256, sm_count() * 8), 256, 0, s>>>(g, u, out, n);
  return cudaGetLastError();
}

// Read-only HBM stream (a measurement helper, not a step of the decode): each
// thread loads its 16-byte words with streaming (evict-first) loads, four in
// flight, and the sum of all 32-bit words modulo 2^32 goes to *sum, so no load
// can be dropped and the sum shows that every byte was read.
__global__ void __launch_bounds__(256) read_probe_kernel(const uint4* __restrict__ p, uint64_t n16, unsigned* sum) {
  constexpr int U = 4;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  unsigned acc = 0;
  for (; i + (U - 1) * stride < n16; i += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = __ldcs(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) acc += v[u].x + v[u].y + v[u].z + v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(p + i);
    acc += v.x + v.y + v.z + v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(sum, acc);
}

cudaError_t launch_read_probe(const void* buf, uint64_t bytes, unsigned* sum, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(sum, 0, sizeof(unsigned), s);
  if (e != cudaSuccess || bytes == 0) return e;
  read_probe_kernel<<<sm_count() * 8, 256, 0, s>>>(static_cast<const uint4*>(buf), bytes / 16, sum);
  return cudaGetLastError();
}

cudaError_t launch_attn(const float* q, const uint16_t* kc, const uint16_t* vc, float* out, float* part, int Hq,
                        int Hkv, int n_ctx, const int* pos_dev, int max_ctx, int n_split, cudaStream_t s, bool pdl) {
  const int G = Hq / Hkv;
  const dim3 grid(n_split, Hkv);
  const dim3 block(kAttnWarps * 32);
  cudaError_t e;
  switch (G) {
    case 1: e = launch_k(attn_split_kernel<1>, grid, block, 0, s, pdl, q, kc, vc, part, n_ctx, pos_dev, max_ctx, n_split, status_ptr()); break;
    case 2: e = launch_k(attn_split_kernel<2>, grid, block, 0, s, pdl, q, kc, vc, part, n_ctx, pos_dev, max_ctx, n_split, status_ptr()); break;
    case 4: e = launch_k(attn_split_kernel<4>, grid, block, 0, s, pdl, q, kc, vc, part, n_ctx, pos_dev, max_ctx, n_split, status_ptr()); break;
    case 8: e = launch_k(attn_split_kernel<8>, grid, block, 0, s, pdl, q, kc, vc, part, n_ctx, pos_dev, max_ctx, n_split, status_ptr()); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_k(attn_combine_kernel, dim3(Hq), dim3(kAttnD), 0, s, pdl, (const float*)part, out, n_split);
}

template <int G>
static cudaError_t attn_cluster_g(const float* q, const uint16_t* kc, const uint16_t* vc, float* out, int Hkv,
                                  int n_ctx, const int* pos_dev, int max_ctx, int cs, cudaStream_t s, bool pdl) {
  static unsigned long long done = 0;
  auto kern = attn_cluster_kernel<G>;
  const int d = current_device();
  if (!(done & (1ull << d))) {
    std::lock_guard<std::mutex> g(g_mu);
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    done |= 1ull << d;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, Hkv);
  cfg.blockDim = dim3(kAttnWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  int na = 1;
  if (pdl) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, q, kc, vc, out, n_ctx, pos_dev, max_ctx, status_ptr());
}

int attn_cluster_size(int Hq, int Hkv, int n_ctx_max) {
  const int need = (n_ctx_max + kAttnMaxChunk - 1) / kAttnMaxChunk;
  if (need > 16 || Hkv <= 0 || Hq % Hkv) return 0;
  int cs = need > 8 ? 16 : 8;
  // largest cluster the device can co-schedule for this kernel shape
  static int cap[kMaxDevices];
  const int d = current_device();
  if (d >= 0 && d < kMaxDevices && cap[d] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, Hkv);
    cfg.blockDim = dim3(kAttnWarps * 32);
    int v = 0;
    cudaFuncSetAttribute(attn_cluster_kernel<8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (cudaOccupancyMaxPotentialClusterSize(&v, attn_cluster_kernel<8>, &cfg) != cudaSuccess || v < 1) v = 8;
    cudaGetLastError();
    cap[d] = v;
  }
  const int c = (d >= 0 && d < kMaxDevices) ? cap[d] : 8;
  if (cs > c) cs = c >= 8 ? 8 : c;
  if ((int64_t)cs * kAttnMaxChunk < n_ctx_max) return 0;
  return cs;
}

cudaError_t launch_attn_cluster(const float* q, const uint16_t* kc, const uint16_t* vc, float* out, int Hq, int Hkv,
                                int n_ctx, const int* pos_dev, int max_ctx, int cs, cudaStream_t s, bool pdl) {
  switch (Hq / Hkv) {
    case 1: return attn_cluster_g<1>(q, kc, vc, out, Hkv, n_ctx, pos_dev, max_ctx, cs, s, pdl);
    case 2: return attn_cluster_g<2>(q, kc, vc, out, Hkv, n_ctx, pos_dev, max_ctx, cs, s, pdl);
    case 4: return attn_cluster_g<4>(q, kc, vc, out, Hkv, n_ctx, pos_dev, max_ctx, cs, s, pdl);
    case 8: return attn_cluster_g<8>(q, kc, vc, out, Hkv, n_ctx, pos_dev, max_ctx, cs, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

int layer_stats_parts(int64_t H) { return gemv_grid(H, 1); }

template <int QT>
constexpr int64_t row_bytes_of(int64_t K) {
  return K / QTraits<QT>::BE * QTraits<QT>::BB;
}

// One decode layer as a chain of kernels; each GEMV takes its own block type
// (Q/K/V share one, gate/up share one).
cudaError_t launch_layer(const LayerArgs& a, cudaStream_t s, bool pdl) {
  const int64_t nq = a.Hq * a.D, nkv = a.Hkv * a.D;
  cudaError_t e;

  // 1. RMSNorm prologue + Q/K/V GEMV + RoPE + KV append
  e = with_qt(a.qt_qkv, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    ProRms pro{a.hidden, a.attn_norm, a.stats_in, a.n_stats_in, (int)a.H, a.eps, 0.f};
    EpiQKV epi{a.q, a.k_cache, a.v_cache, a.pos_dev, a.pos, nq, nkv, (int)a.D, a.max_ctx, a.theta};
    epi.status = status_ptr();
    const int64_t M = nq + 2 * nkv;
    return gemv_tma<QT>(MapQKV{a.wq, a.wk, a.wv, row_bytes_of<QT>(a.H), nq, nkv}, pro, epi, M, a.H,
                        gemv_grid(M, 2), s, pdl);
  });
  if (e != cudaSuccess) return e;
  // 2. split-KV attention: one cluster per KV head (partials merged through
  //    distributed shared memory), or split + combine kernels for long contexts
  if (a.attn_cluster > 0)
    e = launch_attn_cluster(a.q, a.k_cache, a.v_cache, a.attn_out, (int)a.Hq, (int)a.Hkv, a.pos + 1, a.pos_dev,
                            a.max_ctx, a.attn_cluster, s, pdl);
  else
    e = launch_attn(a.q, a.k_cache, a.v_cache, a.attn_out, a.attn_part, (int)a.Hq, (int)a.Hkv, a.pos + 1, a.pos_dev,
                    a.max_ctx, a.n_split, s, pdl);
  if (e != cudaSuccess) return e;
  // 3. O projection + residual: h1 = h + Wo a   (statistics: sum h1^2)
  e = with_qt(a.qt_o, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    EpiResid epi{a.h1, a.hidden, nullptr, a.stats_o, 0.f, 0.f, 0.f};
    return gemv_tma<QT>(MapSingle{a.wo, row_bytes_of<QT>(nq)}, ProPlain{a.attn_out}, epi, a.H, nq,
                        gemv_grid(a.H, 1), s, pdl);
  });
  if (e != cudaSuccess) return e;
  // 4. RMSNorm prologue + gate/up GEMV + SwiGLU
  if (a.probe_begin && (e = cudaEventRecord(a.probe_begin, s)) != cudaSuccess) return e;
  e = with_qt(a.qt_gu, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    ProRms pro{a.h1, a.ffn_norm, a.stats_o, gemv_grid(a.H, 1), (int)a.H, a.eps, 0.f};
    EpiSwiGLU epi{a.u};
    return gemv_tma<QT>(MapPair{a.wg, a.wu, row_bytes_of<QT>(a.H)}, pro, epi, 2 * a.F, a.H,
                        gemv_grid(2 * a.F, 2), s, pdl);
  });
  if (e != cudaSuccess) return e;
  if (a.probe_end && (e = cudaEventRecord(a.probe_end, s)) != cudaSuccess) return e;
  // 5. down projection + residual + cosine statistics: h = h1 + Wd u
  return with_qt(a.qt_down, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    EpiResid epi{a.hidden, a.h1, a.hidden, a.stats_down, 0.f, 0.f, 0.f};
    return gemv_tma<QT>(MapSingle{a.wd, row_bytes_of<QT>(a.F)}, ProPlain{a.u}, epi, a.H, a.F, gemv_grid(a.H, 1), s,
                        pdl);
  });
}

cudaError_t launch_sumsq(const float* h, int64_t n, float* parts, int nparts, cudaStream_t s, bool pdl) {
  return launch_k(sumsq_kernel, dim3(nparts), dim3(256), 0, s, pdl, h, n, parts);
}

cudaError_t launch_embed(const uint16_t* table, int64_t H, int64_t V, const int* tok_param, const int* tok_state,
                         float* h, float* parts, int nparts, cudaStream_t s, bool pdl) {
  return launch_k(embed_kernel, dim3(nparts), dim3(256), 0, s, pdl, table, H, V, tok_param, tok_state, h, parts,
                  status_ptr());
}

int head_parts(int64_t V) { return gemv_grid(V, 1); }

cudaError_t launch_head(int qtype, const void* W, int64_t V, int64_t H, const float* h, const float* final_norm,
                        const float* stats_in, int n_stats_in, float eps, float* logits, float* arg_parts,
                        cudaStream_t s, bool pdl) {
  return with_qt(qtype, [&](auto t) {
    constexpr int QT = decltype(t)::value;
    ProRms pro{h, final_norm, stats_in, n_stats_in, (int)H, eps, 0.f};
    EpiArgmax epi{logits, arg_parts, 0.f, 0};
    return gemv_tma<QT>(MapSingle{static_cast<const uint8_t*>(W), row_bytes_of<QT>(H)}, pro, epi, V, H,
                        gemv_grid(V, 1), s, pdl);
  });
}

cudaError_t launch_argmax_finalize(const float* parts, int nparts, int* token_state, int* next_token, cudaStream_t s,
                                   bool pdl) {
  return launch_k(argmax_finalize_kernel, dim3(1), dim3(32), 0, s, pdl, parts, nparts, token_state, next_token);
}

cudaError_t launch_cos_finalize(const float* stats, int nparts, const int* layers, int nlayers, int64_t layer_stride,
                                float* cos_out, cudaStream_t s, bool pdl) {
  if (nlayers <= 0) return cudaSuccess;
  return launch_k(cos_finalize_kernel, dim3(1), dim3(256), 0, s, pdl, stats, nparts, layers, nlayers, layer_stride,
                  cos_out);
}

int read_device_status(int* code) {
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return (int)e;
  int v = 0;
  cudaError_t e2 = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e2 != cudaSuccess) return (int)e2;
  const int zero = 0;
  e2 = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
  if (e2 != cudaSuccess) return (int)e2;
  *code = v;
  return 0;
}

int read_check_report(int* site, long long* index) {
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return (int)e;
  int v[4] = {0, 0, 0, 0};
  cudaError_t e2 = cudaMemcpyFromSymbol(v, g_status, sizeof v);
  if (e2 != cudaSuccess) return (int)e2;
  const int zero[3] = {0, 0, 0};
  e2 = cudaMemcpyToSymbol(g_status, zero, sizeof zero, sizeof(int));
  if (e2 != cudaSuccess) return (int)e2;
  *site = v[1];
  *index = (long long)(((unsigned long long)(unsigned)v[3] << 32) | (unsigned)v[2]);
  return 0;
}

}  // namespace ntx
