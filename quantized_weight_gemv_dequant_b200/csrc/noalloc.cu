// noalloc.cu -- ntx_attn_decode_static: split-KV decode attention whose
// per-split partial results live in a fixed device array inside libntx, so the
// call needs no workspace and allocates nothing.
//
// Who needs it: callers that cannot hand libntx a scratch buffer at the point
// of the call -- a host whose device memory is entirely owned by another
// allocator with a fixed budget, a plain C program with no allocator of its
// own on that path, or a latency-critical thread that must not take an
// allocator's lock or wait on its implicit synchronisation.  cudaMalloc,
// cudaFree and every allocating library routine are never called here.
//
// The array is a file-scope static __device__ buffer of kStaticScratchBytes
// (2 MiB): every GPU that loads libntx holds one copy until the process exits.
// In host code the array's name is not a device address; the first call on a
// device (with that device current) looks the address up with
// cudaGetSymbolAddress and caches it, so that first call should come before
// any stream capture.  Later calls read the cached address with one atomic
// load and take no lock.  The cache lives as long as the process: after
// cudaDeviceReset on a device the module is loaded again, possibly at another
// address, so this call must not be used on that device after a reset.  All
// calls on a device share the one array and it keeps the contents of the last
// call: calls that overlap on the GPU (for example on two streams) race on it.
// Nothing in it needs to start at zero: the split kernel writes every (head,
// split) partial the combine kernel reads.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "launch.h"
#include "ntx.h"

namespace ntx {
namespace {

constexpr size_t kStaticScratchBytes = 2u << 20;
constexpr int kPartStride = 130;  // floats per (query head, split) partial: o[128], m, l
constexpr size_t kStaticScratchFloats = kStaticScratchBytes / sizeof(float);

static __device__ __align__(256) float g_attn_static_scratch[kStaticScratchFloats];

constexpr int kMaxDev = 64;
std::atomic<float*> g_scratch_ptr[kMaxDev];
std::mutex g_scratch_mu;  // taken only by the first lookup on a device

// Device address of the static scratch for the current device (looked up once
// per device), or nullptr with *err set.
float* static_scratch(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDev) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  float* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> g(g_scratch_mu);
  p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (!p) {
    void* a = nullptr;
    *err = cudaGetSymbolAddress(&a, g_attn_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    p = static_cast<float*>(a);
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace
}  // namespace ntx

extern "C" int ntx_attn_decode_static(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out,
                                      int n_q_heads, int n_kv_heads, int head_dim, int n_ctx, int max_ctx,
                                      void* stream) {
  using namespace ntx;
  if (head_dim != 128) return record_error(NTX_ERR_SHAPE, "ntx_attn_decode_static: head_dim must be 128");
  if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads)
    return record_error(NTX_ERR_SHAPE, "ntx_attn_decode_static: n_q_heads must be a multiple of n_kv_heads");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return record_error(NTX_ERR_SHAPE, "ntx_attn_decode_static: query group must be 1, 2, 4 or 8");
  if (n_ctx < 1 || n_ctx > max_ctx) return record_error(NTX_ERR_SHAPE, "ntx_attn_decode_static: n_ctx outside [1, max_ctx]");
  if (!q || !k_cache || !v_cache || !out) return record_error(NTX_ERR_INVALID_ARG, "ntx_attn_decode_static: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return record_error(NTX_ERR_ALIGN, "ntx_attn_decode_static: q and the caches must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(out) & 3)
    return record_error(NTX_ERR_ALIGN, "ntx_attn_decode_static: out must be 4-byte aligned");
  const int n_split = attn_splits(n_kv_heads, n_ctx);
  const size_t need = (size_t)n_q_heads * n_split * kPartStride;
  if (need > kStaticScratchFloats)
    return record_error(NTX_ERR_NOMEM, "ntx_attn_decode_static: needs more scratch than the 2 MiB static array "
                                       "(n_q_heads x splits x 130 floats must be <= 524288)");
  cudaError_t err = cudaSuccess;
  float* part = static_scratch(&err);
  if (!part) return record_cuda_error(err, "ntx_attn_decode_static: cudaGetSymbolAddress");
  // the split-KV and combine kernels of ntx_attn_decode, with the partials in the static array
  err = launch_attn(q, k_cache, v_cache, out, part, n_q_heads, n_kv_heads, n_ctx, nullptr, max_ctx, n_split,
                    static_cast<cudaStream_t>(stream), false);
  if (err != cudaSuccess) return record_cuda_error(err, "ntx_attn_decode_static");
  return NTX_OK;
}
