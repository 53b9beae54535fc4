// common.cuh -- device helpers shared by the libntx kernels (sm_100a).
//
// Bulk-copy (TMA 1-D) + mbarrier pipelines, programmatic dependent launch, and
// bounded waits.  Every wait in these kernels has a time limit; a kernel that
// runs out records a code in the device status word and returns instead of
// hanging.  No multicast form of any copy is used anywhere in libntx.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ntx {

// Device status word (read and cleared by ntx_device_status()).
enum : int {
  kStatusOk = 0,
  kStatusTmaTimeout = 1,
  // A copy warp that gave up still lets its issued bulk copies land before
  // the CTA exits (a second bounded wait).  If that wait runs out too, copies
  // issued two seconds earlier have not arrived: the memory system has stopped
  // delivering, the CTA exits with them outstanding, and the context must be
  // treated as lost (no further launches on it).
  kStatusDrainTimeout = 2,
  kStatusBadToken = 3,
  kStatusGridTimeout = 4,  // a grid-wide barrier of the persistent decode kernel ran out
};

// Bounds checks of a debug build (compiled with NTX_CHECK): chk() is true
// when i lies in [0, n); otherwise it records the first failing site and
// index after the status word (status[1], status[2..3]) and returns false, and
// the caller skips the access.  It never traps.  In the release build it is
// always true and compiles to nothing.  Sites:
enum : int {
  kChkRingRead = 1,      // persistent kernel: a consumer's row inside its weight slot
  kChkPartialWrite = 2,  // persistent kernel: a row partial inside its partial slot
  kChkPartialRead = 3,   // persistent kernel: the epilogue's read of a row partial
  kChkKvAppend = 4,      // persistent kernel: the KV cache position this step appends
  kChkKvTile = 5,        // persistent kernel: attention K/V tile copy (positions, tile bytes)
  kChkAttnOut = 6,       // persistent kernel: attention output and split-partial stores
  kChkXStage = 7,        // persistent kernel: x staging stores
  kChkSlotWrite = 8,     // persistent kernel: the copy warp's rows inside a slot
  kChkGemvRing = 9,      // per-op GEMV: a consumer's row inside its stage
  kChkGemvPartial = 10,  // per-op GEMV: row partials
  kChkAttnCtx = 11,      // per-op attention: the step's context inside the cache
  kChkKvAppendOp = 12,   // per-op Q/K/V epilogue: the KV cache position it appends
};
#ifdef NTX_CHECK
constexpr bool kCheck = true;
#else
constexpr bool kCheck = false;
#endif
__device__ __forceinline__ bool chk(int* status, int site, int64_t i, int64_t n) {
  if constexpr (!kCheck) {
    return true;
  } else {
    if (i >= 0 && i < n) return true;
    if (status && atomicCAS(status + 1, 0, site) == 0) {
      atomicExch(status + 2, (int)(uint32_t)(uint64_t)i);
      atomicExch(status + 3, (int)(uint32_t)((uint64_t)i >> 32));
    }
    return false;
  }
}

// Limit on any single wait (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about 1 ms passes, instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most
// kWaitLimitNs.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// L2 policy for streamed-once weights: evict first, keep activations and the
// KV cache resident.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_nohint(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Bulk prefetch into L2 (16-byte aligned address, size a multiple of 16); no
// completion to wait for.
__device__ __forceinline__ void l2_prefetch(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: allow the next kernel in the stream to be
// scheduled, and wait for the previous one's results.  Both are no-ops when
// the kernel was not launched with the programmatic-serialisation attribute.
// Every kernel of a PDL chain executes pdl_wait() in every CTA before it exits
// (so that completion of a kernel implies completion of its predecessors).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16 & 0xFFFFu)));
}

__device__ __forceinline__ uint16_t float_to_half_bits(float v) { return __half_as_ushort(__float2half_rn(v)); }

// fp32 value of byte `b` of w when the byte holds u in [0,255]: 2^23 + u.
template <int B>
__device__ __forceinline__ float magic_byte(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7440u | B));
}

__device__ __forceinline__ float4 ldg4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Deterministic sum of n floats by one warp (lane-strided partial sums, then a
// fixed butterfly); every lane returns the same value.
__device__ __forceinline__ float warp_sum_array(const float* p, int n, int stride, int lane) {
  float s = 0.f;
  for (int i = lane; i < n; i += 32) s += p[(int64_t)i * stride];
  return warp_sum(s);
}

}  // namespace ntx
