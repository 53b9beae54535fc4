// persist.cu -- one decode step (embed -> L layers -> head -> argmax) as a
// single persistent kernel: one CTA per SM for the whole step.
//
// Why.  Batch-1 decode streams every weight byte once per token ("NTransformer"
// -- アーキテクチャ概要 and "RTX 3090 1枚でLlama 70B" -- VRAMの壁: the GEMV is
// memory bound), so the step can only approach the HBM roofline if the weight
// stream never pauses.  A chain of per-op kernels pauses at every boundary:
// each kernel's CTAs must drain before the next kernel's CTAs (one per SM, up
// to 227 KB of shared memory each) can start copying.  Here the copy warp of
// each CTA walks one continuous list of weight stages across all phases of the
// step; the weights never depend on activations, so it keeps the copy ring full
// while the other warps wait at a phase boundary or compute attention.
//
// Warps of a CTA (16): 14 consumer warps (x staging, dot products, attention),
// one epilogue warp (row sums, phase epilogues, the phase's grid arrival) and
// one copy warp (bulk copies of the weight rows into the ring).
//
// Phases (index p; one grid-wide counter each):
//   0            EMBED  h = fp16 row of the token, sum(h^2) partials
//   1 + 5k + 0   QKV    RMSNorm(h) prologue, q/k/v rows, RoPE, KV append
//   1 + 5k + 1   ATTN   split-KV GQA attention; the splits of a KV head merge
//                       their outputs (log-sum-exp), each split a share
//   1 + 5k + 2   O      h1 = h + Wo a, sum(h1^2) partials
//   1 + 5k + 3   GU     RMSNorm(h1) prologue, u = silu(Wg n) * (Wu n)
//   1 + 5k + 4   DOWN   h = h1 + Wd u, residual and cosine statistics
//   1 + 5n       HEAD   RMSNorm(h) prologue, logits, argmax (the last CTA to
//                       finish picks the token)
// where k runs over the executed layers (a skip set removes layers from the
// list).  A phase's inputs are complete when every CTA has arrived on the
// previous phase's counter: GEMV phases arrive from the epilogue warp after
// its stores, EMBED and ATTN from the consumer warps.  Every wait is bounded
// (%globaltimer) and any CTA that gives up raises a grid-wide abort word, so
// the other CTAs stop waiting too; the copy warp lets its copies in flight
// land before the CTA exits.
//
// GEMV work inside a phase follows gemv_tma_kernel: rows are split evenly over
// the CTAs; consumer warp (c, g) owns K slice c (2048 columns, x in registers)
// and row group g; row-slice partials go through a ring of partial slots in
// shared memory (its own mbarriers) to the epilogue warp, which sums them in a
// fixed order and runs the epilogue.  All phases share one ring of equal-size
// weight slots; each phase fits as many whole rows in a slot as it can (an
// even count where the epilogue pairs rows), and persist_plan picks the slot
// size.
// Data written by an earlier phase of this launch is read through L2
// (ld.global.cg), never through the non-coherent or L1 paths.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "gemv.cuh"
#include "launch.h"
#include "persist.h"

namespace ntx {
namespace {

extern __shared__ __align__(128) uint8_t p_smem[];  // the kernel's dynamic shared memory

constexpr int kPWarps = kPConsumers + 2;  // + epilogue warp + copy warp
constexpr int kPEpiWarp = kPConsumers, kPCopyWarp = kPConsumers + 1;
constexpr int kPThreads = kPWarps * 32;
constexpr int kPCThreads = kPConsumers * 32;
constexpr float kAttnScale = 0.08838834764831845f;  // 1 / sqrt(128)

__device__ __forceinline__ void cons_bar() { asm volatile("bar.sync 1, %0;" ::"r"(kPCThreads) : "memory"); }

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_acq_rel_add(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// One thread: wait until *ctr >= target.  False if the grid-wide abort word is
// raised or the wait runs out (which raises it).
__device__ bool grid_wait(const unsigned* ctr, unsigned target, unsigned* gabort, int* status, uint64_t limit) {
  if (ld_acquire(ctr) >= target) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    __nanosleep(20);
    if (ld_acquire(ctr) >= target) return true;
    if (*reinterpret_cast<volatile unsigned*>(gabort)) return false;
    if (global_ns() - t0 > limit) {
      atomicExch(status, (int)kStatusGridTimeout);
      atomicExch(gabort, 1u);
      return false;
    }
  }
}

// Warp-uniform bounded wait on an mbarrier phase that also gives up when this
// CTA has aborted.
__device__ bool pwait(uint64_t* bar, uint32_t parity, volatile int* cta_abort, uint64_t limit) {
  bool done = mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  const uint64_t t0 = global_ns();
  while (!__all_sync(0xffffffffu, done)) {
    if (!done) done = mbar_try_wait_sleep(bar, parity);
    const bool give_up = *cta_abort || global_ns() - t0 > limit;
    if (__any_sync(0xffffffffu, !done && give_up)) break;
  }
  return __all_sync(0xffffffffu, done);
}

__device__ __forceinline__ int phase_kind(int p, int n) {
  if (p == 0) return PK_EMBED;
  if (p == 1 + 5 * n) return PK_HEAD;
  return PK_QKV + (p - 1) % 5;
}

struct PRows {
  int r0, r1;  // rows [r0, r1) of this CTA (every phase has fewer than 2^31 rows)
  int n;       // stages
};

__device__ __forceinline__ int64_t phase_M(const PStep& st, int kind) {
  switch (kind) {
    case PK_QKV: return (int64_t)(st.Hq + 2 * st.Hkv) * st.D;
    case PK_O: return st.H;
    case PK_GU: return 2 * (int64_t)st.F;
    case PK_DOWN: return st.H;
    default: return st.V;
  }
}
__device__ __forceinline__ int64_t phase_K(const PStep& st, int kind) {
  switch (kind) {
    case PK_O: return (int64_t)st.Hq * st.D;
    case PK_DOWN: return st.F;
    default: return st.H;
  }
}

__device__ __forceinline__ PRows phase_rows(const PStep& st, int kind) {
  const PGeom& g = st.g[kind];
  const int64_t M = phase_M(st, kind), A = g.align;
  const int64_t units = (M + A - 1) / A;
  PRows r;
  r.r0 = (int)(units * blockIdx.x / gridDim.x * A);
  r.r1 = (int)min64(M, units * (blockIdx.x + 1) / gridDim.x * A);
  const int nr = r.r1 > r.r0 ? r.r1 - r.r0 : 0;
  r.n = (nr + g.TR - 1) / g.TR;
  return r;
}

__device__ __forceinline__ const PLayer* phase_layer(const PStep& st, int p) {
  return (p >= 1 && p < 1 + 5 * st.n_layers) ? st.layers + (p - 1) / 5 : nullptr;
}

// Walks the weight stages of this CTA over all phases, in order.  Entering a
// phase loads its matrix base pointers once, so that the source address of a
// row copy is register arithmetic only.
struct PIssue {
  int p, j, n, kind;
  int64_t r0, r1;
  int TR, rb;
  const uint8_t *b0, *b1, *b2;  // QKV: wq, wk, wv; GU: wg, wu; otherwise b0
  int64_t nq, nkv;
  __device__ void seek(const PStep& st, int from, int np) {
    for (p = from; p < np; ++p) {
      kind = phase_kind(p, st.n_layers);
      if (kind == PK_EMBED || kind == PK_ATTN) continue;
      const PRows r = phase_rows(st, kind);
      if (r.n == 0) continue;
      r0 = r.r0; r1 = r.r1; n = r.n; j = 0;
      TR = st.g[kind].TR;
      rb = st.g[kind].row_bytes;
      const PLayer* L = phase_layer(st, p);
      nq = (int64_t)st.Hq * st.D;
      nkv = (int64_t)st.Hkv * st.D;
      b1 = b2 = nullptr;
      switch (kind) {
        case PK_QKV: b0 = L->wq; b1 = L->wk; b2 = L->wv; break;
        case PK_O: b0 = L->wo; break;
        case PK_GU: b0 = L->wg; b1 = L->wu; break;
        case PK_DOWN: b0 = L->wd; break;
        default: b0 = st.head; break;
      }
      return;
    }
  }
  __device__ __forceinline__ const uint8_t* row(int64_t r) const {
    if (kind == PK_QKV) {
      if (r < nq) return b0 + r * rb;
      if (r < nq + nkv) return b1 + (r - nq) * rb;
      return b2 + (r - nq - nkv) * rb;
    }
    if (kind == PK_GU) return ((r & 1) ? b1 : b0) + (r >> 1) * rb;
    return b0 + r * rb;
  }
  __device__ __forceinline__ bool valid(int np) const { return p < np; }
  __device__ __forceinline__ void advance(const PStep& st, int np) {
    if (++j >= n) seek(st, p + 1, np);
  }
};

// x prologue with L2 loads (x was produced by an earlier phase): RMSNorm(h) w
// when a norm weight is given, x itself otherwise.
struct PX {
  const float* h;
  const float* w;  // nullable
  float r;
  __device__ __forceinline__ float4 ld(int64_t j) const {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(h + j));
    if (!w) return a;
    const float4 b = ldg4(w + j);
    return make_float4(b.x * (a.x * r), b.y * (a.y * r), b.z * (a.z * r), b.w * (a.w * r));
  }
};

// Shared-memory carve, identical on host and device.
struct PSmem {
  uint8_t* ring;    // [S][Z] weight slots
  uint8_t* xst;     // x staging / attention scratch
  uint64_t* full;   // [S] weight slot landed (copy warp -> consumers)
  uint64_t* empty;  // [S] weight slot read (consumers -> copy warp)
  uint64_t* rfull;  // [kPRed] row partials written (consumers -> epilogue warp)
  uint64_t* rempty; // [kPRed] row partials read (epilogue warp -> consumers)
  float* red;       // [kPRed][RF] row partials
  float2* rope;     // [64] RoPE (cos, sin) of this step's position
  int* misc;        // [0] CTA abort, [1..2] phase go flags, [3] last-CTA flag
  float* scr;       // [16] reductions
  struct LRow* lt;  // [n_layers] per-layer pointers the consumer and epilogue warps use
  struct KGeo* kg;  // [7] geometry and this CTA's rows per phase kind
};
// Geometry and row range of one GEMV phase kind for this CTA, computed once.
struct KGeo {
  PGeom g;
  PRows rows;
};
// Per-layer pointers copied to shared memory at kernel start, so a phase
// start does not wait for a global load to learn where its inputs are.
struct LRow {
  const float* attn_norm;
  const float* ffn_norm;
  float* stats_down;
  uint16_t* kc;
  uint16_t* vc;
};
__host__ __device__ inline size_t psmem_bytes(int S, int Z, int XB, int RF, int nl) {
  return (size_t)S * Z + XB + (size_t)S * 16 + (size_t)kPRed * 16 + (size_t)kPRed * RF * 4 + 64 * 8 + 16 * 4 +
         16 * 4 + (size_t)nl * sizeof(LRow) + 7 * sizeof(KGeo);
}
__device__ __forceinline__ PSmem psmem_at(uint8_t* base, int S, int Z, int XB, int RF, int nl) {
  PSmem m;
  m.ring = base;
  m.xst = base + (size_t)S * Z;
  m.full = reinterpret_cast<uint64_t*>(m.xst + XB);
  m.empty = m.full + S;
  m.rfull = m.empty + S;
  m.rempty = m.rfull + kPRed;
  m.red = reinterpret_cast<float*>(m.rempty + kPRed);
  m.rope = reinterpret_cast<float2*>(m.red + (size_t)kPRed * RF);
  m.misc = reinterpret_cast<int*>(m.rope + 64);
  m.scr = reinterpret_cast<float*>(m.misc + 16);
  m.lt = reinterpret_cast<LRow*>(m.scr + 16);
  m.kg = reinterpret_cast<KGeo*>(m.lt + nl);
  return m;
}

// Attention scratch inside the x staging region (consumer warps only).
struct AttnSmem {
  uint8_t* k;   // [kPChunk][128] fp16: one tile of K rows
  uint8_t* v;   // [kPChunk][128] fp16: one tile of V rows
  float* sc;    // [G][kPChunk] scores, then exp(score - running max)
  float* ml;    // [G][2] running (max, sum of exp) of the unit
  float* fac;   // [G] rescale factor of the running output for this tile
  float* sw;    // [G][n_split][2] the splits' (max, sum), then (merge weight, sum)
};
__host__ __device__ inline size_t attn_smem_bytes(int G, int ns) {
  return (size_t)2 * kPChunk * kPD * 2 + (size_t)G * kPChunk * 4 + (size_t)G * 3 * 4 + (size_t)G * ns * 8;
}
__device__ __forceinline__ AttnSmem attn_smem(uint8_t* base, int G) {
  AttnSmem a;
  a.k = base;
  a.v = base + kPChunk * kPD * 2;
  a.sc = reinterpret_cast<float*>(a.v + kPChunk * kPD * 2);
  a.ml = a.sc + G * kPChunk;
  a.fac = a.ml + 2 * G;
  a.sw = a.fac + G;
  return a;
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


// mbarrier operations on 32-bit shared-window addresses (keeps loop state small).
__device__ __forceinline__ bool mbar_test_a(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok)
               : "r"(a), "r"(parity)
               : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_sleep_a(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(a), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive_a(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
// pwait on a 32-bit address; cta_abort is the CTA abort word in shared memory.
__device__ bool pwait_a(uint32_t bar, uint32_t parity, const volatile int* cta_abort, uint64_t limit) {
  bool done = mbar_test_a(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  const uint64_t t0 = global_ns();
  while (!__all_sync(0xffffffffu, done)) {
    if (!done) done = mbar_sleep_a(bar, parity);
    const bool give_up = *cta_abort || global_ns() - t0 > limit;
    if (__any_sync(0xffffffffu, !done && give_up)) break;
  }
  return __all_sync(0xffffffffu, done);
}

// ------------------------------------------------------------ copy warp
// Streams every weight stage of this CTA, phase after phase, into the ring.
// It waits only for slots to be released: weights never depend on
// activations, so the stream runs ahead across phase boundaries.
//
// While the ring is full and the warp waits for a slot -- the consumers are at
// a phase boundary, in the attention phase or working through a full ring --
// it requests further stages into L2 (bulk prefetch, no completion to wait
// for), up to pf_stages beyond the ring, so that HBM keeps streaming; those
// stages later come into the ring from L2.  Nothing is prefetched while slots
// turn over as fast as HBM fills them, so the prefetches never compete with
// the ring's own copies.  Each weight byte still crosses HBM once.
struct Copier {
  const PStep& st;
  PSmem sm;
  int lane, np, n_slots, slot_bytes;
  uint64_t policy;
  PIssue it;   // next stage into the ring
  PIssue pit;  // next stage into L2 (at or ahead of it)
  long issued, done, pfn;  // stages issued into the ring; the L2 frontier (stage count)

  __device__ Copier(const PStep& st_, PSmem sm_, int lane_, int np_)
      : st(st_), sm(sm_), lane(lane_), np(np_), issued(0), done(0), pfn(0) {
    n_slots = st.n_slots;
    slot_bytes = st.slot_bytes;
    policy = l2_evict_first_policy();
    it.seek(st, 0, np);
  }

  __device__ __forceinline__ void issue(int slot) {
    const int64_t rs = it.r0 + (int64_t)it.j * it.TR;
    const int nr = (int)min64(it.TR, it.r1 - rs);
    const int rb = it.rb;
    uint64_t* bar = sm.full + slot;
    // (debug build) rows past the slot are not copied; the slot still completes
    const bool in = chk(st.status, kChkSlotWrite, (int64_t)nr * rb - 1, slot_bytes);
    if (lane == 0) mbar_arrive_expect_tx(bar, in ? (uint32_t)(nr * rb) : 0u);
    __syncwarp();
    uint8_t* dst = sm.ring + (size_t)slot * slot_bytes;
    if (in)
      for (int r = lane; r < nr; r += 32) bulk_g2s(dst + (size_t)r * rb, it.row(rs + r), (uint32_t)rb, bar, policy);
    it.advance(st, np);
    ++issued;
    if (pfn < issued) {  // the L2 frontier never trails the ring
      pit = it;
      pfn = issued;
    }
  }

  __device__ __forceinline__ void prefetch_one() {
    const int64_t rs = pit.r0 + (int64_t)pit.j * pit.TR;
    const int nr = (int)min64(pit.TR, pit.r1 - rs);
    for (int r = lane; r < nr; r += 32) l2_prefetch(pit.row(rs + r), (uint32_t)pit.rb);
    pit.advance(st, np);
    ++pfn;
  }

  // Waits (bounded) for slot s to be released, extending the L2 window while
  // it is not.
  __device__ bool wait_slot(int s, uint32_t ph) {
    uint64_t* bar = sm.empty + s;
    bool ok = mbar_try_wait(bar, ph);
    if (__all_sync(0xffffffffu, ok)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
      if (pfn < issued + st.pf_stages && pit.valid(np)) {
        prefetch_one();
        if (!ok) ok = mbar_try_wait(bar, ph);
      } else if (!ok) {
        ok = mbar_try_wait_sleep(bar, ph);
      }
      if (__all_sync(0xffffffffu, ok)) return true;
      const bool give_up = *reinterpret_cast<volatile int*>(sm.misc) || global_ns() - t0 > st.wait_ns;
      if (__any_sync(0xffffffffu, !ok && give_up)) return false;
    }
  }

  // Lets every issued copy land (bounded) before the warp exits.  A copy that
  // has not landed within the wait limit means the memory system is not
  // completing requests; the warp then records kStatusDrainTimeout and
  // returns rather than wait without a bound, so the step is reported failed
  // and its CTA may exit with that copy still outstanding.
  __device__ void drain() {
    if (lane == 0) {
      const uint64_t t0 = global_ns();
      for (long k = done; k < issued; ++k) {
        uint64_t* bar = sm.full + k % n_slots;
        const uint32_t par = (uint32_t)((k / n_slots) & 1);
        while (!mbar_try_wait(bar, par))
          if (global_ns() - t0 > st.wait_ns) { atomicExch(st.status, (int)kStatusDrainTimeout); return; }
      }
    }
    __syncwarp();
  }

  __device__ void run() {
    for (int k = 0; k < n_slots && it.valid(np); ++k) issue(k);
    int s = 0;
    uint32_t ph = 0;
    while (it.valid(np)) {
      if (!wait_slot(s, ph)) {
        if (lane == 0) {
          atomicExch(sm.misc, 1);
          atomicExch(st.sync + st.abort_index, 1u);
        }
        break;
      }
      issue(s);
      ++done;
      if (++s == n_slots) { s = 0; ph ^= 1u; }
    }
    drain();
  }
};

// Residual epilogue for a CTA row range of at most 64 rows: out = v + resid
// with statistics sum(out^2), sum(hc out), sum(hc^2).  resid and hc (the layer
// input) for all of the CTA's rows are loaded once at the phase start, so the
// epilogue warp does not wait on L2 stage by stage; a stage's values are
// picked with shuffles (all lanes call apply_stage).
struct PEpiResid {
  float* out;
  const float* resid;
  const float* hc;  // nullable
  float* parts;     // [gridDim.x][4]
  int r0;
  float rv[2], hv[2];
  float st0, st1, st2;
  __device__ __forceinline__ void begin(int r0_, int r1_, int lane) {
    r0 = r0_;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = r0 + lane + 32 * k;
      rv[k] = i < r1_ ? __ldcg(resid + i) : 0.f;
      hv[k] = (hc && i < r1_) ? __ldcg(hc + i) : 0.f;
    }
    st0 = st1 = st2 = 0.f;
  }
  __device__ __forceinline__ void apply_stage(int rs, bool mine, int lane, float a) {
    const int idx = rs - r0 + lane;  // this lane's row, relative to r0 (< 64 where mine)
    const int src = idx & 31;
    const float ra = __shfl_sync(0xffffffffu, rv[0], src), rb = __shfl_sync(0xffffffffu, rv[1], src);
    const float ha = __shfl_sync(0xffffffffu, hv[0], src), hb = __shfl_sync(0xffffffffu, hv[1], src);
    if (mine) {
      const float res = idx < 32 ? ra : rb, h = idx < 32 ? ha : hb;
      const float o = a + res;
      if (hc) {
        st1 = fmaf(h, o, st1);
        st2 = fmaf(h, h, st2);
      }
      st0 = fmaf(o, o, st0);
      out[rs + lane] = o;
    }
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

// ------------------------------------------------------------ epilogue warp
// Sums each stage's row partials in a fixed slice order, runs the phase's
// epilogue and, at the end of the phase, publishes its outputs to the grid.
struct Epilogue {
  const PStep& st;
  PSmem sm;
  int lane, red_floats;
  int q;  // partial-ring position (global stage count)

  __device__ Epilogue(const PStep& st_, PSmem sm_, int lane_) : st(st_), sm(sm_), lane(lane_), q(0) {
    red_floats = st.red_floats;
  }

  // 1/rms of the phase's input from the per-CTA sum-of-squares partials
  // (RMSNorm(h) w x = (1/rms) sum_j W_ij w_j h_j: the consumers staged w h).
  __device__ float rms_scale(const float* parts) const {
    float ss = 0.f;
    for (int i = lane; i < (int)gridDim.x; i += 32) ss += __ldcg(parts + (int64_t)i * 4);
    ss = warp_sum(ss);
    return 1.0f / sqrtf(ss / (float)st.H + st.eps);
  }

  template <class Epi>
  __device__ bool run(Epi& epi, const PRows rows, const PGeom g, float scale = 1.f) {
    constexpr int A = Epi::kAlign;
    const int TR = g.TR, nsl = g.n_slices, nst = rows.n;
    const int64_t r0 = rows.r0, r1 = rows.r1;
    const int row_a = A == 1 ? lane : 2 * lane;
    if (nst > 0) epi.preload(r0, (int)min64(TR, r1 - r0), lane);
    for (int i = 0; i < nst; ++i, ++q) {
      const int slot = q % kPRed;
      if (!pwait(sm.rfull + slot, (uint32_t)((q / kPRed) & 1), sm.misc, st.wait_ns)) return false;
      const int64_t rs = r0 + (int64_t)i * TR;
      const int nr = (int)min64(TR, r1 - rs);
      const float* rd = sm.red + (size_t)slot * red_floats;
      float a = 0.f, b = 0.f;
      const bool mine = row_a < nr;
      if (mine && chk(st.status, kChkPartialRead, (row_a + A) * nsl - 1, red_floats)) {
        for (int c = 0; c < nsl; ++c) {
          a += rd[row_a * nsl + c];
          if (A == 2) b += rd[(row_a + 1) * nsl + c];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.rempty + slot);
      a *= scale;
      b *= scale;
      epi.rotate();
      if (i + 1 < nst) epi.preload(rs + TR, (int)min64(TR, r1 - rs - TR), lane);
      if (mine) epi.apply(rs + row_a, a, b);
    }
    return true;
  }

  // run() for the residual epilogue (rows of this CTA <= 64).
  __device__ bool run_resid(PEpiResid& epi, const PRows rows, const PGeom g) {
    const int TR = g.TR, nsl = g.n_slices, nst = rows.n;
    const int r0 = rows.r0, r1 = rows.r1;
    epi.begin(r0, r1, lane);
    for (int i = 0; i < nst; ++i, ++q) {
      const int slot = q % kPRed;
      if (!pwait(sm.rfull + slot, (uint32_t)((q / kPRed) & 1), sm.misc, st.wait_ns)) return false;
      const int rs = r0 + i * TR;
      const int nr = min(TR, r1 - rs);
      const float* rd = sm.red + (size_t)slot * red_floats;
      float a = 0.f;
      const bool mine = lane < nr;
      if (mine && chk(st.status, kChkPartialRead, (lane + 1) * nsl - 1, red_floats))
        for (int c = 0; c < nsl; ++c) a += rd[lane * nsl + c];
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.rempty + slot);
      epi.apply_stage(rs, mine, lane, a);
    }
    return true;
  }
};

// ------------------------------------------------------------ consumers
// Per-lane partial scores of one K row for the G query heads of a group:
// lane l holds dimensions 4l .. 4l + 3 (kp points at them, fp16).
template <int G>
__device__ __forceinline__ void score_parts(const uint8_t* kp, const float (&qr)[G][4], float (&v)[G]) {
  const uint2 kr = *reinterpret_cast<const uint2*>(kp);
  const float k0 = half_bits_to_float(kr.x), k1 = half_bits_to_float(kr.x >> 16);
  const float k2 = half_bits_to_float(kr.y), k3 = half_bits_to_float(kr.y >> 16);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float d = qr[h][0] * k0;
    d = fmaf(qr[h][1], k1, d);
    d = fmaf(qr[h][2], k2, d);
    d = fmaf(qr[h][3], k3, d);
    v[h] = d;
  }
}

// Warp sums of G values at once: each halving step exchanges half of the
// remaining values with the partner lane (lanes with bit o set keep the upper
// half), then plain butterfly steps finish the sums.  On return lane l holds
// the full sum of head l / (32 / G).  log2(G) + 5 - log2(G) steps, G - 1 + 5 -
// log2(G) shuffles in all.
template <int G>
__device__ __forceinline__ float heads_reduce(float (&v)[G], int lane) {
#pragma unroll
  for (int n = G, o = 16; n > 1; n >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = up ? v[j] : v[j + n / 2];
      const float keep = up ? v[j + n / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float s = v[0];
#pragma unroll
  for (int o = 16 / G; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

struct Consumer {
  const PStep& st;
  PSmem sm;  // used outside the GEMV stage loop only
  int warp, lane, ctid;
  int s;
  uint32_t ph;
  int q;  // partial-ring position (global stage count)

  __device__ Consumer(const PStep& st_, PSmem sm_, int warp_, int lane_)
      : st(st_), sm(sm_), warp(warp_), lane(lane_), ctid(warp_ * 32 + lane_), s(0), ph(0), q(0) {}

  // x of a GEMV phase into shared memory (fixed-point limbs or fp32): x = h,
  // or w h for a phase with an RMSNorm prologue -- the 1/rms scale is applied
  // to each row's result by the epilogue warp, so staging waits for nothing but
  // one batch of loads (h, and w).
  template <int QT, bool NORM>
  __device__ void stage(const float* h, const float* w, int64_t K, const XStage& xs) {
    constexpr int kBatch = NORM ? 4 : 8;
    const int nchunk = (int)(K / 128);
    for (int ch0 = warp; ch0 < nchunk; ch0 += kBatch * kPConsumers) {
      float4 hv[kBatch], wv[NORM ? kBatch : 1];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int ch = ch0 + b * kPConsumers;
        const int64_t col = (int64_t)ch * 128 + 4 * lane;
        hv[b] = ch < nchunk ? __ldcg(reinterpret_cast<const float4*>(h + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
        if constexpr (NORM) wv[b] = ch < nchunk ? ldg4(w + col) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int ch = ch0 + b * kPConsumers;
        if (ch >= nchunk) break;  // uniform across the warp
        float4 v = hv[b];
        if constexpr (NORM) v = make_float4(wv[b].x * v.x, wv[b].y * v.y, wv[b].z * v.z, wv[b].w * v.w);
        stage_chunk<QT>(v, (int64_t)ch * 128 + 4 * lane, xs, lane);
      }
    }
  }

  // A kernel built for two types leaves out the Q6_K paths that keep two
  // row slices in flight: with both types' code in one kernel their registers
  // would push the rest into local memory.
  // A GEMV phase in the block type of its kind: QA, or QB where the step's
  // plan gives that kind the second type (QB == QA: one type for all).
  template <int QA, int QB>
  __device__ bool gemv(int kind, const float* h, const float* w) {
    if constexpr (QA != QB) {
      if (st.qt[kind] == QB) return gemv_t<QB, false>(kind, h, w);
      return gemv_t<QA, false>(kind, h, w);
    } else {
      return gemv_t<QA, true>(kind, h, w);
    }
  }

  template <int QT, bool TWO>
  __device__ bool gemv_t(int kind, const float* h, const float* w) {
    const PGeom g = sm.kg[kind].g;
    const PRows rows = sm.kg[kind].rows;
    const int64_t K = phase_K(st, kind);
    const int nsl = g.n_slices, nrg = g.n_rg, TR = g.TR, rbytes = g.row_bytes, nst = rows.n;
    const int r0 = rows.r0, r1 = rows.r1;
    const bool busy = warp < g.NW;
    const int c = warp % nsl, gr = warp / nsl;
    const int64_t c0 = (int64_t)c * kSliceCols;
    const int ucols = (int)min64(kSliceCols, K - c0);
    const bool active = busy && lane_active<QT>(lane, ucols);
    XRegs<QT> xr;
    const XStage xs = xstage_at(sm.xst, K);
    // (debug build) the plan's staging region must hold this phase's x
    if (g.staged && !chk(st.status, kChkXStage, (int64_t)xstage_bytes(QT, K) - 1, st.xstage_bytes)) {
      if (ctid == 0) {
        atomicExch(sm.misc, 1);
        atomicExch(st.sync + st.abort_index, 1u);
      }
      return false;
    }
    if (g.staged) {
      if (w) stage<QT, true>(h, w, K, xs);
      else stage<QT, false>(h, w, K, xs);
      cons_bar();
      if (active) xr.load(xs, c, lane);
    } else {
      if constexpr (QT == QT_Q6_K) {
        if (active) xr.load_direct(PX{h, w, 1.f}, c, lane);
      }
    }
    // Stage loop.  Shared-memory locations are 32-bit offsets recomputed from
    // the plan, so the loop keeps few registers beside x and the weights.
    const uint32_t S = (uint32_t)st.n_slots, Z = (uint32_t)st.slot_bytes, RF = (uint32_t)st.red_floats;
    const uint32_t o_full = S * Z + (uint32_t)st.xstage_bytes;
    const uint32_t o_empty = o_full + 8 * S, o_rfull = o_empty + 8 * S, o_rempty = o_rfull + 8 * kPRed;
    const uint32_t o_red = o_rempty + 8 * kPRed;
    const volatile int* cta_abort = reinterpret_cast<const volatile int*>(p_smem + o_red + kPRed * RF * 4 + 64 * 8);
    const uint32_t sb = smem_addr(p_smem);
    const uint32_t ring_c = (uint32_t)c * QTraits<QT>::SEG;
    for (int i = 0; i < nst; ++i, ++q) {
      const uint32_t rslot = (uint32_t)q % kPRed;
      bool ok = pwait_a(sb + o_full + 8 * s, ph, cta_abort, st.wait_ns);
      if (ok && busy)
        ok = pwait_a(sb + o_rempty + 8 * rslot, (uint32_t)(((q / kPRed) & 1) ^ 1), cta_abort, st.wait_ns);
      if (!ok) {
        if (lane == 0) {
          atomicExch(sm.misc, 1);
          atomicExch(st.sync + st.abort_index, 1u);
        }
        return false;
      }
      if constexpr (QT == QT_Q6_K && TWO) {
        // A Q6_K row slice is a long dependent chain, so a warp keeps two in
        // flight.  With one row per warp per slot (TR == row groups) the next
        // slot is opened too and its row runs beside this one.
        if (TR == nrg && i + 1 < nst) {
          const int s2 = s + 1 == (int)S ? 0 : s + 1;
          const uint32_t ph2 = s + 1 == (int)S ? ph ^ 1u : ph;
          const uint32_t rslot2 = (uint32_t)(q + 1) % kPRed;
          bool ok2 = pwait_a(sb + o_full + 8 * s2, ph2, cta_abort, st.wait_ns);
          if (ok2 && busy)
            ok2 = pwait_a(sb + o_rempty + 8 * rslot2, (uint32_t)((((q + 1) / kPRed) & 1) ^ 1), cta_abort,
                          st.wait_ns);
          if (!ok2) {
            if (lane == 0) {
              atomicExch(sm.misc, 1);
              atomicExch(st.sync + st.abort_index, 1u);
            }
            return false;
          }
          if (busy) {
            const int rsa = r0 + i * TR;
            const int nra = min(TR, r1 - rsa), nrb = min(TR, r1 - rsa - TR);
            const int ra = (gr + nrg - i % nrg) % nrg, rb = (gr + nrg - (i + 1) % nrg) % nrg;
            const bool ha = ra < nra && chk(st.status, kChkRingRead, (int64_t)(ra + 1) * rbytes - 1, Z) &&
                            chk(st.status, kChkPartialWrite, ra * nsl + c, RF);
            const bool hb = rb < nrb && chk(st.status, kChkRingRead, (int64_t)(rb + 1) * rbytes - 1, Z) &&
                            chk(st.status, kChkPartialWrite, rb * nsl + c, RF);
            const uint8_t* sta = p_smem + ring_c + (uint32_t)s * Z + (uint32_t)ra * (uint32_t)rbytes;
            const uint8_t* stb = p_smem + ring_c + (uint32_t)s2 * Z + (uint32_t)rb * (uint32_t)rbytes;
            float va = 0.f, vb = 0.f;
            if (active && ha && hb) {
              va = xr.dot(sta, lane);
              vb = xr.dot(stb, lane);
            } else if (active) {
              if (ha) va = xr.dot(sta, lane);
              if (hb) vb = xr.dot(stb, lane);
            }
            va = warp_sum(va);
            vb = warp_sum(vb);
            if (lane == 0) {
              if (ha) (reinterpret_cast<float*>(p_smem + o_red) + rslot * RF)[ra * nsl + c] = va;
              if (hb) (reinterpret_cast<float*>(p_smem + o_red) + rslot2 * RF)[rb * nsl + c] = vb;
            }
          }
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_a(sb + o_empty + 8 * s);
            mbar_arrive_a(sb + o_rfull + 8 * rslot);
            mbar_arrive_a(sb + o_empty + 8 * s2);
            mbar_arrive_a(sb + o_rfull + 8 * rslot2);
          }
          s = s2;
          ph = ph2;
          if (++s == (int)S) { s = 0; ph ^= 1u; }
          ++i;  // the loop header steps past the second slot
          ++q;
          continue;
        }
      }
      if (busy) {
        const int rs = r0 + i * TR;
        const int nr = min(TR, r1 - rs);
        const uint8_t* stg = p_smem + ring_c + (uint32_t)s * Z;
        float* rd = reinterpret_cast<float*>(p_smem + o_red) + rslot * RF;
        // the row group that takes the extra rows rotates from stage to stage
        int rr = (gr + nrg - i % nrg) % nrg;
        if constexpr (QT == QT_Q6_K && TWO) {
          for (; rr + nrg < nr; rr += 2 * nrg) {  // two rows of this slot side by side
            float va = 0.f, vb = 0.f;
            const bool in = chk(st.status, kChkRingRead, (int64_t)(rr + nrg + 1) * rbytes - 1, Z) &&
                            chk(st.status, kChkPartialWrite, (rr + nrg) * nsl + c, RF);
            if (active && in) {
              va = xr.dot(stg + (uint32_t)rr * (uint32_t)rbytes, lane);
              vb = xr.dot(stg + (uint32_t)(rr + nrg) * (uint32_t)rbytes, lane);
            }
            va = warp_sum(va);
            vb = warp_sum(vb);
            if (lane == 0 && in) {
              rd[rr * nsl + c] = va;
              rd[(rr + nrg) * nsl + c] = vb;
            }
          }
        }
        for (; rr < nr; rr += nrg) {
          const bool in = chk(st.status, kChkRingRead, (int64_t)(rr + 1) * rbytes - 1, Z);
          float v = active && in ? xr.dot(stg + (uint32_t)rr * (uint32_t)rbytes, lane) : 0.f;
          v = warp_sum(v);
          if (lane == 0 && chk(st.status, kChkPartialWrite, rr * nsl + c, RF)) rd[rr * nsl + c] = v;
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_a(sb + o_empty + 8 * s);
        mbar_arrive_a(sb + o_rfull + 8 * rslot);
      }
      if (++s == (int)S) { s = 0; ph ^= 1u; }
    }
    return true;
  }

  // Block-wide (consumer warps) sum; result valid in every consumer thread.
  __device__ float csum(float v) {
    v = warp_sum(v);
    if (lane == 0) sm.scr[warp] = v;
    cons_bar();
    float t = 0.f;
    for (int w2 = 0; w2 < kPConsumers; ++w2) t += sm.scr[w2];
    cons_bar();
    return t;
  }

  __device__ void embed() {
    const int tp = st.params[1];
    int64_t tok = tp >= 0 ? tp : __ldcg(st.token_state);
    if (tok < 0 || tok >= st.V) {
      if (blockIdx.x == 0 && ctid == 0) atomicExch(st.status, (int)kStatusBadToken);
      tok = 0;
    }
    const int64_t H = st.H;
    const int64_t i0 = H * blockIdx.x / gridDim.x, i1 = H * (blockIdx.x + 1) / gridDim.x;
    float ss = 0.f;
    for (int64_t i = i0 + ctid; i < i1; i += kPCThreads) {
      const float v = half_bits_to_float(st.embed[tok * H + i]);
      st.hidden[i] = v;
      ss = fmaf(v, v, ss);
    }
    ss = csum(ss);
    if (ctid == 0) st.stats_embed[blockIdx.x * 4] = ss;
  }

  // Splits of this step's context per KV head: at least kPMinSplit positions
  // each where possible, at most n_split (one unit per CTA).
  __device__ void attn_splits(int n_ctx, int& ns, int& chunk) const {
    ns = (n_ctx + kPMinSplit - 1) / kPMinSplit;
    if (ns > st.n_split) ns = st.n_split;
    chunk = (n_ctx + ns - 1) / ns;
  }

  // Brings the K and V rows this CTA's attention units will read (the
  // positions before this step's) into L2, so the attention phase's tile
  // loads hit L2.  Issued by one thread at the start of the layer's Q/K/V phase.
  __device__ void kv_prefetch(const LRow& L) const {
    const int n_ctx = st.params[0] + 1;
    int ns, chunk;
    attn_splits(n_ctx, ns, chunk);
    for (int u = blockIdx.x; u < st.Hkv * ns; u += gridDim.x) {
      const int kvh = u / ns, split = u % ns;
      const int p0 = split * chunk;
      const int p1 = min(p0 + chunk, n_ctx - 1);
      for (int c0 = p0; c0 < p1; c0 += 128) {  // 32 KB per request
        const uint32_t bytes = (uint32_t)(min(p1 - c0, 128) * kPD * 2);
        const int64_t off = ((int64_t)kvh * st.max_ctx + c0) * kPD;
        l2_prefetch(L.kc + off, bytes);
        l2_prefetch(L.vc + off, bytes);
      }
    }
  }

  // Split-KV attention.  This step's context is cut into ns splits per KV
  // head (attn_splits); a unit walks its positions in tiles of kPChunk rows of
  // K and V (contiguous in the cache, brought to shared memory with 16-byte
  // asynchronous copies) with a running max and sum (online softmax).
  // Scores: a warp per position and group of at most 4 query heads (two
  // positions in flight), each lane 4 dimensions of each of those heads,
  // reduced for all of them at once (heads_reduce).
  // P V: thread (d8, h, pg) keeps dimensions 8 d8 .. 8 d8 + 7 of head h over
  // the tile positions pg, pg + NPG, ...; the NPG position groups are summed
  // in a fixed order at the end of the unit.  With one split the unit writes
  // the head output; otherwise it writes its (max, sum, unnormalised output),
  // waits for the other splits of its KV head and merges its share of the
  // head group's outputs (log-sum-exp).
  template <int G>
  __device__ void attention(const LRow& L, int lk) {
    const int n_ctx = st.params[0] + 1;
    int ns, chunk;
    attn_splits(n_ctx, ns, chunk);
    const AttnSmem a = attn_smem(sm.xst, G);
    const int units = st.Hkv * ns;
    const int S = kAttnPartStride;
    constexpr int NPG = kPCThreads / (16 * G);  // P V position groups
    constexpr int GW = G < 4 ? G : 4;           // query heads per warp in the score step
    constexpr int NH = G / GW;                  // warps per position (head groups)
    constexpr int WPG = kPConsumers / NH;       // warps per head group
    constexpr int LPH = 32 / GW;                // lanes holding one head's score after heads_reduce
    const int hh0 = (warp % NH) * GW, wpos = warp / NH;
    const int d8 = ctid % 16, hv = (ctid / 16) % G, pg = ctid / (16 * G);
    const bool pv_on = pg < NPG;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int kvh = u / ns, split = u % ns;
      const int p0 = split * chunk;
      const int p1 = min(p0 + chunk, n_ctx);
      const int np = p1 > p0 ? p1 - p0 : 0;
      const uint8_t* kbase = reinterpret_cast<const uint8_t*>(L.kc + ((int64_t)kvh * st.max_ctx + p0) * kPD);
      const uint8_t* vbase = reinterpret_cast<const uint8_t*>(L.vc + ((int64_t)kvh * st.max_ctx + p0) * kPD);
      const float* qg = st.q + (int64_t)kvh * G * kPD + 4 * lane;
      if (ctid < G) {
        a.ml[2 * ctid] = -INFINITY;
        a.ml[2 * ctid + 1] = 0.f;
      }
      float o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = 0.f;
      cons_bar();  // the running (max, sum) start values are visible
      for (int t0 = 0; t0 < np; t0 += kPChunk) {
        const int nt = min(kPChunk, np - t0);
        {  // K, V rows of the tile -> shared memory (nt * 256 bytes each)
          const int n16 = nt * (kPD * 2 / 16);
          const int off = t0 * kPD * 2;
          // (debug build) positions past the cache or a tile past its buffer are not copied
          const bool in = chk(st.status, kChkKvTile, p0 + t0 + nt - 1, st.max_ctx) &&
                          chk(st.status, kChkKvTile, (int64_t)nt * kPD * 2 - 1, (int64_t)kPChunk * kPD * 2);
          for (int i = ctid; in && i < 2 * n16; i += kPCThreads) {
            const bool isv = i >= n16;
            const int ob = (isv ? i - n16 : i) * 16;
            cp_async16((isv ? a.v : a.k) + ob, (isv ? vbase : kbase) + off + ob);
          }
          cp_async_commit();
        }
        // this lane's 4 dimensions of every query head of the group, loaded
        // per tile (L2) while the tile lands, so they are not held through P V
        float qr[GW][4];
#pragma unroll
        for (int h = 0; h < GW; ++h) {
          const float4 t = __ldcg(reinterpret_cast<const float4*>(qg + (hh0 + h) * kPD));
          qr[h][0] = t.x; qr[h][1] = t.y; qr[h][2] = t.z; qr[h][3] = t.w;
        }
        cp_async_wait_all();
        cons_bar();
        for (int i = wpos; i < nt; i += 2 * WPG) {
          const int i2 = i + WPG;
          const bool two = i2 < nt;  // warp-uniform
          float v1[GW], v2[GW];
          score_parts<GW>(a.k + (size_t)i * kPD * 2 + 8 * lane, qr, v1);
          if (two) score_parts<GW>(a.k + (size_t)i2 * kPD * 2 + 8 * lane, qr, v2);
          else {
#pragma unroll
            for (int h = 0; h < GW; ++h) v2[h] = 0.f;
          }
          const float s1 = heads_reduce<GW>(v1, lane), s2 = heads_reduce<GW>(v2, lane);
          if (lane % LPH == 0) {
            a.sc[(hh0 + lane / LPH) * kPChunk + i] = s1 * kAttnScale;
            if (two) a.sc[(hh0 + lane / LPH) * kPChunk + i2] = s2 * kAttnScale;
          }
        }
        cons_bar();
        // running max and sum per head (warp h)
        for (int h = warp; h < G; h += kPConsumers) {
          float mt = -INFINITY;
          for (int i = lane; i < nt; i += 32) mt = fmaxf(mt, a.sc[h * kPChunk + i]);
          mt = warp_max(mt);
          const float m_old = a.ml[2 * h], m_new = fmaxf(m_old, mt);
          float l = 0.f;
          for (int i = lane; i < nt; i += 32) {
            const float e = expf(a.sc[h * kPChunk + i] - m_new);
            a.sc[h * kPChunk + i] = e;
            l += e;
          }
          l = warp_sum(l);
          if (lane == 0) {
            const float f = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
            a.fac[h] = f;
            a.ml[2 * h] = m_new;
            a.ml[2 * h + 1] = fmaf(a.ml[2 * h + 1], f, l);
          }
        }
        cons_bar();
        if (pv_on) {
          const float f = a.fac[hv];
#pragma unroll
          for (int k = 0; k < 8; ++k) o[k] *= f;
          const float* e = a.sc + hv * kPChunk;
          for (int i = pg; i < nt; i += NPG) {
            const uint4 w = *reinterpret_cast<const uint4*>(a.v + (size_t)i * kPD * 2 + 16 * d8);
            const float ei = e[i];
            o[0] = fmaf(ei, half_bits_to_float(w.x), o[0]);
            o[1] = fmaf(ei, half_bits_to_float(w.x >> 16), o[1]);
            o[2] = fmaf(ei, half_bits_to_float(w.y), o[2]);
            o[3] = fmaf(ei, half_bits_to_float(w.y >> 16), o[3]);
            o[4] = fmaf(ei, half_bits_to_float(w.z), o[4]);
            o[5] = fmaf(ei, half_bits_to_float(w.z >> 16), o[5]);
            o[6] = fmaf(ei, half_bits_to_float(w.w), o[6]);
            o[7] = fmaf(ei, half_bits_to_float(w.w >> 16), o[7]);
          }
        }
        cons_bar();  // the next tile overwrites K, V and the scores
      }
      // the position groups' partial outputs -> the K tile buffer ([NPG][G][128] floats)
      float* pr = reinterpret_cast<float*>(a.k);
      if (pv_on) {
        float4* dst = reinterpret_cast<float4*>(pr + ((size_t)pg * G + hv) * kPD + 8 * d8);
        dst[0] = make_float4(o[0], o[1], o[2], o[3]);
        dst[1] = make_float4(o[4], o[5], o[6], o[7]);
      }
      cons_bar();
      for (int idx = ctid; idx < G * kPD; idx += kPCThreads) {
        const int h = idx / kPD, d = idx % kPD;
        float sum = 0.f;
#pragma unroll 4
        for (int g2 = 0; g2 < NPG; ++g2) sum += pr[((size_t)g2 * G + h) * kPD + d];
        if (ns == 1) {
          const int64_t oi = (int64_t)(kvh * G + h) * kPD + d;
          if (chk(st.status, kChkAttnOut, oi, (int64_t)st.Hq * kPD)) st.attn_out[oi] = sum / a.ml[2 * h + 1];
        } else {
          const int64_t pi = ((int64_t)(kvh * G + h) * ns + split) * S;
          if (chk(st.status, kChkAttnOut, pi + S - 1, (int64_t)st.Hq * st.n_split * S)) {
            float* dst = st.attn_part + pi;
            dst[2 + d] = sum;
            if (d == 0) {
              dst[0] = a.ml[2 * h];
              dst[1] = a.ml[2 * h + 1];
            }
          }
        }
      }
      if (ns == 1) {
        cons_bar();  // scratch reuse by the next unit
        continue;
      }
      // Publish this split, wait (bounded) until every split of this KV head
      // has published, then merge this unit's share of the head group's
      // outputs: elements [e0, e1) of the G x 128, each a log-sum-exp
      // weighted sum over the splits in split order.  Every unit of a KV head
      // runs on its own CTA (units <= grid), all resident at once.
      cons_bar();
      if (ctid == 0) {
        unsigned* hctr = st.sync + st.head_ctr_index + lk * st.Hkv + kvh;
        red_release_add(hctr, 1u);
        if (!grid_wait(hctr, (unsigned)ns, st.sync + st.abort_index, st.status, st.wait_ns)) atomicExch(sm.misc, 1);
      }
      cons_bar();
      const int E = G * kPD;
      const int e0 = split * E / ns, e1 = (split + 1) * E / ns;
      const float* pk = st.attn_part + (int64_t)kvh * G * ns * S;  // [G][ns][S]
      // (m, l) of every split of every head -> shared memory, and the first
      // element's values of the first kPMergeChunk splits -> registers, in
      // one round of loads
      for (int i = ctid; i < G * ns; i += kPCThreads) {
        const float2 t = __ldcg(reinterpret_cast<const float2*>(pk + (int64_t)i * S));
        a.sw[2 * i] = t.x;
        a.sw[2 * i + 1] = t.y;
      }
      float v[kPMergeChunk];
      {
        const int e = e0 + ctid;
        const float* pe = pk + (int64_t)(e / kPD) * ns * S + 2 + e % kPD;
#pragma unroll
        for (int k = 0; k < kPMergeChunk; ++k) v[k] = (e < e1 && k < ns) ? __ldcg(pe + (int64_t)k * S) : 0.f;
      }
      cons_bar();
      // per head: max over the splits, then weights exp(m_s - M) / L in place of m_s
      for (int h = ctid; h < G; h += kPCThreads) {
        float* mlh = a.sw + 2 * h * ns;
        float M = -INFINITY;
        for (int t = 0; t < ns; ++t) M = fmaxf(M, mlh[2 * t]);
        float Ls = 0.f;
        for (int t = 0; t < ns; ++t) {
          const float w = mlh[2 * t] == -INFINITY ? 0.f : expf(mlh[2 * t] - M);
          mlh[2 * t] = w;
          Ls = fmaf(w, mlh[2 * t + 1], Ls);
        }
        const float inv = 1.f / Ls;
        for (int t = 0; t < ns; ++t) mlh[2 * t] *= inv;
      }
      cons_bar();
      for (int e = e0 + ctid; e < e1; e += kPCThreads) {
        const int h = e / kPD;
        const float* pe = pk + (int64_t)h * ns * S + 2 + e % kPD;
        const float* wt = a.sw + 2 * h * ns;
        float O = 0.f;
        for (int t = 0; t < ns; t += kPMergeChunk) {
          if (e != e0 + ctid || t > 0) {
#pragma unroll
            for (int k = 0; k < kPMergeChunk; ++k) v[k] = t + k < ns ? __ldcg(pe + (int64_t)(t + k) * S) : 0.f;
          }
#pragma unroll
          for (int k = 0; k < kPMergeChunk; ++k)
            if (t + k < ns) O = fmaf(wt[2 * (t + k)], v[k], O);
        }
        if (chk(st.status, kChkAttnOut, (int64_t)kvh * E + e, (int64_t)st.Hq * kPD))
          st.attn_out[(int64_t)kvh * E + e] = O;
      }
      cons_bar();  // scratch reuse by the next unit
    }
  }
};

// QA: the block type of the step's GEMV phases; QB: a second type some phase
// kinds may use instead (st.qt[kind]), e.g. the Q6_K down projections and head
// of a Q4_K_M model.  QA == QB: one type.
template <int QA, int QB>
__global__ void __launch_bounds__(kPThreads, 1) persist_kernel(const __grid_constant__ PStep st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PSmem sm = psmem_at(p_smem, st.n_slots, st.slot_bytes, st.xstage_bytes, st.red_floats, st.n_layers);
  const int n = st.n_layers;
  const int np = 2 + 5 * n;
  const unsigned G = gridDim.x;
  unsigned* gabort = st.sync + st.abort_index;

  if (threadIdx.x == 0) {
    for (int k = 0; k < st.n_slots; ++k) {
      mbar_init(sm.full + k, 1);
      mbar_init(sm.empty + k, kPConsumers);
    }
    for (int k = 0; k < kPRed; ++k) {
      mbar_init(sm.rfull + k, kPConsumers);
      mbar_init(sm.rempty + k, 1);
    }
    sm.misc[0] = 0;
    fence_barrier_init();
  }
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const PLayer& Lg = st.layers[k];
    sm.lt[k] = LRow{Lg.attn_norm, Lg.ffn_norm, Lg.stats_down, Lg.kc, Lg.vc};
  }
  if (threadIdx.x < 7) {
    const int kind = threadIdx.x;
    if (kind == PK_QKV || kind == PK_O || kind == PK_GU || kind == PK_DOWN || kind == PK_HEAD)
      sm.kg[kind] = KGeo{st.g[kind], phase_rows(st, kind)};
  }
  // RMSNorm weights into L2 now, so that a phase start finds them there
  // (layer k's two vectors by CTA k mod grid, the final norm by the next one).
  if (warp == kPCopyWarp && lane == 0) {
    const uint32_t nb = (uint32_t)st.H * 4;
    for (int k = blockIdx.x; k <= n; k += gridDim.x) {
      if (k < n) {
        l2_prefetch(st.layers[k].attn_norm, nb);
        l2_prefetch(st.layers[k].ffn_norm, nb);
      } else {
        l2_prefetch(st.final_norm, nb);
      }
    }
  }
  if (st.probe_ts && threadIdx.x == 0) st.probe_ts[blockIdx.x] = global_ns();
  __syncthreads();

  if (warp == kPCopyWarp) {
    Copier cp(st, sm, lane, np);
    cp.run();
  } else if (warp == kPEpiWarp) {
    // ---------------------------------------------------------- epilogue
    // RoPE table of this step's position (the same for every layer), made
    // here so that the other warps do not wait for it
    {
      const int pos = st.params[0];
      for (int i = lane; i < kPD / 2; i += 32) {
        const double inv_freq = pow((double)st.theta, -2.0 * (double)i / (double)kPD);
        double sn, cn;
        sincos((double)pos * inv_freq, &sn, &cn);
        sm.rope[i] = make_float2((float)cn, (float)sn);
      }
      __syncwarp();
    }
    Epilogue ep(st, sm, lane);
    bool ok = true;
    for (int p = 1; p < np && ok; ++p) {
      const int kind = phase_kind(p, n);
      if (kind == PK_ATTN) continue;
      const LRow* L = (p >= 1 && p < 1 + 5 * n) ? sm.lt + (p - 1) / 5 : nullptr;
      const PRows rows = sm.kg[kind].rows;
      const PGeom g = sm.kg[kind].g;
      // the epilogue reads what earlier phases wrote
      int wok = 1;
      if (lane == 0) wok = grid_wait(st.sync + (p - 1), G, gabort, st.status, st.wait_ns);
      if (!__shfl_sync(0xffffffffu, wok, 0)) { ok = false; break; }
      // RMSNorm phases: the sum-of-squares partials of the phase input
      const float* parts = kind == PK_GU ? st.stats_o
                           : (p == 1 || (kind == PK_HEAD && n == 0)) ? st.stats_embed
                                                                    : sm.lt[(p - 2) / 5].stats_down;
      switch (kind) {
        case PK_QKV: {
          // (debug build) a position outside the cache stops the step instead of appending
          if (!chk(st.status, kChkKvAppend, st.params[0], st.max_ctx)) { ok = false; break; }
          EpiQKV epi{st.q, L->kc, L->vc, nullptr, st.params[0], (int64_t)st.Hq * st.D, (int64_t)st.Hkv * st.D,
                     st.D, st.max_ctx, st.theta, sm.rope};
          epi.status = st.status;
          ok = ep.run(epi, rows, g, ep.rms_scale(parts));
          break;
        }
        case PK_O: {
          if (rows.r1 - rows.r0 <= 64) {
            PEpiResid epi{st.h1, st.hidden, nullptr, st.stats_o};
            ok = ep.run_resid(epi, rows, g);
            if (ok) epi.finish(lane);
          } else {
            EpiResid epi{st.h1, st.hidden, nullptr, st.stats_o};
            epi.init(nullptr, lane);
            ok = ep.run(epi, rows, g);
            if (ok) epi.finish(lane);
          }
          break;
        }
        case PK_GU: {
          EpiSwiGLU epi{st.u};
          ok = ep.run(epi, rows, g, ep.rms_scale(parts));
          break;
        }
        case PK_DOWN: {
          if (rows.r1 - rows.r0 <= 64) {
            PEpiResid epi{st.hidden, st.h1, st.hidden, L->stats_down};
            ok = ep.run_resid(epi, rows, g);
            if (ok) epi.finish(lane);
          } else {
            EpiResid epi{st.hidden, st.h1, st.hidden, L->stats_down};
            epi.init(nullptr, lane);
            ok = ep.run(epi, rows, g);
            if (ok) epi.finish(lane);
          }
          break;
        }
        default: {
          EpiArgmax epi{st.logits, st.arg_parts};
          epi.init(nullptr, lane);
          ok = ep.run(epi, rows, g, ep.rms_scale(parts));
          if (ok) epi.finish(lane);
          break;
        }
      }
      if (!ok) break;
      // publish (release by lane 0 after the warp barrier); the last CTA
      // through the head phase picks the greedy token
      __syncwarp();
      unsigned old = 0;
      if (lane == 0) {
        if (kind == PK_HEAD) old = atom_acq_rel_add(st.sync + p, 1u);
        else red_release_add(st.sync + p, 1u);
        if (st.probe_ts) st.probe_ts[(size_t)(1 + p) * G + blockIdx.x] = global_ns();
      }
      old = __shfl_sync(0xffffffffu, old, 0);
      if (kind == PK_HEAD && old == G - 1) {
        float b = -INFINITY;
        int bi = 0x7fffffff;
        for (int i = lane; i < (int)G; i += 32) {
          const float v = __ldcg(st.arg_parts + i * 4);
          const int vi = __ldcg(reinterpret_cast<const int*>(st.arg_parts) + i * 4 + 1);
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
          *st.token_state = bi;
          if (st.next_token) *st.next_token = bi;
        }
      }
    }
    if (!ok && lane == 0) {
      atomicExch(sm.misc, 1);
      atomicExch(gabort, 1u);
    }
  } else {
    // ---------------------------------------------------------- consumers
    Consumer cs(st, sm, warp, lane);
    const int ctid = cs.ctid;
    for (int p = 0; p < np; ++p) {
      const int kind = phase_kind(p, n);
      int* go = sm.misc + 1 + (p & 1);
      if (ctid == 0) {
        bool ok = !*reinterpret_cast<volatile int*>(sm.misc);
        if (ok && p > 0) ok = grid_wait(st.sync + (p - 1), G, gabort, st.status, st.wait_ns);
        if (!ok) atomicExch(sm.misc, 1);  // the other warps stop waiting for these
        *go = ok;
      }
      cons_bar();
      if (!*go) break;
      const LRow* L = (p >= 1 && p < 1 + 5 * n) ? sm.lt + (p - 1) / 5 : nullptr;
      switch (kind) {
        case PK_EMBED:
          cs.embed();
          break;
        case PK_ATTN: {
          const int Gq = st.Hq / st.Hkv, lk = (p - 1) / 5;
          if (Gq == 8) cs.attention<8>(*L, lk);
          else if (Gq == 4) cs.attention<4>(*L, lk);
          else if (Gq == 2) cs.attention<2>(*L, lk);
          else cs.attention<1>(*L, lk);
          break;
        }
        default: {  // GEMV phases
          if (kind == PK_QKV && ctid == kPCThreads - 32) cs.kv_prefetch(*L);
          const float* h = kind == PK_GU ? st.h1 : kind == PK_O ? st.attn_out : kind == PK_DOWN ? st.u : st.hidden;
          const float* w = kind == PK_QKV ? L->attn_norm : kind == PK_GU ? L->ffn_norm
                           : kind == PK_HEAD ? st.final_norm : nullptr;
          cs.template gemv<QA, QB>(kind, h, w);  // a failed wait raised the CTA abort flag
          break;
        }
      }
      if (kind == PK_EMBED || kind == PK_ATTN) {
        // publish (release by one thread after the CTA barrier); a CTA named
        // by the host's stall setting withholds its embed publication, so
        // that the other CTAs' bounded waits run out (failure-path testing)
        cons_bar();
        if (ctid == 0 && !(p == 0 && (int)blockIdx.x == st.stall_cta)) {
          red_release_add(st.sync + p, 1u);
          if (st.probe_ts) st.probe_ts[(size_t)(1 + p) * G + blockIdx.x] = global_ns();
        }
      }
    }
  }
}

std::mutex g_pmu;

}  // namespace

// The (QA, QB) instantiation that runs a step whose phase kinds have the
// block types kt[] (QKV, O, GU, DOWN, HEAD), or (0, 0) when none does.
void persist_pair(const int* kt, int* qa, int* qb) {
  *qa = *qb = 0;
  const int a = kt[PK_QKV];
  int b = a;
  for (int k : {PK_O, PK_GU, PK_DOWN, PK_HEAD})
    if (kt[k] != a) {
      if (b != a && kt[k] != b) return;
      b = kt[k];
    }
  const bool one = a == b && (a == QT_Q8_0 || a == QT_Q4_0 || a == QT_Q6_K || a == QT_Q4_K || a == QT_Q5_K);
  const bool kq6 = (a == QT_Q4_K || a == QT_Q5_K) && b == QT_Q6_K;
  if (one || kq6) {
    *qa = a;
    *qb = b;
  }
}

// Host-side plan: slot size, stages, per-phase geometry.
int persist_plan(const int* kt, int H, int Hq, int Hkv, int D, int F, int64_t V, int max_ctx, int grid,
                 int n_layers, PStep* st, size_t* smem) {
  (void)V;
  int qa = 0, qb = 0;
  persist_pair(kt, &qa, &qb);
  if (qa == 0) return -1;
  if (D != kPD) return -1;
  if (Hkv <= 0 || Hq % Hkv) return -1;
  const int Gq = Hq / Hkv;
  if (Gq != 1 && Gq != 2 && Gq != 4 && Gq != 8) return -1;
  const int64_t KO = (int64_t)Hq * D;
  struct KInfo {
    int kind;
    int64_t K;
    int align;
  } ks[5] = {{PK_QKV, H, 2}, {PK_O, KO, 1}, {PK_GU, H, 2}, {PK_DOWN, F, 1}, {PK_HEAD, H, 1}};
  for (int k = 0; k < 7; ++k) st->qt[k] = kt[k];
  for (auto& k : ks) {
    const int qt = kt[k.kind];
    if (qt == QT_Q6_K ? (k.K % 2048) : (k.K % 256)) return -1;
    if (k.K > (int64_t)kPConsumers * kSliceCols) return -1;
    PGeom& g = st->g[k.kind];
    g.align = k.align;
    g.row_bytes = (int)(k.K / qt_block_elems(qt) * qt_block_bytes(qt));
    g.n_slices = (int)((k.K + kSliceCols - 1) / kSliceCols);
  }
  // attention scratch lives in the x staging region
  const int ns = persist_splits(grid, Hkv, max_ctx);
  const int attn_bytes = (int)((attn_smem_bytes(Gq, ns) + 15) / 16 * 16);
  const int smem_max = 227 * 1024;
  // Choose the slot size.  In order of priority: every phase can use all its
  // row groups (TR >= consumer warps per slice), at least 3 slots, for Q6_K
  // a slot's rows split evenly over every phase's row groups (its dot
  // products, not DRAM, set the pace, so a row group left without a row is
  // lost time), the most bytes in flight in the worst phase, then the smaller
  // slot.
  int best_Z = 0, best_S = 0;
  int64_t best_key[5] = {-1, -1, -1, -1, -1};
  for (auto& kz : ks) {
    const int rbz = st->g[kz.kind].row_bytes;
    for (int m = 1; m <= kPMaxTR; ++m) {
      const int Z = m * rbz;
      int xbz = attn_bytes, rf = 0;
      int64_t inflight_min = INT64_MAX;
      bool okz = true, full_rg = true, even = true;
      int TRs[8];
      for (auto& k : ks) {
        PGeom& g = st->g[k.kind];
        int tr = Z / g.row_bytes;
        if (tr > kPMaxTR) tr = kPMaxTR;
        if (k.align == 2) tr &= ~1;
        if (tr < 1) { okz = false; break; }
        TRs[k.kind] = tr;
        int nrg_max = kPConsumers / g.n_slices;
        if (nrg_max < 1) nrg_max = 1;
        if (tr < nrg_max) full_rg = false;
        const int nrg = nrg_max > tr ? tr : nrg_max;
        if (kt[k.kind] == QT_Q6_K && tr % nrg) even = false;
        const bool staged = kt[k.kind] != QT_Q6_K || nrg > 1;
        if (staged) {
          const int b = (int)((xstage_bytes(kt[k.kind], k.K) + 15) / 16 * 16);
          if (b > xbz) xbz = b;
        }
        if (tr * g.n_slices > rf) rf = tr * g.n_slices;
      }
      if (!okz) continue;
      xbz = (xbz + 15) / 16 * 16;
      int S = 0;
      while (psmem_bytes(S + 1, Z, xbz, (rf + 3) / 4 * 4, n_layers) <= (size_t)smem_max && S + 1 <= 16) ++S;
      if (S < 2) continue;
      for (auto& k : ks) {
        const int64_t inflight = (int64_t)S * TRs[k.kind] * st->g[k.kind].row_bytes;
        if (inflight < inflight_min) inflight_min = inflight;
      }
      const int64_t key[5] = {full_rg ? 1 : 0, S >= 3 ? 1 : 0, (qb == QT_Q6_K && even) ? 1 : 0, inflight_min,
                              -(int64_t)Z};
      bool better = false;
      for (int i = 0; i < 5; ++i) {
        if (key[i] != best_key[i]) { better = key[i] > best_key[i]; break; }
      }
      if (better) {
        for (int i = 0; i < 5; ++i) best_key[i] = key[i];
        best_Z = Z;
        best_S = S;
      }
    }
  }
  if (best_Z == 0) return -1;
  int rf = 0, xbz = attn_bytes;
  for (auto& k : ks) {
    PGeom& g = st->g[k.kind];
    int tr = best_Z / g.row_bytes;
    if (tr > kPMaxTR) tr = kPMaxTR;
    if (k.align == 2) tr &= ~1;
    g.TR = tr;
    int nrg = kPConsumers / g.n_slices;
    if (nrg < 1) nrg = 1;
    if (nrg > tr) nrg = tr;
    g.n_rg = nrg;
    g.NW = g.n_slices * nrg;
    g.staged = kt[k.kind] != QT_Q6_K || nrg > 1;
    if (g.staged) {
      const int b = (int)((xstage_bytes(kt[k.kind], k.K) + 15) / 16 * 16);
      if (b > xbz) xbz = b;
    }
    if (tr * g.n_slices > rf) rf = tr * g.n_slices;
  }
  st->slot_bytes = best_Z;
  st->n_slots = best_S;
  st->pf_stages = (kPPrefetchBytes + best_Z - 1) / best_Z;
  st->xstage_bytes = (xbz + 15) / 16 * 16;
  st->red_floats = (rf + 3) / 4 * 4;  // keeps the tables after it 16-byte aligned
  *smem = psmem_bytes(best_S, best_Z, st->xstage_bytes, st->red_floats, n_layers);
  return 0;
}

namespace {
// The instantiation for a type pair (see persist_pair) and its index.
using PKern = void (*)(const PStep);
PKern persist_kern(int qa, int qb, int* index) {
  struct {
    int a, b;
    PKern k;
  } const table[] = {{QT_Q8_0, QT_Q8_0, persist_kernel<QT_Q8_0, QT_Q8_0>},
                     {QT_Q4_0, QT_Q4_0, persist_kernel<QT_Q4_0, QT_Q4_0>},
                     {QT_Q6_K, QT_Q6_K, persist_kernel<QT_Q6_K, QT_Q6_K>},
                     {QT_Q4_K, QT_Q4_K, persist_kernel<QT_Q4_K, QT_Q4_K>},
                     {QT_Q5_K, QT_Q5_K, persist_kernel<QT_Q5_K, QT_Q5_K>},
                     {QT_Q4_K, QT_Q6_K, persist_kernel<QT_Q4_K, QT_Q6_K>},
                     {QT_Q5_K, QT_Q6_K, persist_kernel<QT_Q5_K, QT_Q6_K>}};
  for (int i = 0; i < (int)(sizeof table / sizeof table[0]); ++i)
    if (table[i].a == qa && table[i].b == qb) {
      *index = i;
      return table[i].k;
    }
  *index = -1;
  return nullptr;
}
}  // namespace

cudaError_t launch_persist(const PStep& st, size_t smem, int grid, cudaStream_t s) {
  static unsigned long long done[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int qa = 0, qb = 0, ki = -1;
  persist_pair(st.qt, &qa, &qb);
  PKern kern = persist_kern(qa, qb, &ki);
  if (!kern) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(done[ki] & (1ull << dev))) {
    std::lock_guard<std::mutex> g(g_pmu);
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    done[ki] |= 1ull << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once (grid-wide waits)
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, st);
}

int persist_grid(const PStep& st, size_t smem) {
  int qa = 0, qb = 0, ki = -1;
  persist_pair(st.qt, &qa, &qb);
  PKern kern = persist_kern(qa, qb, &ki);
  if (!kern) return 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess) return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPThreads, smem) != cudaSuccess) return 0;
  const int g = sm_count();
  return per_sm >= 1 && g <= 32 * kPPartsPerLane ? g : 0;
}

}  // namespace ntx
