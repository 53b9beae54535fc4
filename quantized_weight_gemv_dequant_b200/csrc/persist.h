// persist.h -- host/device description of one decode step for the persistent
// decode kernel (persist.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ntx {

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // the persistent kernel's wait limit unless a test lowers it
// Weight bytes per CTA requested into L2 beyond the ring (0: none).  Off by
// default: on B200 the extra requests cost more decode throughput than the
// L2 hits they bring (the ring alone keeps enough bytes in flight).
#ifndef NTX_PF_BYTES
#define NTX_PF_BYTES 0
#endif
constexpr int kPPrefetchBytes = NTX_PF_BYTES;
constexpr int kPChunk = 64;          // attention positions per K/V tile
constexpr int kPConsumers = 14;      // consumer warps per CTA (plus an epilogue warp and a copy warp)
constexpr int kPRed = 8;             // depth of the row-partial ring between consumers and the epilogue warp
constexpr int kPPartsPerLane = 8;    // CTAs at most: 32 * this (sum-of-squares partials read per lane)
constexpr int kPMaxTR = 32;          // rows per ring slot at most
constexpr int kPMinSplit = 128;      // attention positions per (KV head, split) unit at least, where possible
constexpr int kPMergeChunk = 18;     // splits whose values a thread loads at once in the split merge
constexpr int kPD = 128;             // head dimension
constexpr int kAttnPartStride = kPD + 2;  // floats per (query head, split) partial: m, l, o[128]

enum PKind : int { PK_EMBED = 0, PK_QKV = 1, PK_ATTN = 2, PK_O = 3, PK_GU = 4, PK_DOWN = 5, PK_HEAD = 6 };

// Geometry of one GEMV phase kind.
struct PGeom {
  int TR;         // rows per ring slot
  int n_slices;   // ceil(K / 2048)
  int n_rg;       // consumer warps per slice
  int NW;         // busy consumer warps = n_slices * n_rg
  int row_bytes;  // bytes of one weight row
  int staged;     // 1: x passes through shared memory, 0: lanes load it directly (Q6_K, one warp per slice)
  int align;      // rows per epilogue unit (2: the epilogue pairs rows)
};

// Device pointers of one executed layer.
struct PLayer {
  const uint8_t *wq, *wk, *wv, *wo, *wg, *wu, *wd;
  const float *attn_norm, *ffn_norm;
  uint16_t *kc, *vc;  // [Hkv][max_ctx][128] fp16
  float* stats_down;  // [grid][4] residual statistics of this layer's down projection
};

struct PStep {
  const PLayer* layers;  // executed layers, in order (device array)
  int n_layers;
  int H, Hq, Hkv, D, F, V, max_ctx;
  float eps, theta;
  const uint16_t* embed;    // [V][H] fp16
  const float* final_norm;  // [H]
  const uint8_t* head;      // [V] rows, same block type as the layers
  float *hidden, *q, *attn_out, *attn_part, *h1, *u;
  float *stats_embed, *stats_o, *arg_parts;  // [grid][4] each
  float* logits;                             // [V]
  const int* params;                         // [0] position, [1] token (-1: the last greedy token)
  int* token_state;                          // greedy token of the last step
  int* next_token;                           // nullable
  unsigned* sync;      // phase counters [2 + 5 n_layers], head counters, abort word: zero at launch
  int head_ctr_index;  // first attention merge counter in sync ([n_layers][Hkv])
  int abort_index;     // grid-wide abort word in sync
  int n_split;         // attention splits per KV head
  PGeom g[7];          // indexed by PKind
  int qt[7];           // block type of each GEMV phase kind (indexed by PKind)
  int slot_bytes, n_slots, xstage_bytes, red_floats;
  int pf_stages;  // stages of weight rows kept requested into L2 ahead of the ring
  int* status;  // device status word
  uint64_t wait_ns;  // limit on every wait of the kernel (nanoseconds of %globaltimer)
  int stall_cta;     // a CTA that withholds its embed publication (failure-path tests), -1: none
  unsigned long long* probe_ts;  // nullable: [1 + phases][grid] %globaltimer ns (row 0: kernel start,
                                 // row 1 + p: when the CTA published phase p)
};

// Fills the geometry fields and phase types of *st and the dynamic shared
// memory size for phase kinds of block types kt[] (indexed by PKind); -1 if
// the shapes or types are outside what the persistent kernel handles.
int persist_plan(const int* kt, int H, int Hq, int Hkv, int D, int F, int64_t V, int max_ctx, int grid,
                 int n_layers, PStep* st, size_t* smem);
// The instantiation (type pair) that runs phase kinds of types kt[]; 0, 0 if none.
void persist_pair(const int* kt, int* qa, int* qb);
// Grid size (one CTA per SM), or 0 if a CTA of this size cannot be resident.
int persist_grid(const PStep& st, size_t smem);
// Attention splits per KV head at most (at most one unit per CTA); a step
// uses fewer when its context is short.
inline int persist_splits(int grid, int Hkv, int max_ctx) {
  (void)max_ctx;
  const int ns = grid / Hkv;
  return ns < 1 ? 1 : ns;
}
// Words of the sync array for n_layers executed layers.
inline int persist_sync_words(int n_layers, int Hkv) { return 2 + 5 * n_layers + n_layers * Hkv + 1; }
cudaError_t launch_persist(const PStep& st, size_t smem, int grid, cudaStream_t s);

}  // namespace ntx
