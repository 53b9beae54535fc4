/*
 * ntx.h -- C ABI of libntx: batch-1 Llama decode over GGUF block-quantized
 * weights on NVIDIA B200 (sm_100a).
 *
 * What the calls compute follows the statement of the method in three pages:
 *   [README]  "NTransformer" -- 主な成果 (key results), 主な機能 (features),
 *             アーキテクチャ概要 (architecture overview), NVMeダイレクトストリーミング.
 *   [ShowHN]  "Show HN: NVMe経由でCPUをバイパスして単一のRTX 3090上で動作するLlama 3.1 70B"
 *             -- 量子化フォーマット対応表 (format table), 3層アダプティブキャッシュ詳細 (3-tier cache).
 *   [Article] "RTX 3090 1枚でLlama 70B — NVMe-to-GPU直結でCPUバイパスする革新技術"
 *             -- SLEP ストリーミングパイプライン, レイヤースキップ機構 (layer skip).
 *
 * Conventions (all calls):
 *  - Pointers are caller-owned.  "device" pointers address CUDA device memory
 *    of the current device; "host" pointers are ordinary or pinned host memory
 *    as stated.  The library never frees caller memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls only enqueue work on it and return; results are ready when the
 *    stream has reached them.  No call synchronises unless documented.
 *  - Every call returns an int status: NTX_OK (0) or a negative NTX_ERR_*.
 *    A failed argument check enqueues nothing.  ntx_last_error() returns a
 *    thread-local description of the most recent failure on the calling thread.
 *  - No exception crosses the ABI; kernels never trap.  A kernel that gives up
 *    waiting (bounded waits only) records a code in a device status word that
 *    ntx_device_status() reads.
 *  - Floating-point activations are fp32; the KV cache is IEEE fp16 stored as
 *    uint16_t bit patterns; quantized weights are raw GGUF block bytes.
 */
#ifndef NTX_H
#define NTX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NTX_API __attribute__((visibility("default")))
#else
#define NTX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status */
#define NTX_OK 0
#define NTX_ERR_INVALID_ARG (-1) /* null pointer, negative size, bad flag        */
#define NTX_ERR_SHAPE (-2)       /* size not a multiple of the block, over limit */
#define NTX_ERR_QTYPE (-3)       /* unsupported weight type                      */
#define NTX_ERR_ALIGN (-4)       /* pointer misaligned for the call              */
#define NTX_ERR_CUDA (-5)        /* CUDA launch / runtime error                  */
#define NTX_ERR_TIMEOUT (-6)     /* a bounded wait ran out                       */
#define NTX_ERR_NOMEM (-7)       /* host allocation or workspace too small       */

/* ------------------------------------------------------------ weight types
 * GGUF type ids.  Block layouts ([ShowHN] 量子化フォーマット対応表 gives the
 * bits per weight and block lengths; the byte layout is GGUF's):
 *   Q8_0: 34 B per 32 weights  = fp16 d | int8 q[32];            w = d q
 *   Q4_0: 18 B per 32 weights  = fp16 d | 16 B, byte j = q_j | q_(j+16) << 4;
 *                                                                 w = d (q - 8)
 *   Q6_K: 210 B per 256 weights = ql[128] | qh[64] | int8 sc[16] | fp16 d;
 *         element n (h = n/128, g = (n%128)/32, l = n%32): low 4 bits in
 *         ql[64h + 32(g%2) + l] (low nibble if g < 2, else high), high 2 bits
 *         at bit 2g of qh[32h + l];                               w = d sc[n/16] (q - 32)
 *   Q4_K: 144 B per 256 weights = fp16 d | fp16 dmin | 12 B scales | qs[128]
 *         (the super-blocks of the table's Q4_K_M, 4.5 bit/weight);
 *   Q5_K: 176 B per 256 weights = fp16 d | fp16 dmin | 12 B scales | qh[32] |
 *         qs[128] (5.5 bit/weight).  Both: eight 32-weight sub-blocks, each a
 *         6-bit scale sc_j and min m_j (j < 4: low six bits of scale bytes j
 *         and j+4; j >= 4: low / high nibble of byte j+4 plus the top two bits
 *         of bytes j-4 / j); element n = 64c + 32h + l: nibble h of
 *         qs[32c + l], Q5_K fifth bit = bit 2c+h of qh[l];    w = d sc_j q - dmin m_j
 *   F16, F32: one IEEE binary16 / binary32 per weight.
 * Weight matrices are row-major (out x in) with each row a run of K/block
 * blocks. */
#define NTX_F32 0
#define NTX_F16 1
#define NTX_Q4_0 2
#define NTX_Q8_0 8
#define NTX_Q4_K 12
#define NTX_Q5_K 13
#define NTX_Q6_K 14
/* ntx_layer_weights.qtype of a layer whose matrices have their own types
 * (mat_qtype[]), e.g. a Q4_K_M model ("mixed", [ShowHN] 量子化フォーマット対応表). */
#define NTX_MIXED (-1)

NTX_API const char* ntx_last_error(void);
NTX_API int ntx_version(void); /* major*10000 + minor*100 + patch */

/* Reads and clears the device status word of the current device (0 = no
 * kernel gave up a bounded wait since the last read).  Synchronises the
 * device.  Returns NTX_OK and stores the word in *code.  Codes: 1 a weight
 * copy did not land in time, 2 copies still outstanding when a CTA that gave
 * up had to exit (the context is then unusable: launch nothing more on it),
 * 3 a token id outside [0, V) reached the embedding, 4 a grid-wide barrier of
 * the persistent decode kernel ran out. */
NTX_API int ntx_device_status(int* code);

/* The bounds-checked debug build (compiled with NTX_CHECK; no counterpart in
 * the pages: a stand-in for a memory checker).  In that build the persistent
 * decode kernel and the per-op GEMV check the indices of their shared-memory
 * weight slots and row partials, the copy warp's slot writes, the KV append
 * position, the attention tile copies and output stores, and the x staging
 * region against their buffers, and the per-op attention and Q/K/V epilogue
 * check the step's cache position; an index outside records the first failing
 * site and index and the access is skipped (never trapped), so the results
 * are wrong but no memory outside a buffer is touched.  Sites: 1 slot read,
 * 2 partial write, 3 partial read, 4 KV append, 5 K/V tile, 6 attention
 * output, 7 x staging, 8 slot write, 9 per-op GEMV stage read, 10 per-op GEMV
 * partial, 11 per-op attention context, 12 per-op KV append.  ntx_check_enabled: 1 in that build, 0 in the release build.
 * ntx_check_report: waits for the device, then returns and clears the
 * record (site 0: every check passed, or the release build). */
NTX_API int ntx_check_enabled(void);
NTX_API int ntx_check_report(int* site, long long* index);

/* Number of SMs the kernels size their grids for on the current device. */
NTX_API int ntx_sm_count(void);

/* Measurement helper, not a step of the decode: reads the device buffer buf
 * (bytes long) once with streaming loads and writes the sum of its 32-bit
 * words modulo 2^32 to the device word *sum (zeroed by the call first), so
 * the read cannot be dropped and its result can be checked.  Timed over a
 * buffer much larger than L2 it gives the read-only HBM bandwidth, the
 * streaming ceiling of a weight-bound decode (the pages put decode time at
 * weight bytes over memory bandwidth: "RTX 3090 1枚でLlama 70B...", VRAMの壁).
 * buf must be 16-byte aligned and bytes a multiple of 16 (NTX_ERR_ALIGN);
 * buf may be NULL only when bytes is 0.  Asynchronous on stream. */
NTX_API int ntx_hbm_read_probe(const void* buf, uint64_t bytes, uint32_t* sum, void* stream);

/* Tuning: persistent GEMV CTAs per SM (1..4, default 1) for launches made
 * after the call, process-wide.  Workspace sizes do not depend on it. */
NTX_API int ntx_set_gemv_ctas_per_sm(int ctas_per_sm);

/* Tuning: programmatic dependent launch for ntx_gemv_q (0 = off, the
 * default; 1 = on), for calls made after it, process-wide.  When on, a
 * ntx_gemv_q kernel may start while the kernels enqueued before it on the
 * same stream are still running: it begins streaming W at once, and reads x,
 * reads residual and writes y only after those kernels have completed.  So,
 * while it is on, W must not be written by any kernel enqueued on the stream
 * since the last host synchronisation of that stream (weights that stay
 * fixed meet this).  Back-to-back GEMVs then overlap one launch's start with
 * the previous one's tail.  NTX_ERR_INVALID_ARG for other values. */
NTX_API int ntx_set_gemv_pdl(int on);

/* Tuning: whether an engine whose GEMV phases use two block types (Q4_K or
 * Q5_K matrices with Q6_K down projections and head, as in Q4_K_M / Q5_K_M
 * models) runs its all-resident steps as the persistent decode kernel (1)
 * or as the per-op kernel chain (0, the default).  With two row decoders in
 * one kernel its registers overflow and the spills are reloaded inside the
 * row loops; on B200 a 70B-shaped Q4_K_M model decoded at 33 tok/s that way
 * and 49 tok/s on the chain.  Applies to
 * engines created after the call, process-wide; NTX_ERR_INVALID_ARG for
 * other values. */
NTX_API int ntx_set_persist_two_types(int on);

/* ------------------------------------------------------------ per-op calls */

/* Dequantize n weights ([README] 主な機能: GGUF Q4_0/Q8_0/Q4_K_M/Q5_K/Q6_K/F16/F32;
 * [ShowHN] 量子化フォーマット対応表).  blocks: device, n/block_elems
 * consecutive blocks, 2-byte aligned (4-byte for F32).  out: device fp32[n].
 * Q8_0, Q4_0, Q6_K, F16, F32 are exact (every value is representable in
 * fp32); Q4_K / Q5_K give d sc q - dmin m rounded once to fp32 (the products
 * are exact).  NTX_ERR_SHAPE if n is not a multiple of the block length;
 * NTX_ERR_QTYPE for other types. */
NTX_API int ntx_dequant(int qtype, const void* blocks, float* out, int64_t n, void* stream);

/* Quantized GEMV y = W_deq x (+ residual) with fp32 accumulation ([README]
 * アーキテクチャ概要: the GEMV kernel; decode cost is weight bytes over
 * memory bandwidth, [Article] VRAMの壁).
 *   W: device, M rows of K/block_elems blocks (row-major), 16-byte aligned.
 *   x: device fp32[K].  y: device fp32[M], must not overlap x.
 *   residual: device fp32[M] or NULL; may be y itself (y = W x + y).
 * Types: Q8_0, Q4_0, Q4_K, Q5_K, Q6_K, F16, F32.
 * Limits: 1 <= M <= 2^31-1, block_elems | K, K <= 262144.  Shapes with
 * K % 2048 == 0 (Q6_K) or K % 256 == 0 (the others) and K <= 30720 take the
 * bulk-copy pipeline; other K take a slower generic kernel with the same
 * results.
 * Errors: NTX_ERR_QTYPE, NTX_ERR_SHAPE, NTX_ERR_ALIGN (W, x, y or residual
 * not 16-B aligned), NTX_ERR_INVALID_ARG (NULL, y overlapping x, residual
 * partially overlapping y). */
NTX_API int ntx_gemv_q(int qtype, const void* W, int64_t M, int64_t K, const float* x, float* y, const float* residual,
               void* stream);

/* RMSNorm y_i = w_i x_i / sqrt(mean_j x_j^2 + eps) ([README] 主な機能:
 * RMSNorm).  x, w, y: device fp32[n]; y may alias x.  1 <= n <= 2^20. */
NTX_API int ntx_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, void* stream);

/* Rotary position embedding in place ([README] 主な機能: RoPE): for every
 * head of q (n_q_heads x head_dim fp32) and of k (n_kv_heads x head_dim, may
 * be NULL when n_kv_heads == 0) the adjacent pair (2i, 2i+1) turns by the
 * angle pos * theta^(-2i/head_dim).  head_dim even, <= 256; pos >= 0.
 * Angles are formed in fp64, the rotation in fp32. */
NTX_API int ntx_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int pos, float theta, void* stream);

/* Grouped-query decode attention over an fp16 KV cache ([README] 主な機能:
 * GQA, KV cache; アーキテクチャ概要: softmax).  For query head h (reading KV
 * head h / (n_q_heads/n_kv_heads)):  out_h = sum_{p < n_ctx} softmax_p(q_h.k_p
 * / sqrt(head_dim)) v_p, split over positions and merged with a log-sum-exp
 * combine.
 *   q: device fp32[n_q_heads * head_dim].  out: device fp32, same size.
 *   k_cache, v_cache: device fp16 bits, [n_kv_heads][max_ctx][head_dim],
 *     16-byte aligned; positions 0..n_ctx-1 are read (n_ctx counts the current
 *     token, whose k, v the caller has already stored).
 *   workspace: device, >= ntx_attn_workspace_bytes(...) bytes, 16-B aligned;
 *     scratch only, contents on entry ignored.
 * Limits: head_dim == 128, n_kv_heads | n_q_heads, group n_q_heads/n_kv_heads
 * in {1, 2, 4, 8}, 1 <= n_ctx <= max_ctx. */
NTX_API size_t ntx_attn_workspace_bytes(int n_q_heads, int n_kv_heads, int head_dim, int max_ctx);
NTX_API int ntx_attn_decode(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out, int n_q_heads,
                    int n_kv_heads, int head_dim, int n_ctx, int max_ctx, void* workspace, size_t ws_bytes,
                    void* stream);

/* ntx_attn_decode without a workspace (the pages have no counterpart: this is
 * a convenience of this library).  Same computation, arguments, limits and
 * results as ntx_attn_decode, but the per-split partials live in a 2 MiB
 * static device array inside libntx, so the call allocates nothing and takes
 * no scratch buffer -- for callers that cannot provide one: hosts whose device
 * memory is owned by another allocator with a fixed budget, C programs with no
 * allocator on that path, latency-critical threads that must not take an
 * allocator's lock.  Limit: n_q_heads x (attention splits) x 130 floats <=
 * 524288, NTX_ERR_NOMEM beyond it (on a 148-SM B200 with 8 KV heads: up to
 * 32256 positions at 32 query heads, 16128 at 64); the size check comes
 * before any CUDA call.  The first call on a device looks up the array's
 * address (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture.  Later calls take no lock.  The cached address does not
 * survive cudaDeviceReset: do not use this call on a device after resetting
 * it.  Every GPU that loads libntx holds the array until exit, all calls share
 * it and it keeps the last call's contents: calls that overlap on the GPU
 * (e.g. on two streams) race. */
NTX_API int ntx_attn_decode_static(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out,
                                   int n_q_heads, int n_kv_heads, int head_dim, int n_ctx, int max_ctx, void* stream);

/* SwiGLU out_i = silu(gate_i) up_i, silu(z) = z / (1 + e^-z) ([README]
 * 主な機能: SwiGLU).  Device fp32[n] each; out may alias either input. */
NTX_API int ntx_swiglu(const float* gate, const float* up, float* out, int64_t n, void* stream);

/* ------------------------------------------------------------ layer / model */
typedef struct {
  int32_t hidden;     /* H */
  int32_t n_heads;    /* Hq */
  int32_t n_kv_heads; /* Hkv */
  int32_t head_dim;   /* D (128) */
  int32_t ffn;        /* F */
  int32_t vocab;      /* V */
  int32_t n_layers;   /* L */
  float eps;          /* RMSNorm epsilon */
  float theta;        /* RoPE base */
  int32_t max_ctx;    /* KV cache capacity in positions */
  float skip_threshold; /* cosine layer-skip threshold tau */
} ntx_model_config;

/* One layer's weights inside one contiguous blob at `base` (device memory or
 * a device slot the layer was streamed into).  Offsets are in bytes from base
 * and 256-B aligned: wq (Hq*D x H), wk, wv (Hkv*D x H), wo (H x Hq*D),
 * wg, wu (F x H), wd (H x F) as quantized blocks of `qtype`; attn_norm and
 * ffn_norm as fp32[H].  The same layout serves resident and pinned-host
 * copies, so streaming a layer is one contiguous copy. */
typedef struct {
  int32_t qtype;  /* block type of every matrix, or NTX_MIXED: mat_qtype[] holds them */
  const void* base;
  uint64_t off_wq, off_wk, off_wv, off_wo, off_wg, off_wu, off_wd, off_attn_norm, off_ffn_norm;
  int32_t mat_qtype[7]; /* wq, wk, wv, wo, wg, wu, wd; read only when qtype == NTX_MIXED */
} ntx_layer_weights;

/* Fills the canonical offsets of a layer blob for cfg and qtype (base left
 * NULL) and returns the blob size in bytes, 0 on bad arguments. */
NTX_API uint64_t ntx_layer_layout(const ntx_model_config* cfg, int qtype, ntx_layer_weights* out);

/* The same for a layer whose seven matrices wq, wk, wv, wo, wg, wu, wd have
 * the block types qtypes[0..6] (host array); sets qtype = NTX_MIXED.  A layer
 * runs only if wq, wk and wv share one type and wg and wu share one type (each
 * pair or triple is one fused GEMV).  0 on bad arguments. */
NTX_API uint64_t ntx_layer_layout_mixed(const ntx_model_config* cfg, const int32_t* qtypes, ntx_layer_weights* out);

/* Workspace one ntx_decode_layer call needs (device bytes). */
NTX_API size_t ntx_layer_workspace_bytes(const ntx_model_config* cfg);

/* One pre-norm Llama decode layer for one token at position pos ([README]
 * 主な機能: Llama architecture RoPE, GQA, SwiGLU, RMSNorm, KV cache;
 * [Article] レイヤースキップ機構 for the cosine):
 *   n1 = RMSNorm(h) w_attn; q,k,v = Wq n1, Wk n1, Wv n1; RoPE(q), RoPE(k);
 *   k, v -> fp16 cache row pos; a = GQA attention over rows 0..pos;
 *   h1 = h + Wo a; n2 = RMSNorm(h1) w_ffn; h = h1 + Wd (silu(Wg n2) (Wu n2)).
 *   hidden: device fp32[H], read and overwritten with the layer output.
 *   k_cache, v_cache: device fp16 bits [Hkv][max_ctx][D] of this layer.
 *   cos_out: device float or NULL; receives cos(h_in, h_out).
 *   workspace: device scratch >= ntx_layer_workspace_bytes(cfg), 256-B aligned.
 * Limits: head_dim 128; query group in {1, 2, 4, 8}; each matrix's input
 * length (H, F or Hq*D) a multiple of 2048 for Q6_K and of 256 for every
 * other type; wq, wk, wv of one type and wg, wu of one type (NTX_MIXED);
 * 0 <= pos < max_ctx; weight offsets 16-B aligned.  hidden, base and the
 * caches 16-B aligned, workspace 256-B aligned. */
NTX_API int ntx_decode_layer(const ntx_model_config* cfg, const ntx_layer_weights* w, uint16_t* k_cache, uint16_t* v_cache,
                     float* hidden, int pos, float* cos_out, void* workspace, size_t ws_bytes, void* stream);

/* Decode engine: the per-token forward over all layers ([README] 3-Tier
 * adaptive cache, 4 data paths 1-2; [ShowHN] 3層アダプティブキャッシュ詳細:
 * tier A resident, tier B pinned RAM + H2D into double buffers; [Article]
 * SLEP ストリーミングパイプライン: copy of the next layer overlapped with the
 * current layer's compute).
 *   layers[l].base: device memory (tier_map[l] == 0) or pinned host memory
 *     (tier_map[l] == 1) holding the layer blob (ntx_layer_layout order).
 *   slot0, slot1: device buffers of slot_bytes each (>= the largest host
 *     layer) into which host layers are copied; may be NULL if no layer is
 *     on the host.
 *   embed: device fp16 bits [V][H].  final_norm: device fp32[H].
 *   head: device quantized [V x H] of head_qtype.
 *   k_caches[l], v_caches[l]: device fp16 bits [Hkv][max_ctx][D].
 *   workspace: device scratch >= ntx_engine_workspace_bytes(cfg).
 *   compute_stream / copy_stream: distinct streams; copy_stream may be NULL
 *     when no layer is on the host.
 * The engine owns only its events, a pinned 16-byte parameter block and the
 * captured CUDA graphs; the caller keeps every buffer alive until
 * ntx_engine_destroy.
 * Execution: when every layer and the head share one block type (or two,
 * after ntx_set_persist_two_types(1)), a step
 * whose executed layers are all resident (tier 0) -- every step of an engine
 * without host layers, and the NTX_USE_SKIP steps of one whose recorded skip
 * set skips every host layer -- runs as ONE persistent kernel (one CTA per
 * SM, grid-wide phase barriers, the weight stream continuing across phases);
 * other steps, or any step with NTX_NO_PERSIST, run as a chain of per-op
 * kernels (about five per layer) joined by programmatic dependent launch. */
typedef struct ntx_engine ntx_engine;

#define NTX_CALIBRATE_SKIP 1 /* run every layer, record cosines, fix the skip set {l : cos_l >= tau} */
#define NTX_USE_SKIP 2       /* skip the layers of the recorded set (not computed, not streamed) */
#define NTX_NO_GRAPH 4       /* launch kernel by kernel instead of replaying the captured graph */
#define NTX_NO_PERSIST 8     /* run the step as a chain of per-op kernels even where the persistent kernel applies */

NTX_API size_t ntx_engine_workspace_bytes(const ntx_model_config* cfg);
NTX_API int ntx_engine_create(const ntx_model_config* cfg, const ntx_layer_weights* layers, const int8_t* tier_map,
                      void* slot0, void* slot1, size_t slot_bytes, const uint16_t* embed, const float* final_norm,
                      const void* head, int head_qtype, uint16_t* const* k_caches, uint16_t* const* v_caches,
                      void* workspace, size_t ws_bytes, void* compute_stream, void* copy_stream,
                      ntx_engine** out);

/* One decode step for `token` at position `pos` (0 <= pos < max_ctx):
 * embed -> layers -> final RMSNorm -> head -> greedy argmax (ties -> lowest id).
 *   token: a token id in [0, V), or -1 to use the engine's previous argmax
 *     (device-side, no host round trip).
 *   logits: device fp32[V] or NULL.  next_token: device int32 or NULL.
 *   cos_out: device fp32[L] or NULL; receives cos(h_in, h_out) of every
 *     layer computed in this step (skipped layers are left untouched).
 * With NTX_CALIBRATE_SKIP the call waits for the step to finish (it reads the
 * cosines back to fix the skip set); otherwise it only enqueues. */
NTX_API int ntx_decode_step(ntx_engine* e, int32_t token, int pos, float* logits, int32_t* next_token, int flags,
                    float* cos_out);

/* Self-speculative decoding ([README] 主な機能: Self-speculative decoding, the
 * VRAM-resident layers as the draft model, no extra model; クイックスタート
 * --self-spec --draft-k 3).  Given `token` at position `pos` (not yet
 * processed), the draft -- the resident (tier 0) layers only, then the head --
 * proposes draft_k greedy tokens for positions pos+1..pos+draft_k, one step
 * each; then the whole model verifies the token and the proposals at
 * positions pos..pos+draft_k in one pass, layer by layer, so each host layer
 * crosses the link once for all draft_k + 1 tokens.  The longest prefix of
 * proposals equal to the whole model's greedy tokens is accepted, followed by
 * the whole model's next token: tokens_out[0..*n_out-1] (host int32,
 * capacity draft_k + 1, 1 <= *n_out <= draft_k + 1) are exactly the greedy
 * continuation t_(pos+1), ..., t_(pos+n_out); the KV caches then hold the
 * positions up to pos + n_out - 1, and the next call passes
 * tokens_out[n_out-1] at position pos + n_out (or ntx_decode_step with
 * token -1).
 *   draft_k: 1..7; pos + draft_k < max_ctx; token in [0, V).
 *   flags: NTX_USE_SKIP (the recorded skip set applies to draft and
 *   verification), NTX_NO_PERSIST (the draft as the per-op chain).
 * Needs executed layers in both tiers (NTX_ERR_INVALID_ARG otherwise).  The
 * call waits for the pass to finish (it reads the tokens back). */
NTX_API int ntx_decode_spec(ntx_engine* e, int32_t token, int pos, int draft_k, int32_t* tokens_out, int* n_out,
                            int flags);

/* Profiling: while set, every ntx_decode_step made with NTX_NO_GRAPH records
 * begin_events[k] and end_events[k] (caller-created cudaEvent_t, passed as
 * void*) on the compute stream.  Per-op chain: immediately before and after
 * the gate/up GEMV of the k-th computed layer of the step -- the largest
 * kernel of a layer.  Persistent kernel: begin_events[0] / end_events[0]
 * bracket the kernel.  n is the capacity of both arrays (layers past it are
 * not probed); n == 0 clears the probe.  Graph replays never record probe
 * events. */
NTX_API int ntx_engine_set_probe(ntx_engine* e, void* const* begin_events, void* const* end_events, int n);

/* Profiling the persistent kernel: while set, every ntx_decode_step made
 * with NTX_NO_GRAPH that runs the persistent kernel writes %globaltimer
 * nanoseconds into dev_ts (device, 8-byte aligned, n_words 64-bit words):
 * dev_ts[b] = start of CTA b, dev_ts[(1 + p) * grid + b] = when CTA b published
 * phase p (p = 0 embed; 1 + 5k + {0..4} = Q/K/V, attention, O, gate/up, down
 * of the k-th executed layer; 1 + 5n = head).  A step whose phases do not fit
 * records nothing.  Returns the grid size (CTAs) of the persistent kernel, 0
 * if this engine does not use it, or a negative error; n_words == 0 clears
 * the probe. */
NTX_API int ntx_engine_set_phase_probe(ntx_engine* e, unsigned long long* dev_ts, size_t n_words);

/* Number of libntx kernels one decode step launched (the last step enqueued
 * or captured by this engine), or a negative error. */
NTX_API int ntx_engine_launches_per_step(ntx_engine* e);

/* The persistent decode kernel's plan for a model whose layers all use block
 * type qtype, as ntx_engine_create makes it (a host computation: no GPU
 * needed; the grid is the current device's SM count, 148 without a device).
 * Outputs (each nullable): *slot_bytes, *n_slots = the weight ring's slot size
 * and slot count; *smem_bytes = dynamic shared memory per CTA;
 * rows_per_slot[5] = whole weight rows per slot for the Q/K/V, O, gate/up,
 * down and head phases.  NTX_ERR_INVALID_ARG for a NULL or non-positive
 * config, NTX_ERR_QTYPE for other types, NTX_ERR_SHAPE when the persistent
 * kernel does not take the model (the engine then runs the per-op chain). */
NTX_API int ntx_persistent_plan(const ntx_model_config* cfg, int qtype, int* slot_bytes, int* n_slots,
                                size_t* smem_bytes, int* rows_per_slot);

/* ------------------------------------------------------------ tier sizing
 * Automatic tier sizing ([README] 3-Tier: tier sizes computed from
 * cudaMemGetInfo() and /proc/meminfo; [ShowHN] 3層アダプティブキャッシュ詳細:
 * VRAM resident > pinned RAM > NVMe/mmap).  The NVMe / mmap tier is not
 * provided here: a model that does not fit the first two is refused. */

/* Device bytes an engine for cfg keeps besides the layer blobs and slots:
 * fp16 embedding table, final norm, the head (head_qtype), the fp16 KV caches
 * of all layers, and the engine workspace.  0 on bad arguments.  Host only. */
NTX_API uint64_t ntx_engine_device_bytes(const ntx_model_config* cfg, int head_qtype);

/* Tier map for cfg->n_layers layers of layer_bytes each (the blob size from
 * ntx_layer_layout), placed in execution order: the first n resident
 * (tier_map[l] = 0), the rest in pinned host memory (1), n the largest count
 * for which n blobs + two device slots of layer_bytes (when n < L) +
 * ntx_engine_device_bytes(cfg, head_qtype) fit in device_free -
 * device_reserve.  The host layers must fit in host_available - host_reserve.
 *   tier_map: host int8[L], written on success.  n_resident: host int or NULL.
 * Errors: NTX_ERR_INVALID_ARG; NTX_ERR_NOMEM when the non-layer buffers or the
 * two slots do not fit the device, or the streamed layers do not fit the host
 * (a third tier would be needed).  Host only; no CUDA call. */
NTX_API int ntx_auto_tier_map(const ntx_model_config* cfg, uint64_t layer_bytes, int head_qtype,
                              uint64_t device_free, uint64_t device_reserve, uint64_t host_available,
                              uint64_t host_reserve, int8_t* tier_map, int* n_resident);

/* Memory the tiers can use: *device_free and *device_total from
 * cudaMemGetInfo on the current device (skipped when both are NULL), and
 * *host_available = MemAvailable of meminfo_path (NULL: /proc/meminfo), in
 * bytes.  NTX_ERR_CUDA if the device query fails, NTX_ERR_INVALID_ARG if the
 * file cannot be read or has no MemAvailable line. */
NTX_API int ntx_memory_budget(uint64_t* device_free, uint64_t* device_total, uint64_t* host_available,
                              const char* meminfo_path);

/* Copies the recorded skip set (1 = skipped) into mask_host[L]; returns the
 * number of skipped layers, or a negative error. */
NTX_API int ntx_engine_skip_mask(ntx_engine* e, uint8_t* mask_host);

/* Waits (bounded, see ntx_set_host_wait_limit) for the engine's streams and
 * frees the engine.  NTX_ERR_TIMEOUT if its work has not completed in time:
 * the engine is then kept (nothing is freed under running work) and the call
 * may be repeated. */
NTX_API int ntx_engine_destroy(ntx_engine* e);

/* Failure detection.  Every host wait of the engine (ntx_engine_create,
 * the parameter ring of ntx_decode_step, the calibration read-back,
 * ntx_engine_destroy) polls its stream with a deadline of `ms` milliseconds
 * (default 60000, process-wide) and returns NTX_ERR_TIMEOUT past it, leaving
 * the GPU work running.  NTX_ERR_INVALID_ARG for 0.  Environment hook for
 * tests: NTX_FAULT=<name>[,<name>...] makes the named point fail as if its
 * operation had failed, before the call enqueues anything: pinned_alloc
 * (ntx_engine_create: NTX_ERR_NOMEM), h2d_submit (ntx_decode_step of a step
 * that streams host layers: NTX_ERR_CUDA), host_wait (every bounded host
 * wait: NTX_ERR_TIMEOUT). */
NTX_API int ntx_set_host_wait_limit(uint64_t ms);

/* Failure-path testing of the persistent kernel: for steps enqueued after the
 * call without a graph (NTX_NO_GRAPH; captured graphs keep their settings),
 * CTA stall_cta (-1: none) withholds its publication of the embed phase, and
 * every wait of the kernel gives up after wait_ns nanoseconds (0: the default
 * 2 s).  With a stalled CTA the others' grid-wide waits run out: the kernel
 * returns with device status 4 (ntx_device_status) and no CTA left waiting. */
NTX_API int ntx_engine_set_fault(ntx_engine* e, int stall_cta, uint64_t wait_ns);

#ifdef __cplusplus
}
#endif

#endif /* NTX_H */
