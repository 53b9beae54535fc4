// api.cu -- the extern "C" boundary of libntx: argument checks, error
// reporting, the layer blob layout, the single-layer call and the decode
// engine (resident + pinned-host tiers, double-buffered device slots, cosine
// layer skip, CUDA-graph replay of the per-token launch sequence).
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <string>
#include <thread>
#include <tuple>
#include <vector>

#include "launch.h"
#include "ntx.h"
#include "persist.h"

namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(NTX_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int block_elems(int qt) {
  switch (qt) {
    case NTX_F32: case NTX_F16: return 1;
    case NTX_Q4_0: case NTX_Q8_0: return 32;
    case NTX_Q4_K: case NTX_Q5_K: case NTX_Q6_K: return 256;
    default: return 0;
  }
}
int block_bytes(int qt) {
  switch (qt) {
    case NTX_F32: return 4;
    case NTX_F16: return 2;
    case NTX_Q4_0: return 18;
    case NTX_Q8_0: return 34;
    case NTX_Q4_K: return 144;
    case NTX_Q5_K: return 176;
    case NTX_Q6_K: return 210;
    default: return 0;
  }
}
bool qtype_ok(int qt) { return block_elems(qt) != 0; }

// Block type of matrix i (0..6 = wq, wk, wv, wo, wg, wu, wd) of a layer.
int mat_qt(const ntx_layer_weights* w, int i) { return w->qtype == NTX_MIXED ? w->mat_qtype[i] : w->qtype; }

int64_t mat_bytes(int qt, int64_t M, int64_t K) { return M * (K / block_elems(qt)) * block_bytes(qt); }

uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// ------------------------------------------------------------ host waits
// Every host wait of the engine polls with a deadline instead of blocking:
// a stream or event that has not completed within the limit gives
// NTX_ERR_TIMEOUT (the GPU work is left running; the caller decides).
std::atomic<uint64_t> g_host_wait_ms{60000};

// Engines created while this is set run two-block-type steps on the
// persistent kernel (ntx_set_persist_two_types).
std::atomic<int> g_persist_two{0};

// Host-side fault injection for tests: NTX_FAULT is a comma-separated list
// of names; a call that reaches the named point fails as if the underlying
// operation had failed, before it enqueues any work.
//   pinned_alloc  ntx_engine_create's pinned parameter block
//   h2d_submit    ntx_decode_step of a step that streams host layers
//   host_wait     every bounded host wait (reports NTX_ERR_TIMEOUT at once)
bool fault(const char* name) {
  const char* env = getenv("NTX_FAULT");
  if (!env || !*env) return false;
  const size_t n = strlen(name);
  for (const char* p = env; *p;) {
    const char* q = strchr(p, ',');
    const size_t len = q ? (size_t)(q - p) : strlen(p);
    if (len == n && strncmp(p, name, n) == 0) return true;
    if (!q) break;
    p = q + 1;
  }
  return false;
}

// Waits for `ev` (already recorded) with the host deadline: cudaSuccess,
// cudaErrorTimeout, or the event's error.
cudaError_t wait_event(cudaEvent_t ev) {
  if (fault("host_wait")) return cudaErrorTimeout;
  const auto t0 = std::chrono::steady_clock::now();
  const auto limit = std::chrono::milliseconds(g_host_wait_ms.load());
  for (unsigned spin = 0;; ++spin) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e != cudaErrorNotReady) return e;
    if (std::chrono::steady_clock::now() - t0 > limit) return cudaErrorTimeout;
    if (spin > 64) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

// Records `ev` on stream s and waits for it with the host deadline.
cudaError_t wait_stream(cudaStream_t s, cudaEvent_t ev) {
  const cudaError_t e = cudaEventRecord(ev, s);
  return e == cudaSuccess ? wait_event(ev) : e;
}

int wait_fail(cudaError_t e, const char* what) {
  if (e == cudaErrorTimeout) return fail(NTX_ERR_TIMEOUT, "%s: the GPU work did not complete within %llu ms", what,
                                         (unsigned long long)g_host_wait_ms.load());
  return cuda_fail(e, what);
}

// K constraint of the fused (bulk-copy) GEMV path.
bool k_ok_fused(int qt, int64_t K) { return qt == NTX_Q6_K ? K % 2048 == 0 : K % 256 == 0; }

int check_dims(const ntx_model_config* c) {
  if (!c) return fail(NTX_ERR_INVALID_ARG, "config is NULL");
  if (c->hidden <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->ffn <= 0 || c->n_layers < 0 || c->max_ctx <= 0)
    return fail(NTX_ERR_SHAPE, "non-positive dimension in config");
  if (c->head_dim != 128) return fail(NTX_ERR_SHAPE, "head_dim %d unsupported (128 only)", c->head_dim);
  if (c->n_heads % c->n_kv_heads) return fail(NTX_ERR_SHAPE, "n_heads %% n_kv_heads != 0");
  const int G = c->n_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(NTX_ERR_SHAPE, "query group %d unsupported (1,2,4,8)", G);
  if (!(c->eps >= 0.f) || !(c->theta > 0.f)) return fail(NTX_ERR_INVALID_ARG, "bad eps/theta");
  return NTX_OK;
}

// Dimensions and the block type of every matrix of a layer: each type known,
// each matrix's input length a whole number of bulk-copy units, and the
// matrices that share one GEMV (wq/wk/wv, wg/wu) of one type.
int check_config(const ntx_model_config* c, const ntx_layer_weights* w) {
  int rc = check_dims(c);
  if (rc) return rc;
  if (w->qtype != NTX_MIXED && !qtype_ok(w->qtype)) return fail(NTX_ERR_QTYPE, "unsupported weight type %d", w->qtype);
  const int64_t Q = (int64_t)c->n_heads * c->head_dim;
  const int64_t K[7] = {c->hidden, c->hidden, c->hidden, Q, c->hidden, c->hidden, c->ffn};
  static const char* names[7] = {"wq", "wk", "wv", "wo", "wg", "wu", "wd"};
  for (int i = 0; i < 7; ++i) {
    const int qt = mat_qt(w, i);
    if (!qtype_ok(qt)) return fail(NTX_ERR_QTYPE, "%s: unsupported weight type %d", names[i], qt);
    if (!k_ok_fused(qt, K[i]))
      return fail(NTX_ERR_SHAPE, "%s: input length %lld must be a multiple of %d for type %d", names[i],
                  (long long)K[i], qt == NTX_Q6_K ? 2048 : 256, qt);
  }
  if (mat_qt(w, 1) != mat_qt(w, 0) || mat_qt(w, 2) != mat_qt(w, 0))
    return fail(NTX_ERR_QTYPE, "wq, wk and wv must share one block type (one fused GEMV)");
  if (mat_qt(w, 5) != mat_qt(w, 4)) return fail(NTX_ERR_QTYPE, "wg and wu must share one block type (one fused GEMV)");
  return NTX_OK;
}

// ------------------------------------------------------------ workspace
struct Carve {
  uint8_t* base;
  uint64_t off = 0;
  template <class T>
  T* take(uint64_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align256(off + count * sizeof(T));
    return p;
  }
};

int max_parts() { return ntx::sm_count() * 4; }

constexpr int kMaxDraft = 7;  // draft tokens per self-speculative step at most

struct LayerWs {
  float *q, *attn_out, *attn_part, *h1, *u, *stats_in, *stats_o, *stats_down, *cos_tmp;
};

uint64_t carve_layer(const ntx_model_config* c, int n_split, uint8_t* base, LayerWs* w) {
  Carve k{base};
  const int64_t Q = (int64_t)c->n_heads * c->head_dim;
  const int P = max_parts();
  LayerWs t;
  t.q = k.take<float>(Q);
  t.attn_out = k.take<float>(Q);
  t.attn_part = k.take<float>((uint64_t)c->n_heads * n_split * (c->head_dim + 2));
  t.h1 = k.take<float>(c->hidden);
  t.u = k.take<float>(c->ffn);
  t.stats_in = k.take<float>((uint64_t)P * 4);
  t.stats_o = k.take<float>((uint64_t)P * 4);
  t.stats_down = k.take<float>((uint64_t)P * 4);
  t.cos_tmp = k.take<float>(4);
  if (w) *w = t;
  return k.off;
}

}  // namespace

namespace ntx {
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
int record_cuda_error(cudaError_t e, const char* what) { return cuda_fail(e, what); }
}  // namespace ntx

// ======================================================================
extern "C" {

const char* ntx_last_error(void) { return t_err.c_str(); }

int ntx_version(void) { return 100; }

int ntx_device_status(int* code) {
  if (!code) return fail(NTX_ERR_INVALID_ARG, "code is NULL");
  const int e = ntx::read_device_status(code);
  if (e) return cuda_fail((cudaError_t)e, "ntx_device_status");
  return NTX_OK;
}

int ntx_sm_count(void) { return ntx::sm_count(); }

int ntx_check_enabled(void) {
#ifdef NTX_CHECK
  return 1;
#else
  return 0;
#endif
}

int ntx_check_report(int* site, long long* index) {
  if (!site || !index) return fail(NTX_ERR_INVALID_ARG, "site or index is NULL");
  const int e = ntx::read_check_report(site, index);
  if (e) return cuda_fail((cudaError_t)e, "ntx_check_report");
  return NTX_OK;
}

int ntx_dequant(int qtype, const void* blocks, float* out, int64_t n, void* stream) {
  if (!qtype_ok(qtype)) return fail(NTX_ERR_QTYPE, "unsupported weight type %d", qtype);
  if (n < 0 || n % block_elems(qtype)) return fail(NTX_ERR_SHAPE, "n=%lld not a multiple of %d", (long long)n,
                                                   block_elems(qtype));
  if (n == 0) return NTX_OK;
  if (!blocks || !out) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(out, 4)) return fail(NTX_ERR_ALIGN, "out not 4-byte aligned");
  const cudaError_t e = ntx::launch_dequant(qtype, blocks, out, n / block_elems(qtype), S(stream));
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_dequant");
}

int ntx_gemv_q(int qtype, const void* W, int64_t M, int64_t K, const float* x, float* y, const float* residual,
               void* stream) {
  if (!qtype_ok(qtype)) return fail(NTX_ERR_QTYPE, "unsupported weight type %d", qtype);
  if (M < 1 || M > 2147483647LL || K < 1 || K > 262144 || K % block_elems(qtype))
    return fail(NTX_ERR_SHAPE, "bad shape M=%lld K=%lld for type %d", (long long)M, (long long)K, qtype);
  if (!W || !x || !y) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(W, 16) || !aligned(x, 16) || !aligned(y, 16) || (residual && !aligned(residual, 16)))
    return fail(NTX_ERR_ALIGN, "W, x, y, residual must be 16-byte aligned");
  if (ranges_overlap(x, (size_t)K * 4, y, (size_t)M * 4)) return fail(NTX_ERR_INVALID_ARG, "y overlaps x");
  if (residual && residual != y && ranges_overlap(residual, (size_t)M * 4, y, (size_t)M * 4))
    return fail(NTX_ERR_INVALID_ARG, "residual partially overlaps y");
  const cudaError_t e = ntx::launch_gemv(qtype, W, M, K, x, y, residual, S(stream), ntx::gemv_pdl());
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_gemv_q");
}

int ntx_set_gemv_ctas_per_sm(int cps) {
  if (cps < 1 || cps > 4) return fail(NTX_ERR_INVALID_ARG, "ctas per SM must be 1..4");
  ntx::set_gemv_ctas_per_sm(cps);
  return NTX_OK;
}

int ntx_set_persist_two_types(int on) {
  if (on != 0 && on != 1) return fail(NTX_ERR_INVALID_ARG, "two-type persistent switch must be 0 or 1");
  g_persist_two = on;
  return NTX_OK;
}

int ntx_set_gemv_pdl(int on) {
  if (on != 0 && on != 1) return fail(NTX_ERR_INVALID_ARG, "programmatic launch switch must be 0 or 1");
  ntx::set_gemv_pdl(on == 1);
  return NTX_OK;
}

int ntx_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, void* stream) {
  if (n < 1 || n > (1 << 20)) return fail(NTX_ERR_SHAPE, "n=%lld out of range", (long long)n);
  if (!x || !w || !y) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!(eps >= 0.f)) return fail(NTX_ERR_INVALID_ARG, "eps must be >= 0");
  if (!aligned(x, 4) || !aligned(w, 4) || !aligned(y, 4)) return fail(NTX_ERR_ALIGN, "pointers must be 4-byte aligned");
  const cudaError_t e = ntx::launch_rmsnorm(x, w, y, n, eps, S(stream));
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_rmsnorm");
}

int ntx_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int pos, float theta, void* stream) {
  if (head_dim < 2 || head_dim > 256 || head_dim % 2) return fail(NTX_ERR_SHAPE, "head_dim %d", head_dim);
  if (n_q_heads < 0 || n_kv_heads < 0 || pos < 0) return fail(NTX_ERR_INVALID_ARG, "negative heads or pos");
  if ((n_q_heads > 0 && !q) || (n_kv_heads > 0 && !k)) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!(theta > 0.f)) return fail(NTX_ERR_INVALID_ARG, "theta must be > 0");
  const cudaError_t e = ntx::launch_rope(q, k, n_q_heads, n_kv_heads, head_dim, pos, theta, S(stream));
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_rope");
}

size_t ntx_attn_workspace_bytes(int n_q_heads, int n_kv_heads, int head_dim, int max_ctx) {
  if (n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || max_ctx <= 0) return 0;
  const int ns = ntx::attn_splits(n_kv_heads, max_ctx);
  return (size_t)n_q_heads * ns * (head_dim + 2) * sizeof(float);
}

int ntx_attn_decode(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out, int n_q_heads,
                    int n_kv_heads, int head_dim, int n_ctx, int max_ctx, void* workspace, size_t ws_bytes,
                    void* stream) {
  if (head_dim != 128) return fail(NTX_ERR_SHAPE, "head_dim %d unsupported (128 only)", head_dim);
  if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads) return fail(NTX_ERR_SHAPE, "bad head counts");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(NTX_ERR_SHAPE, "query group %d unsupported", G);
  if (n_ctx < 1 || n_ctx > max_ctx) return fail(NTX_ERR_SHAPE, "n_ctx %d outside [1, max_ctx=%d]", n_ctx, max_ctx);
  if (!q || !k_cache || !v_cache || !out || !workspace) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(q, 16) || !aligned(out, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(workspace, 16))
    return fail(NTX_ERR_ALIGN, "q, caches and workspace must be 16-byte aligned");
  if (ws_bytes < ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx))
    return fail(NTX_ERR_NOMEM, "workspace too small (%zu < %zu)", ws_bytes,
                ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx));
  const int ns = ntx::attn_splits(n_kv_heads, n_ctx);
  const cudaError_t e = ntx::launch_attn(q, k_cache, v_cache, out, static_cast<float*>(workspace), n_q_heads,
                                         n_kv_heads, n_ctx, nullptr, max_ctx, ns, S(stream), false);
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_attn_decode");
}

int ntx_swiglu(const float* gate, const float* up, float* out, int64_t n, void* stream) {
  if (n < 0) return fail(NTX_ERR_SHAPE, "n < 0");
  if (n == 0) return NTX_OK;
  if (!gate || !up || !out) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  const cudaError_t e = ntx::launch_swiglu(gate, up, out, n, S(stream));
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_swiglu");
}

int ntx_hbm_read_probe(const void* buf, uint64_t bytes, uint32_t* sum, void* stream) {
  if (!sum || (!buf && bytes)) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (bytes % 16 || reinterpret_cast<uintptr_t>(buf) % 16)
    return fail(NTX_ERR_ALIGN, "buffer must be 16-byte aligned and a multiple of 16 bytes long");
  const cudaError_t e = ntx::launch_read_probe(buf, bytes, sum, S(stream));
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_hbm_read_probe");
}

uint64_t ntx_layer_layout_mixed(const ntx_model_config* cfg, const int32_t* qtypes, ntx_layer_weights* out) {
  if (!cfg || !out || !qtypes || cfg->hidden <= 0 || cfg->ffn <= 0 || cfg->n_heads <= 0 || cfg->n_kv_heads <= 0 ||
      cfg->head_dim <= 0)
    return 0;
  const int64_t H = cfg->hidden, F = cfg->ffn, Q = (int64_t)cfg->n_heads * cfg->head_dim,
                KV = (int64_t)cfg->n_kv_heads * cfg->head_dim;
  const int64_t M[7] = {Q, KV, KV, H, F, F, H}, K[7] = {H, H, H, Q, H, H, F};
  for (int i = 0; i < 7; ++i)
    if (!qtype_ok(qtypes[i]) || K[i] % block_elems(qtypes[i])) return 0;
  ntx_layer_weights w;
  memset(&w, 0, sizeof w);
  w.qtype = NTX_MIXED;
  for (int i = 0; i < 7; ++i) w.mat_qtype[i] = qtypes[i];
  uint64_t* offs[7] = {&w.off_wq, &w.off_wk, &w.off_wv, &w.off_wo, &w.off_wg, &w.off_wu, &w.off_wd};
  uint64_t o = 0;
  for (int i = 0; i < 7; ++i) {
    *offs[i] = o;
    o = align256(o + mat_bytes(qtypes[i], M[i], K[i]));
  }
  w.off_attn_norm = o; o = align256(o + 4 * H);
  w.off_ffn_norm = o; o = align256(o + 4 * H);
  *out = w;
  return o;
}

uint64_t ntx_layer_layout(const ntx_model_config* cfg, int qtype, ntx_layer_weights* out) {
  if (!qtype_ok(qtype)) return 0;
  const int32_t t[7] = {qtype, qtype, qtype, qtype, qtype, qtype, qtype};
  const uint64_t n = ntx_layer_layout_mixed(cfg, t, out);
  if (n) out->qtype = qtype;  // one type: the per-matrix list is informational
  return n;
}

size_t ntx_layer_workspace_bytes(const ntx_model_config* cfg) {
  if (!cfg || cfg->n_kv_heads <= 0 || cfg->max_ctx <= 0) return 0;
  return carve_layer(cfg, ntx::attn_splits(cfg->n_kv_heads, cfg->max_ctx), nullptr, nullptr);
}

}  // extern "C"

namespace {

// Extent of a layer blob given its offsets (for copies and bounds).
uint64_t layer_extent(const ntx_model_config* c, const ntx_layer_weights* w) {
  const int64_t H = c->hidden, F = c->ffn, Q = (int64_t)c->n_heads * c->head_dim,
                KV = (int64_t)c->n_kv_heads * c->head_dim;
  uint64_t e = 0;
  auto upd = [&](uint64_t off, uint64_t n) { if (off + n > e) e = off + n; };
  upd(w->off_wq, mat_bytes(mat_qt(w, 0), Q, H));
  upd(w->off_wk, mat_bytes(mat_qt(w, 1), KV, H));
  upd(w->off_wv, mat_bytes(mat_qt(w, 2), KV, H));
  upd(w->off_wo, mat_bytes(mat_qt(w, 3), H, Q));
  upd(w->off_wg, mat_bytes(mat_qt(w, 4), F, H));
  upd(w->off_wu, mat_bytes(mat_qt(w, 5), F, H));
  upd(w->off_wd, mat_bytes(mat_qt(w, 6), H, F));
  upd(w->off_attn_norm, 4 * H);
  upd(w->off_ffn_norm, 4 * H);
  return e;
}

int check_offsets(const ntx_layer_weights* w) {
  const uint64_t offs[7] = {w->off_wq, w->off_wk, w->off_wv, w->off_wo, w->off_wg, w->off_wu, w->off_wd};
  for (uint64_t o : offs)
    if (o % 16) return fail(NTX_ERR_ALIGN, "weight matrix offsets must be 16-byte aligned");
  if (w->off_attn_norm % 16 || w->off_ffn_norm % 16) return fail(NTX_ERR_ALIGN, "norm offsets must be 16-byte aligned");
  return NTX_OK;
}

ntx::LayerArgs layer_args(const ntx_model_config* c, const uint8_t* base, const ntx_layer_weights* w) {
  ntx::LayerArgs a;
  memset(&a, 0, sizeof a);
  a.qt_qkv = mat_qt(w, 0);
  a.qt_o = mat_qt(w, 3);
  a.qt_gu = mat_qt(w, 4);
  a.qt_down = mat_qt(w, 6);
  a.H = c->hidden; a.Hq = c->n_heads; a.Hkv = c->n_kv_heads; a.D = c->head_dim; a.F = c->ffn;
  a.max_ctx = c->max_ctx; a.eps = c->eps; a.theta = c->theta;
  a.wq = base + w->off_wq; a.wk = base + w->off_wk; a.wv = base + w->off_wv; a.wo = base + w->off_wo;
  a.wg = base + w->off_wg; a.wu = base + w->off_wu; a.wd = base + w->off_wd;
  a.attn_norm = reinterpret_cast<const float*>(base + w->off_attn_norm);
  a.ffn_norm = reinterpret_cast<const float*>(base + w->off_ffn_norm);
  return a;
}

}  // namespace

extern "C" int ntx_decode_layer(const ntx_model_config* cfg, const ntx_layer_weights* w, uint16_t* k_cache,
                                uint16_t* v_cache, float* hidden, int pos, float* cos_out, void* workspace,
                                size_t ws_bytes, void* stream) {
  if (!w) return fail(NTX_ERR_INVALID_ARG, "weights NULL");
  int rc = check_config(cfg, w);
  if (rc) return rc;
  if (!w->base || !k_cache || !v_cache || !hidden || !workspace) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (pos < 0 || pos >= cfg->max_ctx) return fail(NTX_ERR_SHAPE, "pos %d outside [0, max_ctx)", pos);
  if ((rc = check_offsets(w))) return rc;
  if (!aligned(w->base, 16) || !aligned(hidden, 16) || !aligned(workspace, 256) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16))
    return fail(NTX_ERR_ALIGN, "base, hidden, caches must be 16-byte and workspace 256-byte aligned");
  if (ws_bytes < ntx_layer_workspace_bytes(cfg)) return fail(NTX_ERR_NOMEM, "workspace too small");
  const int n_split = ntx::attn_splits(cfg->n_kv_heads, pos + 1);
  LayerWs ws;
  carve_layer(cfg, ntx::attn_splits(cfg->n_kv_heads, cfg->max_ctx), static_cast<uint8_t*>(workspace), &ws);
  ntx::LayerArgs a = layer_args(cfg, static_cast<const uint8_t*>(w->base), w);
  a.k_cache = k_cache; a.v_cache = v_cache; a.hidden = hidden;
  const int nin = ntx::layer_stats_parts(cfg->hidden);
  a.stats_in = ws.stats_in; a.n_stats_in = nin;
  a.stats_o = ws.stats_o; a.stats_down = ws.stats_down;
  a.q = ws.q; a.attn_out = ws.attn_out; a.attn_part = ws.attn_part; a.h1 = ws.h1; a.u = ws.u;
  a.pos = pos; a.pos_dev = nullptr; a.n_split = n_split;
  a.attn_cluster = ntx::attn_cluster_size(cfg->n_heads, cfg->n_kv_heads, cfg->max_ctx);
  cudaStream_t s = S(stream);
  cudaError_t e = ntx::launch_sumsq(hidden, cfg->hidden, ws.stats_in, nin, s, false);
  if (e == cudaSuccess) e = ntx::launch_layer(a, s, true);
  if (e == cudaSuccess && cos_out)
    e = ntx::launch_cos_finalize(ws.stats_down, ntx::layer_stats_parts(cfg->hidden), nullptr, 1, 0, cos_out, s, true);
  return e == cudaSuccess ? NTX_OK : cuda_fail(e, "ntx_decode_layer");
}

// ======================================================================
// Decode engine
struct ntx_engine {
  ntx_model_config cfg;
  std::vector<ntx_layer_weights> layers;
  std::vector<int8_t> tier;
  std::vector<uint64_t> extent;
  uint8_t* slot[2];
  size_t slot_bytes;
  const uint16_t* embed;
  const float* final_norm;
  const void* head;
  int head_qtype;
  std::vector<uint16_t*> kc, vc;
  cudaStream_t cs, xs;
  int n_split;
  int dev;
  // workspace regions
  float *hidden, *q, *attn_out, *attn_part, *h1, *u, *stats_embed, *stats_o, *stats_down, *arg_parts, *cos_int,
      *logits_int;
  int *params, *token_state, *layer_list;
  int64_t stats_stride;  // floats between layers in stats_down
  // pinned parameter ring
  int* pinned;
  cudaEvent_t ring_ev[64];
  int ring_pos;
  cudaEvent_t copy_done[2], slot_free[2], fork_ev, join_ev, sync_ev;
  // skip set
  std::vector<uint8_t> skip;
  bool skip_valid;
  // graphs, keyed by (use_skip | no_persist << 1, logits, next_token, cos_out)
  std::map<std::tuple<int, float*, int32_t*, float*>, cudaGraphExec_t> graphs;
  // profiling probe (kernel-by-kernel steps only) and launch count
  std::vector<cudaEvent_t> probe_b, probe_e;
  int launches;
  // persistent decode kernel (one block type; runs a step whose executed
  // layers are all resident)
  bool persist;       // the plan and launch parameters are valid
  bool persist_full;  // every layer is resident: steps without the skip set
  bool persist_skip;  // every layer of the recorded skip set's run list is resident
  ntx::PStep pst;
  size_t psmem;
  int pgrid;
  ntx::PLayer *pl_all, *pl_skip, *pl_draft;
  int n_skip_run;  // executed layers under the skip set
  // self-speculative decoding: the draft model is the resident layers
  int n_draft;         // resident layers (the draft's run list without a skip set)
  bool persist_draft;  // the draft runs as the persistent kernel over pl_draft
  float* spec_hidden;  // [kMaxDraft + 1][H] residual streams of the verified tokens
  float* spec_stats;   // [kMaxDraft + 1][2][P * 4] their statistics (ping-pong by layer)
  int* spec_tok;       // [kMaxDraft + 1] the token and the draft's proposals
  int* verify_tok;     // [kMaxDraft + 1] the full model's greedy token after each
  unsigned* psync;
  unsigned long long* phase_ts;  // phase probe (kernel-by-kernel steps only)
  size_t phase_ts_words;
};

size_t engine_carve(const ntx_model_config* c, uint8_t* base, ntx_engine* e) {
  Carve k{base};
  const int64_t Q = (int64_t)c->n_heads * c->head_dim;
  const int P = max_parts();
  const int ns = ntx::attn_splits(c->n_kv_heads, c->max_ctx);
  const int ns_p = ntx::persist_splits(ntx::sm_count(), c->n_kv_heads, c->max_ctx);
  const int L = c->n_layers > 0 ? c->n_layers : 1;
  float* hidden = k.take<float>(c->hidden);
  float* q = k.take<float>(Q);
  float* ao = k.take<float>(Q);
  float* ap = k.take<float>((uint64_t)c->n_heads * (ns > ns_p ? ns : ns_p) * (c->head_dim + 2));
  float* h1 = k.take<float>(c->hidden);
  float* u = k.take<float>(c->ffn);
  float* se = k.take<float>((uint64_t)P * 4);
  float* so = k.take<float>((uint64_t)P * 4);
  float* sd = k.take<float>((uint64_t)L * P * 4);
  float* apart = k.take<float>((uint64_t)P * 4);
  float* ci = k.take<float>(L);
  float* li = k.take<float>(c->vocab > 0 ? c->vocab : 1);
  int* params = k.take<int>(4);
  int* ts = k.take<int>(4);
  int* ll = k.take<int>(L);
  ntx::PLayer* pla = k.take<ntx::PLayer>(L);
  ntx::PLayer* pls = k.take<ntx::PLayer>(L);
  ntx::PLayer* pld = k.take<ntx::PLayer>(L);
  unsigned* psync = k.take<unsigned>(ntx::persist_sync_words(L, c->n_kv_heads));
  float* sph = k.take<float>((uint64_t)(kMaxDraft + 1) * c->hidden);
  float* sps = k.take<float>((uint64_t)(kMaxDraft + 1) * 2 * P * 4);
  int* spt = k.take<int>(16);
  int* vft = k.take<int>(16);
  if (e) {
    e->pl_all = pla; e->pl_skip = pls; e->pl_draft = pld; e->psync = psync;
    e->spec_hidden = sph; e->spec_stats = sps; e->spec_tok = spt; e->verify_tok = vft;
    e->hidden = hidden; e->q = q; e->attn_out = ao; e->attn_part = ap; e->h1 = h1; e->u = u;
    e->stats_embed = se; e->stats_o = so; e->stats_down = sd; e->arg_parts = apart; e->cos_int = ci;
    e->logits_int = li; e->params = params; e->token_state = ts; e->layer_list = ll;
    e->stats_stride = (int64_t)P * 4; e->n_split = ns;
  }
  return k.off;
}

extern "C" size_t ntx_engine_workspace_bytes(const ntx_model_config* cfg) {
  if (!cfg || cfg->n_kv_heads <= 0 || cfg->max_ctx <= 0 || cfg->n_layers < 0) return 0;
  return engine_carve(cfg, nullptr, nullptr);
}

namespace {

constexpr int kEmbedParts = 16;

void engine_free(ntx_engine* e) {
  if (!e) return;
  for (auto& kv : e->graphs) cudaGraphExecDestroy(kv.second);
  e->graphs.clear();
  for (int i = 0; i < 64; ++i)
    if (e->ring_ev[i]) cudaEventDestroy(e->ring_ev[i]);
  for (int i = 0; i < 2; ++i) {
    if (e->copy_done[i]) cudaEventDestroy(e->copy_done[i]);
    if (e->slot_free[i]) cudaEventDestroy(e->slot_free[i]);
  }
  if (e->fork_ev) cudaEventDestroy(e->fork_ev);
  if (e->join_ev) cudaEventDestroy(e->join_ev);
  if (e->sync_ev) cudaEventDestroy(e->sync_ev);
  if (e->pinned) cudaFreeHost(e->pinned);
  delete e;
}

// Device table of the executed layers for the persistent kernel.
cudaError_t upload_players(ntx_engine* e, const std::vector<int>& list, ntx::PLayer* dst) {
  std::vector<ntx::PLayer> t(list.size());
  for (size_t i = 0; i < list.size(); ++i) {
    const int l = list[i];
    const ntx::LayerArgs a = layer_args(&e->cfg, static_cast<const uint8_t*>(e->layers[l].base), &e->layers[l]);
    ntx::PLayer& p = t[i];
    p.wq = a.wq; p.wk = a.wk; p.wv = a.wv; p.wo = a.wo; p.wg = a.wg; p.wu = a.wu; p.wd = a.wd;
    p.attn_norm = a.attn_norm; p.ffn_norm = a.ffn_norm;
    p.kc = e->kc[l]; p.vc = e->vc[l];
    p.stats_down = e->stats_down + l * e->stats_stride;
  }
  if (t.empty()) return cudaSuccess;
  return cudaMemcpy(dst, t.data(), sizeof(ntx::PLayer) * t.size(), cudaMemcpyHostToDevice);
}

// The whole step as one persistent kernel (plus the cosine finalisation when
// asked) over the run list `table` of nrun layers (NULL: the skip set's or all).
cudaError_t persist_enqueue(ntx_engine* e, bool use_skip, float* logits, int32_t* next_token, float* cos_out,
                            bool calibrate, bool probe, const ntx::PLayer* table = nullptr, int ntable = 0) {
  const ntx_model_config& c = e->cfg;
  cudaStream_t s = e->cs;
  const bool sk = use_skip && e->skip_valid;
  const int nrun = table ? ntable : sk ? e->n_skip_run : c.n_layers;
  ntx::PStep st = e->pst;
  st.layers = table ? table : sk ? e->pl_skip : e->pl_all;
  st.n_layers = nrun;
  st.logits = logits ? logits : e->logits_int;
  st.next_token = next_token;
  st.head_ctr_index = 2 + 5 * nrun;
  st.abort_index = st.head_ctr_index + nrun * c.n_kv_heads;
  // phase timestamps only in uncaptured steps, and only if the buffer holds them all
  const size_t need = (size_t)(1 + 2 + 5 * nrun) * e->pgrid;
  st.probe_ts = (probe && e->phase_ts && e->phase_ts_words >= need) ? e->phase_ts : nullptr;
  cudaError_t err =
      cudaMemsetAsync(e->psync, 0, sizeof(unsigned) * ntx::persist_sync_words(nrun, c.n_kv_heads), s);
  if (err == cudaSuccess && probe && !e->probe_b.empty()) err = cudaEventRecord(e->probe_b[0], s);
  if (err == cudaSuccess) err = ntx::launch_persist(st,
                                                    e->psmem, e->pgrid, s);
  if (err == cudaSuccess && probe && !e->probe_e.empty()) err = cudaEventRecord(e->probe_e[0], s);
  if (err != cudaSuccess) return err;
  e->launches = 1;
  float* cdst = calibrate ? e->cos_int : cos_out;
  if (cdst && nrun > 0) {
    e->launches += 1;
    err = ntx::launch_cos_finalize(e->stats_down, e->pgrid, sk ? e->layer_list : nullptr, nrun, e->stats_stride, cdst,
                                   s, false);
    if (err == cudaSuccess && calibrate && cos_out)
      err = cudaMemcpyAsync(cos_out, e->cos_int, sizeof(float) * c.n_layers, cudaMemcpyDeviceToDevice, s);
  }
  return err;
}

// Enqueue the per-token launch sequence (everything after the parameter copy).
cudaError_t engine_enqueue(ntx_engine* e, bool use_skip, float* logits, int32_t* next_token, float* cos_out,
                           bool calibrate, bool probe, bool no_persist, bool draft = false) {
  if (draft) {  // the resident layers only (minus the skip set): no host layer, no cosines
    const bool sk = use_skip && e->skip_valid;
    if (e->persist_draft && !no_persist && !sk)
      return persist_enqueue(e, false, logits, next_token, nullptr, false, false, e->pl_draft, e->n_draft);
    if (e->persist_draft && !no_persist && sk && e->persist_skip)  // the skip run list is all resident
      return persist_enqueue(e, true, logits, next_token, nullptr, false, false, e->pl_skip, e->n_skip_run);
    cos_out = nullptr;
    calibrate = false;
  } else if (e->persist && !no_persist) {
    const bool sk = use_skip && e->skip_valid;
    if (sk ? e->persist_skip : e->persist_full)
      return persist_enqueue(e, use_skip, logits, next_token, cos_out, calibrate, probe);
  }
  const ntx_model_config& c = e->cfg;
  cudaStream_t s = e->cs;
  const bool pdl = true;
  cudaError_t err = ntx::launch_embed(e->embed, c.hidden, c.vocab, e->params + 1, e->token_state, e->hidden,
                                      e->stats_embed, kEmbedParts, s, pdl);
  if (err != cudaSuccess) return err;
  const float* stats_in = e->stats_embed;
  int n_in = kEmbedParts;
  const int nparts = ntx::layer_stats_parts(c.hidden);

  // host-tier layers in execution order
  std::vector<int> host_layers;
  for (int l = 0; l < c.n_layers; ++l)
    if (e->tier[l] == 1 && !(use_skip && e->skip[l]) && !draft) host_layers.push_back(l);
  auto issue_copy = [&](int k) -> cudaError_t {
    const int l = host_layers[k], sl = k & 1;
    cudaError_t r = cudaStreamWaitEvent(e->xs, e->slot_free[sl], 0);
    if (r == cudaSuccess)
      r = cudaMemcpyAsync(e->slot[sl], e->layers[l].base, e->extent[l], cudaMemcpyHostToDevice, e->xs);
    if (r == cudaSuccess) r = cudaEventRecord(e->copy_done[sl], e->xs);
    return r;
  };
  if (!host_layers.empty()) {
    // fork the copy stream from the compute stream; both slots start free
    err = cudaEventRecord(e->fork_ev, s);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(e->xs, e->fork_ev, 0);
    if (err == cudaSuccess) err = cudaEventRecord(e->slot_free[0], s);
    if (err == cudaSuccess) err = cudaEventRecord(e->slot_free[1], s);
    for (int k = 0; k < (int)host_layers.size() && k < 2 && err == cudaSuccess; ++k) err = issue_copy(k);
    if (err != cudaSuccess) return err;
  }
  int hk = 0;  // index into host_layers
  std::vector<int> computed;
  for (int l = 0; l < c.n_layers; ++l) {
    if ((use_skip && e->skip[l]) || (draft && e->tier[l] == 1)) continue;
    const uint8_t* base = static_cast<const uint8_t*>(e->layers[l].base);
    bool on_host = e->tier[l] == 1;
    if (on_host) {
      const int sl = hk & 1;
      err = cudaStreamWaitEvent(s, e->copy_done[sl], 0);
      if (err != cudaSuccess) return err;
      base = e->slot[sl];
    }
    ntx::LayerArgs a = layer_args(&c, base, &e->layers[l]);
    a.k_cache = e->kc[l]; a.v_cache = e->vc[l]; a.hidden = e->hidden;
    a.stats_in = stats_in; a.n_stats_in = n_in;
    a.stats_o = e->stats_o;
    a.stats_down = e->stats_down + l * e->stats_stride;
    a.q = e->q; a.attn_out = e->attn_out; a.attn_part = e->attn_part; a.h1 = e->h1; a.u = e->u;
    a.pos = 0; a.pos_dev = e->params; a.n_split = e->n_split;
    a.attn_cluster = ntx::attn_cluster_size(c.n_heads, c.n_kv_heads, c.max_ctx);
    const size_t k = computed.size();
    if (probe && k < e->probe_b.size()) {
      a.probe_begin = e->probe_b[k];
      a.probe_end = e->probe_e[k];
    }
    err = ntx::launch_layer(a, s, pdl);
    if (err != cudaSuccess) return err;
    stats_in = a.stats_down;
    n_in = nparts;
    computed.push_back(l);
    if (on_host) {
      err = cudaEventRecord(e->slot_free[hk & 1], s);
      if (err == cudaSuccess && hk + 2 < (int)host_layers.size()) err = issue_copy(hk + 2);
      if (err != cudaSuccess) return err;
      ++hk;
    }
  }
  if (!host_layers.empty()) {
    err = cudaEventRecord(e->join_ev, e->xs);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(s, e->join_ev, 0);
    if (err != cudaSuccess) return err;
  }
  err = ntx::launch_head(e->head_qtype, e->head, c.vocab, c.hidden, e->hidden, e->final_norm, stats_in, n_in, c.eps,
                         logits ? logits : e->logits_int, e->arg_parts, s, pdl);
  if (err != cudaSuccess) return err;
  err = ntx::launch_argmax_finalize(e->arg_parts, ntx::head_parts(c.vocab), e->token_state, next_token, s, pdl);
  if (err != cudaSuccess) return err;
  ntx::LayerArgs probe_args;
  memset(&probe_args, 0, sizeof probe_args);
  probe_args.attn_cluster = ntx::attn_cluster_size(c.n_heads, c.n_kv_heads, c.max_ctx);
  e->launches = 1 + ntx::layer_launches(probe_args) * (int)computed.size() + 2;
  float* cdst = calibrate ? e->cos_int : cos_out;
  if (cdst && !computed.empty()) {
    e->launches += 1;
    // the layer list is the identity when nothing is skipped
    const int* list = (use_skip && e->skip_valid) ? e->layer_list : nullptr;
    err = ntx::launch_cos_finalize(e->stats_down, nparts, list, (int)computed.size(), e->stats_stride, cdst, s, pdl);
    if (err == cudaSuccess && calibrate && cos_out)
      err = cudaMemcpyAsync(cos_out, e->cos_int, sizeof(float) * c.n_layers, cudaMemcpyDeviceToDevice, s);
  }
  return err;
}

}  // namespace

extern "C" int ntx_engine_create(const ntx_model_config* cfg, const ntx_layer_weights* layers, const int8_t* tier_map,
                                 void* slot0, void* slot1, size_t slot_bytes, const uint16_t* embed,
                                 const float* final_norm, const void* head, int head_qtype,
                                 uint16_t* const* k_caches, uint16_t* const* v_caches, void* workspace,
                                 size_t ws_bytes, void* compute_stream, void* copy_stream, ntx_engine** out) {
  if (!out) return fail(NTX_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg || (cfg->n_layers > 0 && (!layers || !k_caches || !v_caches)))
    return fail(NTX_ERR_INVALID_ARG, "NULL config, layers or caches");
  int rc = check_dims(cfg);
  if (rc) return rc;
  if (!qtype_ok(head_qtype) || !k_ok_fused(head_qtype, cfg->hidden))
    return fail(NTX_ERR_QTYPE, "unsupported head type %d for hidden %d", head_qtype, cfg->hidden);
  if (cfg->vocab <= 0) return fail(NTX_ERR_SHAPE, "vocab must be > 0");
  if (!embed || !final_norm || !head || !workspace) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  if (!compute_stream) return fail(NTX_ERR_INVALID_ARG, "compute_stream must be a created (non-default) stream");
  if (!aligned(workspace, 256) || !aligned(head, 16) || !aligned(final_norm, 16))
    return fail(NTX_ERR_ALIGN, "workspace 256-byte, head and final_norm 16-byte aligned");
  if (ws_bytes < ntx_engine_workspace_bytes(cfg)) return fail(NTX_ERR_NOMEM, "workspace too small");
  bool any_host = false;
  for (int l = 0; l < cfg->n_layers; ++l) {
    if ((rc = check_config(cfg, &layers[l]))) return rc;
    if ((rc = check_offsets(&layers[l]))) return rc;
    if (!layers[l].base || !k_caches[l] || !v_caches[l]) return fail(NTX_ERR_INVALID_ARG, "layer %d: NULL pointer", l);
    const int t = tier_map ? tier_map[l] : 0;
    if (t != 0 && t != 1) return fail(NTX_ERR_INVALID_ARG, "tier_map[%d] = %d (0 or 1)", l, t);
    if (t == 1) any_host = true;
    if (!aligned(layers[l].base, 16)) return fail(NTX_ERR_ALIGN, "layer %d base not 16-byte aligned", l);
  }
  if (any_host && (!slot0 || !slot1 || !copy_stream || copy_stream == compute_stream || !aligned(slot0, 256) ||
                   !aligned(slot1, 256)))
    return fail(NTX_ERR_INVALID_ARG, "host-tier layers need two 256-byte aligned slots and a separate copy stream");
  ntx_engine* e = new (std::nothrow) ntx_engine();
  if (!e) return fail(NTX_ERR_NOMEM, "engine allocation");
  e->cfg = *cfg;
  e->layers.assign(layers, layers + cfg->n_layers);
  e->tier.resize(cfg->n_layers);
  e->extent.resize(cfg->n_layers);
  for (int l = 0; l < cfg->n_layers; ++l) {
    e->tier[l] = tier_map ? tier_map[l] : 0;
    e->extent[l] = layer_extent(cfg, &layers[l]);
    if (e->tier[l] == 1 && e->extent[l] > slot_bytes) {
      engine_free(e);
      return fail(NTX_ERR_NOMEM, "layer %d (%llu bytes) does not fit a slot of %zu bytes", l,
                  (unsigned long long)e->extent[l], slot_bytes);
    }
  }
  e->slot[0] = static_cast<uint8_t*>(slot0);
  e->slot[1] = static_cast<uint8_t*>(slot1);
  e->slot_bytes = slot_bytes;
  e->embed = embed; e->final_norm = final_norm; e->head = head; e->head_qtype = head_qtype;
  e->kc.assign(k_caches, k_caches + cfg->n_layers);
  e->vc.assign(v_caches, v_caches + cfg->n_layers);
  e->cs = S(compute_stream);
  e->xs = S(copy_stream);
  cudaGetDevice(&e->dev);
  engine_carve(cfg, static_cast<uint8_t*>(workspace), e);
  e->skip.assign(cfg->n_layers, 0);
  e->skip_valid = false;
  if (fault("pinned_alloc")) {
    engine_free(e);
    return fail(NTX_ERR_NOMEM, "ntx_engine_create: pinned parameter block allocation failed (injected)");
  }
  cudaError_t err = cudaHostAlloc(reinterpret_cast<void**>(&e->pinned), (64 * 4 + 64) * sizeof(int),
                                  cudaHostAllocDefault);
  for (int i = 0; i < 64 && err == cudaSuccess; ++i) err = cudaEventCreateWithFlags(&e->ring_ev[i], cudaEventDisableTiming);
  for (int i = 0; i < 2 && err == cudaSuccess; ++i) {
    err = cudaEventCreateWithFlags(&e->copy_done[i], cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->slot_free[i], cudaEventDisableTiming);
  }
  if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->fork_ev, cudaEventDisableTiming);
  if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->join_ev, cudaEventDisableTiming);
  if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->sync_ev, cudaEventDisableTiming);
  // persistent kernel: each GEMV phase kind (Q/K/V, O, gate/up, down, head) of one block type over all
  // layers, a type pair it is built for, shapes and alignment it handles; it runs the steps whose executed
  // layers are all resident (all steps without a host tier; with one, the steps under a skip set that skips
  // every host layer)
  e->persist = e->persist_full = e->persist_skip = e->persist_draft = false;
  e->n_draft = 0;
  for (int l = 0; l < cfg->n_layers; ++l) e->n_draft += e->tier[l] == 0;
  int kt[7] = {0, 0, 0, 0, 0, 0, 0};
  kt[ntx::PK_HEAD] = head_qtype;
  bool uniform = true;
  if (cfg->n_layers > 0) {
    kt[ntx::PK_QKV] = mat_qt(&layers[0], 0);
    kt[ntx::PK_O] = mat_qt(&layers[0], 3);
    kt[ntx::PK_GU] = mat_qt(&layers[0], 4);
    kt[ntx::PK_DOWN] = mat_qt(&layers[0], 6);
  } else {
    kt[ntx::PK_QKV] = kt[ntx::PK_O] = kt[ntx::PK_GU] = kt[ntx::PK_DOWN] = head_qtype;
  }
  for (int l = 1; l < cfg->n_layers && uniform; ++l)
    uniform = mat_qt(&layers[l], 0) == kt[ntx::PK_QKV] && mat_qt(&layers[l], 3) == kt[ntx::PK_O] &&
              mat_qt(&layers[l], 4) == kt[ntx::PK_GU] && mat_qt(&layers[l], 6) == kt[ntx::PK_DOWN];
  bool one_type = true;
  for (int k : {ntx::PK_O, ntx::PK_GU, ntx::PK_DOWN, ntx::PK_HEAD}) one_type = one_type && kt[k] == kt[ntx::PK_QKV];
  if (err == cudaSuccess && uniform && (one_type || g_persist_two.load())) {
    ntx::PStep st;
    memset(&st, 0, sizeof st);
    size_t psm = 0;
    if (ntx::persist_plan(kt, cfg->hidden, cfg->n_heads, cfg->n_kv_heads, cfg->head_dim, cfg->ffn, cfg->vocab,
                          cfg->max_ctx, ntx::sm_count(), cfg->n_layers, &st, &psm) == 0) {
      const int grid = ntx::persist_grid(st, psm);
      bool ok = grid > 0 && grid == ntx::sm_count() && ntx::gemv_tma_ok(head_qtype, head, cfg->hidden);
      for (int l = 0; l < cfg->n_layers && ok; ++l) {
        const ntx::LayerArgs a = layer_args(cfg, static_cast<const uint8_t*>(layers[l].base), &layers[l]);
        const int64_t KO = (int64_t)cfg->n_heads * cfg->head_dim;
        ok = ntx::gemv_tma_ok(a.qt_qkv, a.wq, cfg->hidden) && ntx::gemv_tma_ok(a.qt_qkv, a.wk, cfg->hidden) &&
             ntx::gemv_tma_ok(a.qt_qkv, a.wv, cfg->hidden) && ntx::gemv_tma_ok(a.qt_o, a.wo, KO) &&
             ntx::gemv_tma_ok(a.qt_gu, a.wg, cfg->hidden) && ntx::gemv_tma_ok(a.qt_gu, a.wu, cfg->hidden) &&
             ntx::gemv_tma_ok(a.qt_down, a.wd, cfg->ffn) && aligned(a.attn_norm, 16) &&
             aligned(a.ffn_norm, 16) && aligned(e->kc[l], 16) && aligned(e->vc[l], 16);
      }
      if (ok) {
        st.H = cfg->hidden; st.Hq = cfg->n_heads; st.Hkv = cfg->n_kv_heads; st.D = cfg->head_dim; st.F = cfg->ffn;
        st.V = cfg->vocab; st.max_ctx = cfg->max_ctx; st.eps = cfg->eps; st.theta = cfg->theta;
        st.embed = embed; st.final_norm = final_norm; st.head = static_cast<const uint8_t*>(head);
        st.hidden = e->hidden; st.q = e->q; st.attn_out = e->attn_out; st.attn_part = e->attn_part;
        st.h1 = e->h1; st.u = e->u; st.stats_embed = e->stats_embed; st.stats_o = e->stats_o;
        st.arg_parts = e->arg_parts; st.params = e->params; st.token_state = e->token_state;
        st.sync = e->psync;
        st.n_split = ntx::persist_splits(grid, cfg->n_kv_heads, cfg->max_ctx);
        st.status = ntx::device_status_ptr();
        st.wait_ns = ntx::kDefaultWaitNs;
        st.stall_cta = -1;
        if (!any_host) {
          std::vector<int> all(cfg->n_layers);
          for (int l = 0; l < cfg->n_layers; ++l) all[l] = l;
          err = upload_players(e, all, e->pl_all);
        }
        std::vector<int> resident;
        for (int l = 0; l < cfg->n_layers; ++l)
          if (e->tier[l] == 0) resident.push_back(l);
        if (err == cudaSuccess && !resident.empty()) {
          err = upload_players(e, resident, e->pl_draft);
          e->persist_draft = err == cudaSuccess;
        }
        if (err == cudaSuccess) {
          e->pst = st;
          e->psmem = psm;
          e->pgrid = grid;
          e->persist = true;
          e->persist_full = !any_host;
        }
      }
    }
  }
  // token state starts at 0
  if (err == cudaSuccess) err = cudaMemsetAsync(e->token_state, 0, 4 * sizeof(int), e->cs);
  if (err == cudaSuccess) {
    err = wait_stream(e->cs, e->sync_ev);
    if (err == cudaErrorTimeout) return wait_fail(err, "ntx_engine_create");  // work in flight: leak, do not free
  }
  if (err != cudaSuccess) {
    engine_free(e);
    return cuda_fail(err, "ntx_engine_create");
  }
  *out = e;
  return NTX_OK;
}

namespace {

// Step parameters (position, token) through a ring of pinned host slots to the
// device words the kernels read, on the compute stream.
int enqueue_params(ntx_engine* e, int pos, int token) {
  const int slot = e->ring_pos;
  cudaError_t err = wait_event(e->ring_ev[slot]);
  if (err != cudaSuccess) return wait_fail(err, "param ring");
  e->ring_pos = (e->ring_pos + 1) % 64;
  e->pinned[slot * 4 + 0] = pos;
  e->pinned[slot * 4 + 1] = token;
  err = cudaMemcpyAsync(e->params, e->pinned + slot * 4, 2 * sizeof(int), cudaMemcpyHostToDevice, e->cs);
  if (err == cudaSuccess) err = cudaEventRecord(e->ring_ev[slot], e->cs);
  if (err != cudaSuccess) return cuda_fail(err, "param copy");
  return NTX_OK;
}

}  // namespace

extern "C" int ntx_decode_step(ntx_engine* e, int32_t token, int pos, float* logits, int32_t* next_token, int flags,
                               float* cos_out) {
  if (!e) return fail(NTX_ERR_INVALID_ARG, "engine is NULL");
  const ntx_model_config& c = e->cfg;
  if (pos < 0 || pos >= c.max_ctx) return fail(NTX_ERR_SHAPE, "pos %d outside [0, max_ctx=%d)", pos, c.max_ctx);
  if (token < -1 || token >= c.vocab) return fail(NTX_ERR_INVALID_ARG, "token %d outside [-1, vocab)", token);
  if (flags & ~(NTX_CALIBRATE_SKIP | NTX_USE_SKIP | NTX_NO_GRAPH | NTX_NO_PERSIST))
    return fail(NTX_ERR_INVALID_ARG, "unknown flags");
  const bool no_persist = (flags & NTX_NO_PERSIST) != 0;
  const bool calibrate = flags & NTX_CALIBRATE_SKIP;
  const bool use_skip = !calibrate && (flags & NTX_USE_SKIP) && e->skip_valid;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != e->dev) return fail(NTX_ERR_INVALID_ARG, "engine was created on device %d, current is %d", e->dev, cur);

  // a step that streams host layers: the copies are submitted below (injected failure: nothing enqueued)
  if (fault("h2d_submit")) {
    bool streams = false;
    for (int l = 0; l < c.n_layers && !streams; ++l)
      streams = e->tier[l] == 1 && !(use_skip && e->skip[l]);
    if (streams) return fail(NTX_ERR_CUDA, "ntx_decode_step: host-to-device copy submission failed (injected)");
  }
  // step parameters: pinned ring slot -> device
  int rc = enqueue_params(e, pos, token);
  if (rc) return rc;
  cudaError_t err = cudaSuccess;

  if ((flags & NTX_NO_GRAPH) || calibrate) {
    err = engine_enqueue(e, use_skip, logits, next_token, cos_out, calibrate, (flags & NTX_NO_GRAPH) != 0,
                         no_persist);
    if (err != cudaSuccess) return cuda_fail(err, "ntx_decode_step");
  } else {
    const auto key = std::make_tuple((use_skip ? 1 : 0) | (no_persist ? 2 : 0), logits, next_token, cos_out);
    auto it = e->graphs.find(key);
    if (it == e->graphs.end()) {
      cudaGraph_t g = nullptr;
      err = cudaStreamBeginCapture(e->cs, cudaStreamCaptureModeThreadLocal);
      if (err != cudaSuccess) return cuda_fail(err, "begin capture");
      const cudaError_t err_enq = engine_enqueue(e, use_skip, logits, next_token, cos_out, false, false, no_persist);
      err = cudaStreamEndCapture(e->cs, &g);
      if (err_enq != cudaSuccess || err != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        return cuda_fail(err_enq != cudaSuccess ? err_enq : err, "capture of the decode step");
      }
      cudaGraphExec_t ge = nullptr;
      err = cudaGraphInstantiate(&ge, g, 0);
      cudaGraphDestroy(g);
      if (err != cudaSuccess) return cuda_fail(err, "graph instantiate");
      it = e->graphs.emplace(key, ge).first;
    }
    err = cudaGraphLaunch(it->second, e->cs);
    if (err != cudaSuccess) return cuda_fail(err, "graph launch");
  }

  if (calibrate) {
    std::vector<float> cs(c.n_layers);
    err = cudaMemcpyAsync(cs.data(), e->cos_int, sizeof(float) * c.n_layers, cudaMemcpyDeviceToHost, e->cs);
    if (err == cudaSuccess) err = wait_stream(e->cs, e->sync_ev);
    if (err != cudaSuccess) return wait_fail(err, "calibration read-back");
    std::vector<int> list;
    for (int l = 0; l < c.n_layers; ++l) {
      e->skip[l] = cs[l] >= c.skip_threshold ? 1 : 0;
      if (!e->skip[l]) list.push_back(l);
    }
    bool all_resident = true;
    for (int l : list) all_resident = all_resident && e->tier[l] == 0;
    e->persist_skip = false;
    if (!list.empty()) {
      err = cudaMemcpy(e->layer_list, list.data(), sizeof(int) * list.size(), cudaMemcpyHostToDevice);
      if (err == cudaSuccess && e->persist && all_resident) err = upload_players(e, list, e->pl_skip);
      if (err != cudaSuccess) return cuda_fail(err, "layer list");
    }
    e->persist_skip = e->persist && all_resident;
    e->n_skip_run = (int)list.size();
    e->skip_valid = true;
    // graphs built with an older skip set are stale
    for (auto itg = e->graphs.begin(); itg != e->graphs.end();) {
      if (std::get<0>(itg->first) & 1) {
        cudaGraphExecDestroy(itg->second);
        itg = e->graphs.erase(itg);
      } else {
        ++itg;
      }
    }
  }
  return NTX_OK;
}

namespace {

// The verification pass of a self-speculative step: the tokens spec_tok[0..k]
// at positions pos..pos+k through every executed layer, layer by layer (each
// host layer crosses the link once for all k+1 tokens), then the head and the
// greedy token of each into verify_tok[0..k].  The kernels and their order
// for one token are those of an ordinary per-op step, so each token's logits
// are the ones an ordinary step at that position would give.
cudaError_t verify_enqueue(ntx_engine* e, int pos, int k, bool use_skip) {
  const ntx_model_config& c = e->cfg;
  cudaStream_t s = e->cs;
  const bool pdl = true;
  const int P4 = max_parts() * 4;
  const int nparts = ntx::layer_stats_parts(c.hidden);
  auto hid = [&](int t) { return e->spec_hidden + (int64_t)t * c.hidden; };
  auto stats = [&](int t, int par) { return e->spec_stats + ((int64_t)t * 2 + par) * P4; };
  cudaError_t err = cudaSuccess;
  for (int t = 0; t <= k && err == cudaSuccess; ++t)
    err = ntx::launch_embed(e->embed, c.hidden, c.vocab, e->spec_tok + t, e->token_state, hid(t), stats(t, 0),
                            kEmbedParts, s, pdl);
  if (err != cudaSuccess) return err;
  std::vector<int> host_layers;
  for (int l = 0; l < c.n_layers; ++l)
    if (e->tier[l] == 1 && !(use_skip && e->skip[l])) host_layers.push_back(l);
  auto issue_copy = [&](int j) -> cudaError_t {
    const int l = host_layers[j], sl = j & 1;
    cudaError_t r = cudaStreamWaitEvent(e->xs, e->slot_free[sl], 0);
    if (r == cudaSuccess)
      r = cudaMemcpyAsync(e->slot[sl], e->layers[l].base, e->extent[l], cudaMemcpyHostToDevice, e->xs);
    if (r == cudaSuccess) r = cudaEventRecord(e->copy_done[sl], e->xs);
    return r;
  };
  if (!host_layers.empty()) {
    err = cudaEventRecord(e->fork_ev, s);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(e->xs, e->fork_ev, 0);
    if (err == cudaSuccess) err = cudaEventRecord(e->slot_free[0], s);
    if (err == cudaSuccess) err = cudaEventRecord(e->slot_free[1], s);
    for (int j = 0; j < (int)host_layers.size() && j < 2 && err == cudaSuccess; ++j) err = issue_copy(j);
    if (err != cudaSuccess) return err;
  }
  int hk = 0, par = 0, n_in = kEmbedParts;
  for (int l = 0; l < c.n_layers; ++l) {
    if (use_skip && e->skip[l]) continue;
    const uint8_t* base = static_cast<const uint8_t*>(e->layers[l].base);
    const bool on_host = e->tier[l] == 1;
    if (on_host) {
      err = cudaStreamWaitEvent(s, e->copy_done[hk & 1], 0);
      if (err != cudaSuccess) return err;
      base = e->slot[hk & 1];
    }
    for (int t = 0; t <= k; ++t) {
      ntx::LayerArgs a = layer_args(&c, base, &e->layers[l]);
      a.k_cache = e->kc[l]; a.v_cache = e->vc[l]; a.hidden = hid(t);
      a.stats_in = stats(t, par); a.n_stats_in = n_in;
      a.stats_o = e->stats_o;
      a.stats_down = stats(t, par ^ 1);
      a.q = e->q; a.attn_out = e->attn_out; a.attn_part = e->attn_part; a.h1 = e->h1; a.u = e->u;
      a.pos = pos + t; a.pos_dev = nullptr; a.n_split = e->n_split;
      a.attn_cluster = ntx::attn_cluster_size(c.n_heads, c.n_kv_heads, c.max_ctx);
      err = ntx::launch_layer(a, s, pdl);
      if (err != cudaSuccess) return err;
    }
    par ^= 1;
    n_in = nparts;
    if (on_host) {
      err = cudaEventRecord(e->slot_free[hk & 1], s);
      if (err == cudaSuccess && hk + 2 < (int)host_layers.size()) err = issue_copy(hk + 2);
      if (err != cudaSuccess) return err;
      ++hk;
    }
  }
  if (!host_layers.empty()) {
    err = cudaEventRecord(e->join_ev, e->xs);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(s, e->join_ev, 0);
    if (err != cudaSuccess) return err;
  }
  for (int t = 0; t <= k && err == cudaSuccess; ++t) {
    err = ntx::launch_head(e->head_qtype, e->head, c.vocab, c.hidden, hid(t), e->final_norm, stats(t, par), n_in,
                           c.eps, e->logits_int, e->arg_parts, s, pdl);
    if (err == cudaSuccess)
      err = ntx::launch_argmax_finalize(e->arg_parts, ntx::head_parts(c.vocab), e->token_state, e->verify_tok + t, s,
                                        pdl);
  }
  return err;
}

}  // namespace

extern "C" int ntx_decode_spec(ntx_engine* e, int32_t token, int pos, int draft_k, int32_t* tokens_out, int* n_out,
                               int flags) {
  if (!e || !tokens_out || !n_out) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  const ntx_model_config& c = e->cfg;
  if (draft_k < 1 || draft_k > kMaxDraft) return fail(NTX_ERR_INVALID_ARG, "draft_k %d outside [1, %d]", draft_k, kMaxDraft);
  if (pos < 0 || pos + draft_k >= c.max_ctx)
    return fail(NTX_ERR_SHAPE, "positions %d..%d outside [0, max_ctx=%d)", pos, pos + draft_k, c.max_ctx);
  if (token < 0 || token >= c.vocab) return fail(NTX_ERR_INVALID_ARG, "token %d outside [0, vocab)", token);
  if (flags & ~(NTX_USE_SKIP | NTX_NO_PERSIST)) return fail(NTX_ERR_INVALID_ARG, "unknown flags");
  const bool use_skip = (flags & NTX_USE_SKIP) && e->skip_valid;
  int n_res = 0, n_host = 0;
  for (int l = 0; l < c.n_layers; ++l) {
    if (use_skip && e->skip[l]) continue;
    if (e->tier[l] == 0) ++n_res;
    else ++n_host;
  }
  if (n_res == 0 || n_host == 0)
    return fail(NTX_ERR_INVALID_ARG,
                "self-speculative decoding needs executed layers in both tiers (the resident ones are the draft)");
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != e->dev) return fail(NTX_ERR_INVALID_ARG, "engine was created on device %d, current is %d", e->dev, cur);
  if (fault("h2d_submit")) return fail(NTX_ERR_CUDA, "ntx_decode_spec: host-to-device copy submission failed (injected)");
  cudaStream_t s = e->cs;
  int* hp = e->pinned + 64 * 4;  // [0..15] read-back area, [16] token
  // the pinned read-back area is reused: the previous call's copies have completed (it waited for them)
  hp[16] = token;
  cudaError_t err = cudaMemcpyAsync(e->spec_tok, hp + 16, sizeof(int), cudaMemcpyHostToDevice, s);
  if (err != cudaSuccess) return cuda_fail(err, "ntx_decode_spec: token copy");
  // draft: k steps of the resident layers, each proposing the next token
  for (int i = 0; i < draft_k; ++i) {
    int rc = enqueue_params(e, pos + i, i == 0 ? token : -1);
    if (rc) return rc;
    err = engine_enqueue(e, use_skip, nullptr, e->spec_tok + i + 1, nullptr, false, false,
                         (flags & NTX_NO_PERSIST) != 0, true);
    if (err != cudaSuccess) return cuda_fail(err, "ntx_decode_spec: draft step");
  }
  // verification of the token and the k proposals by the whole model
  err = verify_enqueue(e, pos, draft_k, use_skip);
  if (err != cudaSuccess) return cuda_fail(err, "ntx_decode_spec: verification");
  err = cudaMemcpyAsync(hp, e->spec_tok, sizeof(int) * (draft_k + 1), cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess)
    err = cudaMemcpyAsync(hp + 8, e->verify_tok, sizeof(int) * (draft_k + 1), cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess) err = wait_stream(s, e->sync_ev);
  if (err != cudaSuccess) return wait_fail(err, "ntx_decode_spec: read-back");
  // accept the longest prefix of proposals the whole model agrees with, then its own next token
  int n = 0;
  while (n < draft_k && hp[1 + n] == hp[8 + n]) ++n;
  for (int i = 0; i <= n; ++i) tokens_out[i] = hp[8 + i];
  *n_out = n + 1;
  // the engine's greedy state continues from the last emitted token
  err = cudaMemcpyAsync(e->token_state, hp + 8 + n, sizeof(int), cudaMemcpyHostToDevice, s);
  if (err == cudaSuccess) err = wait_stream(s, e->sync_ev);
  if (err != cudaSuccess) return wait_fail(err, "ntx_decode_spec: token state");
  e->launches = -1;  // not a single-step launch sequence
  return NTX_OK;
}

extern "C" int ntx_engine_skip_mask(ntx_engine* e, uint8_t* mask_host) {
  if (!e || !mask_host) return fail(NTX_ERR_INVALID_ARG, "NULL pointer");
  int n = 0;
  for (int l = 0; l < e->cfg.n_layers; ++l) {
    mask_host[l] = e->skip_valid ? e->skip[l] : 0;
    n += mask_host[l];
  }
  return n;
}

extern "C" int ntx_engine_set_probe(ntx_engine* e, void* const* begin_events, void* const* end_events, int n) {
  if (!e) return fail(NTX_ERR_INVALID_ARG, "engine is NULL");
  if (n < 0 || (n > 0 && (!begin_events || !end_events))) return fail(NTX_ERR_INVALID_ARG, "bad probe arrays");
  e->probe_b.clear();
  e->probe_e.clear();
  for (int k = 0; k < n; ++k) {
    if (!begin_events[k] || !end_events[k]) return fail(NTX_ERR_INVALID_ARG, "probe event %d is NULL", k);
    e->probe_b.push_back(static_cast<cudaEvent_t>(begin_events[k]));
    e->probe_e.push_back(static_cast<cudaEvent_t>(end_events[k]));
  }
  return NTX_OK;
}

extern "C" int ntx_engine_set_phase_probe(ntx_engine* e, unsigned long long* dev_ts, size_t n_words) {
  if (!e) return fail(NTX_ERR_INVALID_ARG, "engine is NULL");
  if (n_words && !dev_ts) return fail(NTX_ERR_INVALID_ARG, "NULL probe buffer with nonzero size");
  if (dev_ts && !aligned(dev_ts, 8)) return fail(NTX_ERR_ALIGN, "probe buffer must be 8-byte aligned");
  e->phase_ts = n_words ? dev_ts : nullptr;
  e->phase_ts_words = n_words;
  return (e->persist_full || e->persist_skip) ? e->pgrid : 0;
}

extern "C" int ntx_persistent_plan(const ntx_model_config* cfg, int qtype, int* slot_bytes, int* n_slots,
                                   size_t* smem_bytes, int* rows_per_slot) {
  if (!cfg || cfg->hidden <= 0 || cfg->n_heads <= 0 || cfg->n_kv_heads <= 0 || cfg->head_dim <= 0 || cfg->ffn <= 0 ||
      cfg->vocab <= 0 || cfg->n_layers <= 0 || cfg->max_ctx <= 0)
    return fail(NTX_ERR_INVALID_ARG, "NULL or non-positive model config");
  if (!qtype_ok(qtype)) return fail(NTX_ERR_QTYPE, "unsupported weight type %d", qtype);
  ntx::PStep st;
  memset(&st, 0, sizeof st);
  size_t smem = 0;
  const int kt[7] = {qtype, qtype, qtype, qtype, qtype, qtype, qtype};
  if (ntx::persist_plan(kt, cfg->hidden, cfg->n_heads, cfg->n_kv_heads, cfg->head_dim, cfg->ffn, cfg->vocab,
                        cfg->max_ctx, ntx::sm_count(), cfg->n_layers, &st, &smem) != 0)
    return fail(NTX_ERR_SHAPE, "the persistent kernel does not take this model");
  if (slot_bytes) *slot_bytes = st.slot_bytes;
  if (n_slots) *n_slots = st.n_slots;
  if (smem_bytes) *smem_bytes = smem;
  if (rows_per_slot) {
    const int kinds[5] = {ntx::PK_QKV, ntx::PK_O, ntx::PK_GU, ntx::PK_DOWN, ntx::PK_HEAD};
    for (int i = 0; i < 5; ++i) rows_per_slot[i] = st.g[kinds[i]].TR;
  }
  return NTX_OK;
}

extern "C" int ntx_engine_launches_per_step(ntx_engine* e) {
  if (!e) return fail(NTX_ERR_INVALID_ARG, "engine is NULL");
  if (e->launches < 0) return fail(NTX_ERR_INVALID_ARG, "the last call was a self-speculative step");
  return e->launches;
}

extern "C" int ntx_engine_destroy(ntx_engine* e) {
  if (!e) return NTX_OK;
  cudaError_t err = wait_stream(e->cs, e->sync_ev);
  if (err == cudaSuccess && e->xs) err = wait_stream(e->xs, e->sync_ev);
  if (err == cudaErrorTimeout) return wait_fail(err, "ntx_engine_destroy");  // work in flight: the engine is kept
  engine_free(e);
  return err == cudaSuccess ? NTX_OK : cuda_fail(err, "ntx_engine_destroy");
}

extern "C" int ntx_set_host_wait_limit(uint64_t ms) {
  if (ms == 0) return fail(NTX_ERR_INVALID_ARG, "host wait limit must be > 0 ms");
  g_host_wait_ms.store(ms);
  return NTX_OK;
}

extern "C" int ntx_engine_set_fault(ntx_engine* e, int stall_cta, uint64_t wait_ns) {
  if (!e) return fail(NTX_ERR_INVALID_ARG, "engine is NULL");
  if (stall_cta < -1) return fail(NTX_ERR_INVALID_ARG, "stall_cta must be >= -1");
  e->pst.stall_cta = stall_cta;
  e->pst.wait_ns = wait_ns ? wait_ns : ntx::kDefaultWaitNs;
  return NTX_OK;
}
