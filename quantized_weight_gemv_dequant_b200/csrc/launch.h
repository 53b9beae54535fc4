// launch.h -- host-side launchers of the libntx kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ntx {

int sm_count();
void set_gemv_ctas_per_sm(int cps);
int gemv_ctas_per_sm();
void set_gemv_pdl(bool on);
bool gemv_pdl();

// Grid of a GEMV over M logical rows (rows grouped in pairs when align == 2).
int gemv_grid(int64_t M, int align);
// Split count of the attention kernel for contexts up to n_ctx.
int attn_splits(int n_kv_heads, int n_ctx);

bool gemv_tma_ok(int qtype, const void* W, int64_t K);

cudaError_t launch_dequant(int qtype, const void* blocks, float* out, int64_t nblocks, cudaStream_t s);
cudaError_t launch_gemv(int qtype, const void* W, int64_t M, int64_t K, const float* x, float* y, const float* resid,
                        cudaStream_t s, bool pdl);
cudaError_t launch_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, cudaStream_t s);
cudaError_t launch_rope(float* q, float* k, int nq, int nkv, int head_dim, int pos, float theta, cudaStream_t s);
cudaError_t launch_swiglu(const float* g, const float* u, float* out, int64_t n, cudaStream_t s);
cudaError_t launch_read_probe(const void* buf, uint64_t bytes, unsigned* sum, cudaStream_t s);
cudaError_t launch_attn(const float* q, const uint16_t* kc, const uint16_t* vc, float* out, float* part, int Hq,
                        int Hkv, int n_ctx, const int* pos_dev, int max_ctx, int n_split, cudaStream_t s, bool pdl);

// The pieces of one fused decode layer.
struct LayerArgs {
  int qt_qkv, qt_o, qt_gu, qt_down;  // block types of wq/wk/wv, wo, wg/wu, wd
  int64_t H, Hq, Hkv, D, F;
  int max_ctx;
  float eps, theta;
  const uint8_t *wq, *wk, *wv, *wo, *wg, *wu, *wd;
  const float *attn_norm, *ffn_norm;
  uint16_t *k_cache, *v_cache;
  float* hidden;          // residual stream, in/out
  const float* stats_in;  // sum(hidden^2) partials (slot 0 of 4), n_stats_in CTAs
  int n_stats_in;
  float* stats_o;     // O projection statistics  [grid][4]
  float* stats_down;  // down projection statistics [grid][4]
  float *q, *attn_out, *attn_part, *h1, *u;
  int pos;             // used when pos_dev is null
  const int* pos_dev;  // device position word (engine)
  int n_split;       // split + combine attention (when attn_cluster == 0)
  int attn_cluster;  // CTAs per KV-head cluster of the fused attention, 0 = split + combine
  cudaEvent_t probe_begin, probe_end;  // recorded around the gate/up GEMV when set
};
// Kernels one launch_layer() enqueues.
inline int layer_launches(const LayerArgs& a) { return a.attn_cluster > 0 ? 5 : 6; }
// Cluster size for the fused attention over contexts up to n_ctx_max (0: use split + combine).
int attn_cluster_size(int Hq, int Hkv, int n_ctx_max);
cudaError_t launch_attn_cluster(const float* q, const uint16_t* kc, const uint16_t* vc, float* out, int Hq, int Hkv,
                                int n_ctx, const int* pos_dev, int max_ctx, int cs, cudaStream_t s, bool pdl);
cudaError_t launch_layer(const LayerArgs& a, cudaStream_t s, bool pdl);
// Number of statistics partials the down projection of a layer writes.
int layer_stats_parts(int64_t H);

cudaError_t launch_sumsq(const float* h, int64_t n, float* parts, int nparts, cudaStream_t s, bool pdl);
// token = *tok_param if >= 0, else *tok_state (the previous step's argmax).
cudaError_t launch_embed(const uint16_t* table, int64_t H, int64_t V, const int* tok_param, const int* tok_state,
                         float* h, float* parts, int nparts, cudaStream_t s, bool pdl);
// Head: logits = W (RMSNorm(h) w_final), per-CTA argmax partials.
cudaError_t launch_head(int qtype, const void* W, int64_t V, int64_t H, const float* h, const float* final_norm,
                        const float* stats_in, int n_stats_in, float eps, float* logits, float* arg_parts,
                        cudaStream_t s, bool pdl);
int head_parts(int64_t V);
cudaError_t launch_argmax_finalize(const float* parts, int nparts, int* token_state, int* next_token, cudaStream_t s,
                                   bool pdl);
// cos_out[layers[k]] (layers may be null: identity) from per-layer statistics
// at stats + layers[k] * layer_stride.
cudaError_t launch_cos_finalize(const float* stats, int nparts, const int* layers, int nlayers, int64_t layer_stride,
                                float* cos_out, cudaStream_t s, bool pdl);

int read_device_status(int* code);
int read_check_report(int* site, long long* index);
int* device_status_ptr();

// Record a failure for ntx_last_error() on the calling thread; returns code.
int record_error(int code, const char* msg);
int record_cuda_error(cudaError_t e, const char* what);

}  // namespace ntx
