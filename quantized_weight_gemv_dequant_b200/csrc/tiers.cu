// tiers.cu -- automatic tier sizing: which layers stay resident in device
// memory (tier A) and which are streamed from pinned host memory (tier B),
// from the free device memory (cudaMemGetInfo) and the host's available
// memory (/proc/meminfo), as "NTransformer" -- 3-Tier describes (tier sizes
// computed from cudaMemGetInfo() and /proc/meminfo) and "Show HN: NVMe経由で
// CPUをバイパスして単一のRTX 3090上で動作するLlama 3.1 70B" -- 3層アダプティブ
// キャッシュ詳細 (VRAM resident > pinned RAM > NVMe/mmap).  The third tier
// (NVMe / mmap) is not provided: a model that does not fit the first two is
// refused.
//
// Rule: layers are placed in execution order; the first n are resident,
// where n is the largest count whose blobs, plus the two device slots the
// streamed layers need (when n < L), plus everything else the engine keeps on
// the device (embedding table, final norm, output head, KV caches, engine
// workspace), fit in (free device memory - reserve).  The remaining L - n
// layers go to pinned host memory, which must hold them within the host's
// available memory less its reserve.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>

#include "launch.h"
#include "ntx.h"

namespace {

uint64_t mat_bytes(int qt, int64_t M, int64_t K) {
  int be = 0, bb = 0;
  switch (qt) {
    case NTX_F32: be = 1; bb = 4; break;
    case NTX_F16: be = 1; bb = 2; break;
    case NTX_Q4_0: be = 32; bb = 18; break;
    case NTX_Q8_0: be = 32; bb = 34; break;
    case NTX_Q4_K: be = 256; bb = 144; break;
    case NTX_Q5_K: be = 256; bb = 176; break;
    case NTX_Q6_K: be = 256; bb = 210; break;
    default: return 0;
  }
  if (K % be) return 0;
  return (uint64_t)M * (uint64_t)(K / be) * (uint64_t)bb;
}

}  // namespace

extern "C" uint64_t ntx_engine_device_bytes(const ntx_model_config* cfg, int head_qtype) {
  if (!cfg || cfg->hidden <= 0 || cfg->vocab <= 0 || cfg->n_layers < 0 || cfg->n_kv_heads <= 0 ||
      cfg->head_dim <= 0 || cfg->max_ctx <= 0)
    return 0;
  const uint64_t head = mat_bytes(head_qtype, cfg->vocab, cfg->hidden);
  if (!head) return 0;
  const uint64_t H = (uint64_t)cfg->hidden, V = (uint64_t)cfg->vocab;
  const uint64_t kv = 2ull * (uint64_t)cfg->n_layers * (uint64_t)cfg->n_kv_heads * (uint64_t)cfg->max_ctx *
                      (uint64_t)cfg->head_dim * 2ull;
  return V * H * 2ull + 4ull * H + head + kv + (uint64_t)ntx_engine_workspace_bytes(cfg);
}

extern "C" int ntx_auto_tier_map(const ntx_model_config* cfg, uint64_t layer_bytes, int head_qtype,
                                 uint64_t device_free, uint64_t device_reserve, uint64_t host_available,
                                 uint64_t host_reserve, int8_t* tier_map, int* n_resident) {
  if (!cfg || !tier_map || cfg->n_layers < 0 || layer_bytes == 0)
    return ntx::record_error(NTX_ERR_INVALID_ARG, "ntx_auto_tier_map: NULL config or tier map, or zero layer size");
  const uint64_t fixed = ntx_engine_device_bytes(cfg, head_qtype);
  if (!fixed) return ntx::record_error(NTX_ERR_INVALID_ARG, "ntx_auto_tier_map: bad config or head type");
  const int L = cfg->n_layers;
  const uint64_t dev_budget = device_free > device_reserve ? device_free - device_reserve : 0;
  if (fixed > dev_budget) {
    char msg[200];
    snprintf(msg, sizeof msg,
             "ntx_auto_tier_map: the non-layer device buffers need %llu bytes, %llu are available",
             (unsigned long long)fixed, (unsigned long long)dev_budget);
    return ntx::record_error(NTX_ERR_NOMEM, msg);
  }
  const uint64_t room = dev_budget - fixed;
  int n = 0;
  if ((uint64_t)L * layer_bytes <= room) {
    n = L;
  } else if (room >= 2 * layer_bytes) {
    n = (int)((room - 2 * layer_bytes) / layer_bytes);  // two slots for the streamed layers
    if (n > L) n = L;
  } else {
    return ntx::record_error(NTX_ERR_NOMEM, "ntx_auto_tier_map: no room for the two device slots of tier B");
  }
  const uint64_t host_budget = host_available > host_reserve ? host_available - host_reserve : 0;
  if ((uint64_t)(L - n) * layer_bytes > host_budget) {
    char msg[240];
    snprintf(msg, sizeof msg,
             "ntx_auto_tier_map: %d layers (%llu bytes) do not fit %llu bytes of host memory; a third tier "
             "(NVMe / mmap) would be needed and is not provided",
             L - n, (unsigned long long)((uint64_t)(L - n) * layer_bytes), (unsigned long long)host_budget);
    return ntx::record_error(NTX_ERR_NOMEM, msg);
  }
  for (int l = 0; l < L; ++l) tier_map[l] = l < n ? 0 : 1;
  if (n_resident) *n_resident = n;
  return NTX_OK;
}

extern "C" int ntx_memory_budget(uint64_t* device_free, uint64_t* device_total, uint64_t* host_available,
                                 const char* meminfo_path) {
  if (device_free || device_total) {
    size_t f = 0, t = 0;
    const cudaError_t e = cudaMemGetInfo(&f, &t);
    if (e != cudaSuccess) return ntx::record_cuda_error(e, "ntx_memory_budget: cudaMemGetInfo");
    if (device_free) *device_free = f;
    if (device_total) *device_total = t;
  }
  if (host_available) {
    FILE* fp = fopen(meminfo_path ? meminfo_path : "/proc/meminfo", "r");
    if (!fp) return ntx::record_error(NTX_ERR_INVALID_ARG, "ntx_memory_budget: cannot open the meminfo file");
    char line[256];
    bool found = false;
    unsigned long long kb = 0;
    while (fgets(line, sizeof line, fp)) {
      if (sscanf(line, "MemAvailable: %llu kB", &kb) == 1) {
        found = true;
        break;
      }
    }
    fclose(fp);
    if (!found) return ntx::record_error(NTX_ERR_INVALID_ARG, "ntx_memory_budget: no MemAvailable line");
    *host_available = (uint64_t)kb * 1024ull;
  }
  return NTX_OK;
}
