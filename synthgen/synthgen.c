/*
 * synthgen.c -- host build of the seeded synthetic-input generator.
 *
 * Test and benchmark infrastructure: produces the random inputs (fp32 / fp16
 * tensors, token ids, quantized weight matrices) that both the CPU oracle and
 * the CUDA path consume.  Compiled with -O2 -ffp-contract=off so that every
 * floating-point operation in sg_core.h rounds exactly as its CUDA twin does.
 * Work is split over rows/elements with pthreads; every output element is a
 * pure function of (seed, tensor id, index), so the bytes do not depend on the
 * thread count.
 */
#include "sg_core.h"

#include <pthread.h>
#include <stdlib.h>

uint32_t sg_tensor_id(const char* name) { return sg_fnv1a(name); }

void sg_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  sg_philox4x32_10(ctr, key, out);
}

double sg_normal_at(uint32_t seed, uint32_t tid, uint64_t idx) { return sg_normal(seed, tid, idx); }
double sg_ln(double s) { return sg_ln_unit(s); }
uint16_t sg_half_from_float(float f) { return sg_f32_to_f16(f); }
float sg_half_to_float(uint16_t h) { return sg_f16_to_f32(h); }
int sg_qblock_elems(int qtype) { return sg_block_elems(qtype); }
int sg_qblock_bytes(int qtype) { return sg_block_bytes(qtype); }

/* ---------------------------------------------------------------- threads */
typedef struct {
  int kind; /* 0 f32, 1 f16, 2 quant rows, 3 tokens */
  uint32_t seed, tid;
  int64_t begin, end; /* elements (kinds 0,1,3) or rows (kind 2) */
  double mean, sigma;
  int qtype;
  int64_t K;
  int64_t row_base; /* kind 2: first row held by `out` */
  uint32_t V;
  void* out;
} sg_job;

static void* sg_run(void* p) {
  sg_job* j = (sg_job*)p;
  if (j->kind == 0) {
    float* o = (float*)j->out;
    for (int64_t i = j->begin; i < j->end; ++i) o[i] = sg_normal_f32(j->seed, j->tid, (uint64_t)i, j->mean, j->sigma);
  } else if (j->kind == 1) {
    uint16_t* o = (uint16_t*)j->out;
    for (int64_t i = j->begin; i < j->end; ++i)
      o[i] = sg_f32_to_f16(sg_normal_f32(j->seed, j->tid, (uint64_t)i, j->mean, j->sigma));
  } else if (j->kind == 2) {
    const int be = sg_block_elems(j->qtype), bb = sg_block_bytes(j->qtype);
    const int64_t nb = j->K / be;
    uint8_t* o = (uint8_t*)j->out;
    float w[256];
    for (int64_t r = j->begin; r < j->end; ++r)
      for (int64_t b = 0; b < nb; ++b) {
        const uint64_t base = (uint64_t)r * (uint64_t)j->K + (uint64_t)(b * be);
        for (int i = 0; i < be; ++i) w[i] = sg_normal_f32(j->seed, j->tid, base + (uint64_t)i, j->mean, j->sigma);
        sg_quant_block(j->qtype, w, o + ((r - j->row_base) * nb + b) * bb);
      }
  } else {
    int32_t* o = (int32_t*)j->out;
    for (int64_t i = j->begin; i < j->end; ++i) o[i] = sg_token(j->seed, j->tid, (uint64_t)i, j->V);
  }
  return NULL;
}

static void sg_parallel(sg_job proto, int64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < nthreads) nthreads = n > 0 ? (int)n : 1;
  if (nthreads == 1) {
    proto.begin = 0; proto.end = n;
    sg_run(&proto);
    return;
  }
  pthread_t th[256];
  sg_job jobs[256];
  int started[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = proto;
    jobs[t].begin = n * t / nthreads;
    jobs[t].end = n * (t + 1) / nthreads;
    started[t] = pthread_create(&th[t], NULL, sg_run, &jobs[t]) == 0;
    if (!started[t]) sg_run(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (started[t]) pthread_join(th[t], NULL);
}

/* out[i] = fp32(mean + sigma * z_i), i in [0, n). */
void sg_fill_f32(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, float* out, int nthreads) {
  sg_job j = {0};
  j.kind = 0; j.seed = seed; j.tid = tid; j.mean = mean; j.sigma = sigma; j.out = out;
  sg_parallel(j, n, nthreads);
}

/* out[i] = fp16(fp32(mean + sigma * z_i)). */
void sg_fill_f16(uint32_t seed, uint32_t tid, int64_t n, double mean, double sigma, uint16_t* out, int nthreads) {
  sg_job j = {0};
  j.kind = 1; j.seed = seed; j.tid = tid; j.mean = mean; j.sigma = sigma; j.out = out;
  sg_parallel(j, n, nthreads);
}

/* Rows [row0, row0 + nrows) of an M x K matrix whose fp32 weights are
 * mean + sigma * z_(r*K + c), quantized block by block into `out`
 * (nrows * K/block_elems * block_bytes bytes).  Returns 0, or -1 if K is not
 * a multiple of the block size or the type is unknown. */
int sg_quant_rows(int qtype, uint32_t seed, uint32_t tid, int64_t row0, int64_t nrows, int64_t K, double mean,
                  double sigma, uint8_t* out, int nthreads) {
  const int be = sg_block_elems(qtype);
  if (be == 0 || K <= 0 || K % be) return -1;
  sg_job j = {0};
  j.kind = 2; j.seed = seed; j.tid = tid; j.mean = mean; j.sigma = sigma; j.qtype = qtype; j.K = K;
  j.row_base = row0; /* row r is written at (r - row0) */
  j.out = out;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
  pthread_t th[256];
  sg_job jobs[256];
  int started[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = j;
    jobs[t].begin = row0 + nrows * t / nthreads;
    jobs[t].end = row0 + nrows * (t + 1) / nthreads;
    started[t] = (nthreads > 1) && pthread_create(&th[t], NULL, sg_run, &jobs[t]) == 0;
    if (!started[t]) sg_run(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (started[t]) pthread_join(th[t], NULL);
  return 0;
}

/* Quantize caller-given fp32 values (n a multiple of the block size). */
int sg_quantize(int qtype, const float* w, int64_t n, uint8_t* out) {
  const int be = sg_block_elems(qtype), bb = sg_block_bytes(qtype);
  if (be == 0 || n % be) return -1;
  for (int64_t b = 0; b < n / be; ++b) sg_quant_block(qtype, w + b * be, out + b * bb);
  return 0;
}

void sg_fill_tokens(uint32_t seed, uint32_t tid, int64_t n, uint32_t V, int32_t* out) {
  sg_job j = {0};
  j.kind = 3; j.seed = seed; j.tid = tid; j.V = V; j.out = out;
  sg_parallel(j, n, 1);
}
