/*
 * inputgen.cu -- host and device fill routines over sa_inputgen.h.
 *
 * Test and benchmark infrastructure: produces the seeded synthetic Q/K/V
 * blocks of the rolling KV-cache workloads. Host and device produce the same
 * bits for the same coordinates. Layout of one block: [tok][head][d].
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>
#include "sa_inputgen.h"

#define IG_MAX_STREAMS 64

extern "C" {

/* Fill tokens [tok0, tok0+n_tok) of one block. dtype IG_F32 -> float*,
 * IG_BF16 -> uint16_t* (bf16 bits). Returns 0, or -1 on a bad argument. */
int ig_fill_host(const ig_spec* sp, int64_t stream, int64_t chunk, int32_t tensor,
                 int64_t tok0, int64_t n_tok, int32_t H, int32_t D, int32_t dtype,
                 void* out) {
  if (!sp || !out || tensor < 0 || tensor > 2 || H <= 0 || D <= 0 || n_tok < 0 || tok0 < 0)
    return -1;
  const uint64_t key = ig_key(sp->seed, stream, chunk, tensor);
  const uint64_t okey = ig_key(sp->seed, stream, chunk, IG_OUTLIER);
  const uint64_t thr = tensor == IG_K ? ig_outlier_threshold(sp->outlier_frac) : 0;
  const int64_t n = n_tok * (int64_t)H * D;
  const uint64_t base = (uint64_t)tok0 * (uint64_t)H * (uint64_t)D;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    float x = ig_value_keyed(sp->dist[tensor], key, okey, thr, tensor == IG_K,
                             base + (uint64_t)i, D, sp->outlier_scale);
    if (dtype == IG_BF16) ((uint16_t*)out)[i] = ig_f32_to_bf16_rne(x);
    else ((float*)out)[i] = x;
  }
  return 0;
}

/* Gate inputs of tokens [tok0, tok0+n_tok) of one chunk of one stream:
 * g and beta, [n_tok][H] fp32 each (either may be NULL). Returns 0, or -1 on a
 * bad argument. */
int ig_fill_gates_host(const ig_spec* sp, int64_t stream, int64_t chunk, int64_t tok0,
                       int64_t n_tok, int32_t H, float g_scale, float* g, float* beta) {
  if (!sp || H <= 0 || n_tok < 0 || tok0 < 0) return -1;
  const uint64_t gkey = ig_key(sp->seed, stream, chunk, IG_GATE);
  const uint64_t bkey = ig_key(sp->seed, stream, chunk, IG_BETA);
  const int64_t n = n_tok * (int64_t)H;
  const uint64_t base = (uint64_t)tok0 * (uint64_t)H;
  for (int64_t i = 0; i < n; ++i) {
    if (g) g[i] = ig_gate_log_decay(gkey, base + (uint64_t)i, g_scale);
    if (beta) beta[i] = ig_gate_beta(bkey, base + (uint64_t)i);
  }
  return 0;
}

struct IgDevArgs {
  uint64_t key[IG_MAX_STREAMS];
  uint64_t okey[IG_MAX_STREAMS];
  int32_t skip[IG_MAX_STREAMS];
  uint64_t thr;
  int32_t dist;
  int32_t is_k;
  float outlier_scale;
  int32_t D;
  int64_t per_stream; /* Lc*H*D */
  int32_t n_streams;
  int32_t dtype;
};

__global__ void ig_fill_kernel(const __grid_constant__ IgDevArgs a, void* out) {
  const int64_t total = a.per_stream * a.n_streams;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = (int)(i / a.per_stream);
    if (a.skip[s]) continue;
    const uint64_t idx = (uint64_t)(i - (int64_t)s * a.per_stream);
    float x = ig_value_keyed(a.dist, a.key[s], a.okey[s], a.thr, a.is_k, idx, a.D,
                             a.outlier_scale);
    if (a.dtype == IG_BF16) ((uint16_t*)out)[i] = ig_f32_to_bf16_rne(x);
    else ((float*)out)[i] = x;
  }
}

/* Fill a device buffer [n_streams][Lc][H][D] with block (stream_ids[i], chunks[i])
 * in slot i; chunks[i] < 0 leaves slot i untouched. Asynchronous on `stream`.
 * Returns 0, -1 on a bad argument, or the CUDA error code. */
int ig_fill_device(const ig_spec* sp, int32_t n_streams, const int64_t* stream_ids,
                   const int64_t* chunks, int32_t tensor, int64_t Lc, int32_t H, int32_t D,
                   int32_t dtype, void* out, void* cuda_stream) {
  if (!sp || !out || !stream_ids || !chunks || n_streams <= 0 ||
      n_streams > IG_MAX_STREAMS || tensor < 0 || tensor > 2 || Lc <= 0 || H <= 0 || D <= 0)
    return -1;
  IgDevArgs a;
  memset(&a, 0, sizeof(a));
  for (int i = 0; i < n_streams; ++i) {
    a.skip[i] = chunks[i] < 0;
    a.key[i] = ig_key(sp->seed, stream_ids[i], chunks[i], tensor);
    a.okey[i] = ig_key(sp->seed, stream_ids[i], chunks[i], IG_OUTLIER);
  }
  a.thr = tensor == IG_K ? ig_outlier_threshold(sp->outlier_frac) : 0;
  a.dist = sp->dist[tensor];
  a.is_k = tensor == IG_K;
  a.outlier_scale = sp->outlier_scale;
  a.D = D;
  a.per_stream = Lc * (int64_t)H * D;
  a.n_streams = n_streams;
  a.dtype = dtype;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  ig_fill_kernel<<<nsm * 8, 256, 0, (cudaStream_t)cuda_stream>>>(a, out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? 0 : (int)e;
}

}  /* extern "C" */
