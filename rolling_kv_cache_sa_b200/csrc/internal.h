// internal.h -- launch parameter blocks and kernel entry points of libsa.so.
// Every parameter block is passed by value (__grid_constant__), so a launch
// needs no host->device copy and can be captured in a CUDA graph.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sa.h"

namespace sa {

constexpr int kMaxEntries = 32;   // (stream, frame) entries per append launch
constexpr int kMaxF8Heads = 128;   // heads of an e4m3 cache
constexpr int kMaxRefresh = 16;   // streams, and (stream, sink frame) entries, per refresh launch
constexpr int kMaxDt2 = 64;       // d_t / 2 <= 64
constexpr int kMaxAttnStreams = SA_MAX_STREAMS;
constexpr int kDeviceErrTimeout = 1;

// Debug build (compiled with -DSA_DEBUG_BOUNDS, libsa_debug.so): every
// computed index into a buffer (cache rows, partial-result slots, arrival
// counters, workspace offsets, TMA tile coordinates) is range-checked before
// the access. A violation sets bit `site` of the source file's bounds word
// and the access is skipped (a store) or replaced (a load reads zero, a tile
// coordinate is clamped to 0), so the kernel still ends normally; no trap,
// no fault. sa_debug_bounds_status reads and clears the words. In the normal
// build SA_BOUNDS(ok, site) is `true` and costs nothing.
#ifdef SA_DEBUG_BOUNDS
#define SA_BOUNDS(ok, site) sa_bounds_ok_((ok), (site))
// one word per source file (no relocatable device code: each .cu file keeps
// its own word and host reader, named by the file)
#define SA_DEFINE_BOUNDS_WORD(reader)                                                 \
  static __device__ unsigned int g_sa_bounds_word;                                    \
  static __device__ __forceinline__ bool sa_bounds_ok_(bool ok, int site) {           \
    if (!ok) atomicOr(&g_sa_bounds_word, 1u << site);                                 \
    return ok;                                                                        \
  }                                                                                   \
  cudaError_t reader(unsigned int* word, cudaStream_t st) {                           \
    unsigned int w = 0, z = 0;                                                        \
    cudaError_t e = cudaMemcpyFromSymbolAsync(&w, g_sa_bounds_word, sizeof(w), 0,     \
                                              cudaMemcpyDeviceToHost, st);            \
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);                              \
    if (e == cudaSuccess && w)                                                        \
      e = cudaMemcpyToSymbolAsync(g_sa_bounds_word, &z, sizeof(z), 0,                 \
                                  cudaMemcpyHostToDevice, st);                        \
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);                              \
    *word = w;                                                                        \
    return e;                                                                         \
  }
#else
#define SA_BOUNDS(ok, site) true
#define SA_DEFINE_BOUNDS_WORD(reader)
#endif
// Host readers of the per-file bounds words (debug build only).
cudaError_t bounds_word_attend_tc(unsigned int* word, cudaStream_t st);
cudaError_t bounds_word_attend_simt(unsigned int* word, cudaStream_t st);
cudaError_t bounds_word_rope_append(unsigned int* word, cudaStream_t st);
cudaError_t bounds_word_gdn(unsigned int* word, cudaStream_t st);
// Debug build: one thread records a check failure at site 31 of the
// attention file's word without touching memory (shows the recording path).
cudaError_t bounds_selftest(cudaStream_t st);

// Fused 3D-RoPE + append (one launch covers up to kMaxEntries (stream, frame)
// entries; entry e = a*C + i is frame i of the a-th stream of the launch).
struct AppendParams {
  const void* q;
  const void* k;
  const void* v;
  void* q_ws;        // [B][H][Lc][D]
  void* k_cache;     // [B][H][ntok][D]
  void* v_cache;     // [B][H][ntok][D]
  void* k_raw;       // [B][H][S*F][D]
  const float2* htab;  // [fh][d_h/2] (cos, sin)
  const float2* wtab;  // [fw][d_w/2]
  int32_t H, D, fw, F, C, Lc;
  int64_t ntok, sf;    // cache rows per (b, h); sink rows per (b, h)
  int32_t dt2, dh2, dw2;
  int32_t n_streams;   // streams in this launch
  int32_t batch;       // B (the extent of q, k, v and the caches; bounds checks)
  const float* fp8_scale;  // e4m3 cache: [3][H] per-head scales of q, k, v (device)
  int32_t stream_of[kMaxEntries];
  int64_t dest_row[kMaxEntries];   // cache row of the frame's first token
  int64_t raw_row[kMaxEntries];    // raw-sink row of the frame, or -1
  float2 tcs[kMaxEntries][kMaxDt2];  // temporal band (cos, sin) per entry
};

// RoPE refresh: ring keys' temporal band rotated by -Delta in place; sink keys
// re-derived from raw keys at their new positions.
struct RefreshParams {
  void* k_cache;
  void* k_raw;
  // sink update (update != 0): raw sink keys and sink values become
  // (1 - alpha) * old + alpha * new before the sink keys are re-derived;
  // k_new / v_new are [B][S*F][H][D]; ring_rows must be 0
  void* v_cache;
  const void* k_new;
  const void* v_new;
  float alpha;
  int32_t update;
  const float* fp8_scale;  // e4m3 cache: [3][H] per-head scales of q, k, v (device)
  const float2* htab;
  const float2* wtab;
  int32_t H, D, fw, F, S;
  int64_t ntok, sf;
  int32_t dt2, dh2, dw2;
  int32_t n_streams;
  int32_t batch;       // B (bounds checks)
  int32_t stream_of[kMaxRefresh];
  int64_t ring_rows[kMaxRefresh];    // valid ring rows of the stream
  int64_t sink_rows[kMaxRefresh];    // valid sink rows of the stream
  float2 dcs[kMaxRefresh][kMaxDt2];  // (cos, sin) of -Delta * theta_j, per stream
  float2 scs[kMaxRefresh][kMaxDt2];  // (cos, sin) of t * theta_j per sink entry a*S + s
};

// Attention over the contiguous key prefix [0, n_keys) of each (b, h).
struct AttnParams {
  int32_t H, Lc;
  int64_t ntok;
  int32_t n_q_tiles;   // ceil(Lc / 128)
  int32_t n_streams;
  float scale_log2;    // softmax_scale * log2(e)
  int32_t pad_;
  void* out;           // [B][Lc][H][D]
  const void* q_ws;    // [B][H][Lc][D] (SIMT path)
  const void* k_cache; // (SIMT path)
  const void* v_cache; // (SIMT path)
  int* status;
  int32_t fp8;         // e4m3 operands (SA_BF16_E4M3)
  int32_t batch;       // B (bounds checks)
  int32_t stream_of[kMaxAttnStreams];
  int32_t n_keys[kMaxAttnStreams];
  float inv_qk[kMaxF8Heads];  // e4m3: 1 / (q_scale * k_scale) per head
  float inv_v[kMaxF8Heads];   // e4m3: 1 / v_scale per head
};

// Workspace the bf16 attention may use for split work units: per slot (two
// per CTA) the unnormalised fp32 O of two 128-row tiles and their (m, l),
// then one arrival counter per (unit, tile, row) for max_units units (a unit
// is a stream, a head and a pair of 128-row query tiles). The counters must
// be zero before the first launch; every launch that completes leaves them
// zero again.
size_t attend_partials_bytes(int D, int num_sms, int64_t max_units);

// Gated DeltaNet block (gdn.cu): T tokens of each listed stream; q, k, v, out
// [B][T][H][D], g and beta [B][T][H], state [B][H][D][D] fp32 in place.
// workspace: a 1 KiB header (the call's device status word), then per
// (listed stream, head, 64-token sub-chunk) the prep kernel's output: the
// bf16 hi/lo operand images of the sequential tensor-core kernel (128 key
// dims wide for D = 64 too); gdn_workspace_bytes(n_streams, H, D, T) bytes,
// 16-byte aligned.
struct GdnParams {
  float* state;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  void* out;
  float* workspace;
  int64_t T;
  int32_t H;
  float scale;
  int32_t n_streams;
  int32_t n_sub;       // ceil(T / 64)
  int32_t batch;       // B (bounds checks)
  int32_t j_begin;     // sub-chunks [j_begin, j_end) of this launch (tensor-core path)
  int32_t j_end;
  int32_t pdl_wait;    // prep launched ahead of the previous pass piece: see launch_gdn_t
  int32_t stream_of[SA_MAX_STREAMS];
};
size_t gdn_workspace_bytes(int B, int H, int D, int64_t T);
cudaError_t launch_gdn(const GdnParams& p, int D, int dtype, cudaStream_t st);

cudaError_t launch_append(const AppendParams& p, int dtype, int num_sms, cudaStream_t st);
// Bounded-wait check (wait_probe.cu); synchronises `st` and returns the
// device status word and the two warps' waiting times.
cudaError_t run_wait_probe(uint64_t limit_ns, cudaStream_t st, int* status,
                           unsigned long long waited_ns[2]);
cudaError_t launch_refresh(const RefreshParams& p, int dtype, int num_sms, cudaStream_t st);
cudaError_t launch_attend_simt_f32(const AttnParams& p, int D, cudaStream_t st);
// bf16 tensor-core attention. `partials` (attend_partials_bytes) lets the
// persistent kernel split work units at equal-work boundaries (the last
// piece of each row to finish merges the pieces); with partials == nullptr
// every CTA takes whole units. *n_kernels (if non-null) receives the kernels
// launched.
cudaError_t launch_attend_tc_bf16(const AttnParams& p, int D, const CUtensorMap* tm_q,
                                  const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                  void* partials, size_t partials_bytes, int num_sms,
                                  cudaStream_t st, int* n_kernels);

}  // namespace sa
