// sa_api.cu -- host side of libsa.so: the C ABI declared in include/sa.h.
//
// Host planner (per active stream, per call): local chunk index, cache row of
// each appended frame (sink slot f, or ring slot S + (f - S) mod R), temporal
// RoPE position t = f - pos_base with its (cos, sin) values computed in fp64,
// and the visible key count. Because sink frames fill the first S*F rows and
// later frames fill the ring from its first slot, the keys a chunk sees are
// always the contiguous row prefix [0, n_keys) of its (stream, head) cache:
// while the sink is not full no frame has reached the ring; once it is full,
// the sink rows are followed by the occupied ring rows. The attention kernel
// therefore needs one number per stream. Everything is passed by value in
// launch parameters: no host->device copy, no synchronisation on the hot path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

namespace {

thread_local std::string g_last_error = "no error";

sa_status fail(sa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

sa_status cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaErrorMemoryAllocation)
    return fail(SA_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
  return fail(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Host fault injection for tests of the error paths (no GPU fault involved),
// read from SA_FAULT when a handle is created: "alloc" makes the cache
// allocation report out-of-memory; "launch" makes every hot call report a
// launch failure before anything is launched; "launch_once" does so once.
enum { FAULT_NONE = 0, FAULT_ALLOC = 1, FAULT_LAUNCH = 2, FAULT_LAUNCH_ONCE = 3 };
int fault_from_env() {
  const char* f = getenv("SA_FAULT");
  if (!f) return FAULT_NONE;
  if (!strcmp(f, "alloc")) return FAULT_ALLOC;
  if (!strcmp(f, "launch")) return FAULT_LAUNCH;
  if (!strcmp(f, "launch_once")) return FAULT_LAUNCH_ONCE;
  return FAULT_NONE;
}

// ---------------------------------------------------------------- config
sa_status validate_config(const sa_config* c) {
  if (!c) return fail(SA_ERR_INVALID_ARG, "config is NULL");
  if (c->batch < 1 || c->batch > SA_MAX_STREAMS)
    return fail(SA_ERR_INVALID_ARG, "batch must be in [1, %d], got %d", SA_MAX_STREAMS, c->batch);
  if (c->heads < 1) return fail(SA_ERR_INVALID_ARG, "heads must be >= 1");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(SA_ERR_INVALID_ARG, "head_dim must be 64 or 128, got %d", c->head_dim);
  if (c->frame_h < 1 || c->frame_w < 1) return fail(SA_ERR_INVALID_ARG, "frame_h, frame_w >= 1");
  if (c->chunk_frames < 1 || c->chunk_frames > SA_MAX_CHUNK_FRAMES)
    return fail(SA_ERR_INVALID_ARG, "chunk_frames must be in [1, %d]", SA_MAX_CHUNK_FRAMES);
  if (c->sink_frames < 0 || c->sink_frames > SA_MAX_SINK_FRAMES)
    return fail(SA_ERR_INVALID_ARG, "sink_frames must be in [0, %d]", SA_MAX_SINK_FRAMES);
  if (c->window_frames < 0) return fail(SA_ERR_INVALID_ARG, "window_frames must be >= 0");
  int sum = 0;
  for (int i = 0; i < 3; ++i) {
    if (c->rope_dims[i] < 0 || (c->rope_dims[i] & 1))
      return fail(SA_ERR_INVALID_ARG, "rope_dims must be even and >= 0");
    sum += c->rope_dims[i];
  }
  if (sum != c->head_dim) return fail(SA_ERR_INVALID_ARG, "rope_dims must sum to head_dim");
  if (c->rope_dims[0] / 2 > sa::kMaxDt2) return fail(SA_ERR_INVALID_ARG, "d_t must be <= 128");
  if (!(c->rope_base > 0.f)) return fail(SA_ERR_INVALID_ARG, "rope_base must be > 0");
  if (c->softmax_scale < 0.f || !isfinite(c->softmax_scale))
    return fail(SA_ERR_INVALID_ARG, "softmax_scale must be >= 0 (0 = 1/sqrt(D))");
  if (c->dtype != SA_F32 && c->dtype != SA_BF16 && c->dtype != SA_BF16_E4M3)
    return fail(SA_ERR_INVALID_ARG, "dtype must be SA_F32, SA_BF16 or SA_BF16_E4M3");
  if (c->dtype == SA_BF16_E4M3 && (c->head_dim != 128 || c->heads > sa::kMaxF8Heads))
    return fail(SA_ERR_UNSUPPORTED, "SA_BF16_E4M3 needs head_dim 128 and at most %d heads",
                sa::kMaxF8Heads);
  const int64_t F = (int64_t)c->frame_h * c->frame_w;
  const int64_t Lc = F * c->chunk_frames;
  const int64_t ntok = F * ((int64_t)c->sink_frames + c->window_frames + c->chunk_frames);
  if (Lc * c->heads * (int64_t)c->head_dim * c->batch > ((int64_t)1 << 31) / 2)
    return fail(SA_ERR_UNSUPPORTED, "B*C*F*H*D too large for one call");
  if (ntok > ((int64_t)1 << 30)) return fail(SA_ERR_UNSUPPORTED, "cache rows per head too large");
  if ((int64_t)c->batch * c->heads > ((int64_t)1 << 30))
    return fail(SA_ERR_UNSUPPORTED, "batch*heads too large");
  return SA_OK;
}

double theta(const sa_config* c, int band, int j) {
  return pow((double)c->rope_base, -2.0 * (double)j / (double)c->rope_dims[band]);
}

sa_status plan_chunk(const sa_config* c, int64_t fw_, int64_t base, sa_chunk_plan* pl) {
  const int64_t C = c->chunk_frames, S = c->sink_frames, R = (int64_t)c->window_frames + C;
  const int64_t F = (int64_t)c->frame_h * c->frame_w;
  if (fw_ < 0 || fw_ % C != 0)
    return fail(SA_ERR_STATE, "frames_written (%lld) is not a multiple of the chunk size",
                (long long)fw_);
  memset(pl, 0, sizeof(*pl));
  pl->chunk = fw_ / C;
  pl->n_frames = (int32_t)C;
  for (int64_t i = 0; i < C; ++i) {
    const int64_t f = fw_ + i;
    pl->is_sink[i] = f < S;
    pl->dest_row[i] = (f < S ? f : S + (f - S) % R) * F;
    pl->t_pos[i] = f - base;
  }
  const int64_t after = fw_ + C;
  pl->sink_len = std::min(S, after) * F;
  pl->ring_len = std::min(std::max<int64_t>(0, after - S), R) * F;
  pl->n_keys = pl->sink_len + pl->ring_len;
  return SA_OK;
}

int64_t refresh_delta(const sa_config* c, int64_t fw_, int64_t base) {
  const int64_t C = c->chunk_frames;
  const int64_t next = fw_ / C;
  const int64_t first = std::max<int64_t>(c->sink_frames, next * C - c->window_frames);
  return first - base;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3D map over [planes][rows][D] with 128-byte x 128-row x 1 boxes (64 bf16 or
// 128 e4m3 elements per row), 128-byte swizzle. Rows past `rows` of a plane
// read as zeros.
bool make_map(CUtensorMap* m, void* base, int64_t D, int64_t rows, int64_t planes,
              bool e4m3 = false) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const int64_t es_b = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)(D * es_b), (cuuint64_t)(rows * D * es_b)};
  cuuint32_t box[3] = {(cuuint32_t)(128 / es_b), 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
             dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

enum { KIND_APPEND = 0, KIND_ATTEND = 1, KIND_REFRESH = 2 };

}  // namespace

struct sa_cache {
  sa_config cfg;
  int dev = 0;
  int num_sms = 148;
  cudaStream_t create_stream = nullptr;
  int64_t F = 0, Lc = 0, R = 0, ntok = 0, sf = 0;
  size_t esz = 2;   // q, k, v, out elements
  size_t cesz = 2;  // cache and rotated-query elements (1 for e4m3)
  float scale = 0.f;
  float* d_fp8_scale = nullptr;     // e4m3: [3][H] q, k, v scales (device)
  std::vector<float> fp8_scale;     // host copy
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  void* k_raw = nullptr;
  int32_t sink_mode = SA_SINK_SHIFT;  // how the sink's positions follow a refresh
  int fault = 0;                      // injected host fault (SA_FAULT), tests only
  void* q_ws = nullptr;
  float2* htab = nullptr;
  float2* wtab = nullptr;
  int* d_status = nullptr;
  void* partials = nullptr;  // split-unit workspace of the bf16 attention
  size_t partials_bytes = 0;
  std::vector<int64_t> frames_written, pos_base;
  CUtensorMap tm_q, tm_k, tm_v;
  // host-buffer staging (allocated by the first sa_append_attend_host)
  void* stage[4] = {nullptr, nullptr, nullptr, nullptr};
  // pipelined host path (sa_append_attend_host_async): staging slots of
  // q, k, v, out, two copy streams and per-slot events
  static constexpr int kSlots = 3;
  void* slot_buf[kSlots][4] = {};
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t in_done[kSlots] = {}, comp_done[kSlots] = {}, out_done[kSlots] = {};
  int64_t async_calls = 0;
  // profiling
  bool profiling = false;
  std::vector<cudaEvent_t> ev;
  std::vector<int> ev_kind;
  size_t ev_used = 0;
  int64_t kernels = 0;  // kernel launches since sa_profile_begin
};

namespace {

// NVTX range around a library call or launch (a no-op unless a profiler is
// attached): sa.append, sa.attend, sa.refresh, sa.sink_update.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Base that the sink's temporal positions are taken against: t = f - base.
// Shift: the stream's base (the sink moves with every rebase). Re-pin: a
// refresh sets base >= S and the sink then sits right before the oldest
// window frame (t = f - S); before the first refresh base = 0.
int64_t sink_base(const sa_cache* h, int64_t base) {
  if (h->sink_mode == SA_SINK_REPIN && base > h->cfg.sink_frames) return h->cfg.sink_frames;
  return base;
}

// A record into a capturing stream is made an external event node, so the event
// still carries a time after each replay; the external flag is refused outside
// capture, where a plain record does the same.
void prof_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

void prof_before(sa_cache* h, cudaStream_t st, int kind) {
  if (!h->profiling || h->ev_used + 2 > h->ev.size()) return;
  prof_record(h->ev[h->ev_used], st);
  h->ev_kind[h->ev_used / 2] = kind;
}

void prof_after(sa_cache* h, cudaStream_t st) {
  if (!h->profiling || h->ev_used + 2 > h->ev.size()) return;
  prof_record(h->ev[h->ev_used + 1], st);
  h->ev_used += 2;
}

void free_all(sa_cache* h) {
  if (h->copy_in) cudaStreamSynchronize(h->copy_in);
  if (h->copy_out) cudaStreamSynchronize(h->copy_out);
  void* ptrs[] = {h->k_cache, h->v_cache, h->k_raw, h->q_ws, h->htab, h->wtab, h->d_status,
                  h->partials, h->stage[0], h->stage[1], h->stage[2], h->stage[3],
                  h->d_fp8_scale};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  for (int s = 0; s < sa_cache::kSlots; ++s) {
    for (int t = 0; t < 4; ++t)
      if (h->slot_buf[s][t]) cudaFree(h->slot_buf[s][t]);
    for (cudaEvent_t e : {h->in_done[s], h->comp_done[s], h->out_done[s]})
      if (e) cudaEventDestroy(e);
  }
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
}

sa_status active_list(const sa_cache* h, const uint8_t* active, std::vector<int>& out) {
  out.clear();
  for (int b = 0; b < h->cfg.batch; ++b)
    if (!active || active[b]) out.push_back(b);
  return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int32_t sa_abi_version(void) { return SA_ABI_VERSION; }

sa_status sa_wait_probe(uint64_t limit_ns, int64_t* waited_ns, sa_stream_t stream) {
  if (limit_ns < 100000ull || limit_ns > 10000000000ull)
    return fail(SA_ERR_INVALID_ARG, "limit_ns %llu outside [1e5, 1e10]",
                (unsigned long long)limit_ns);
  int dev = 0;
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return fail(SA_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  if (prop.major != 10)
    return fail(SA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100a (B200)",
                dev, prop.major, prop.minor);
  int status = 0;
  unsigned long long w[2] = {0, 0};
  e = sa::run_wait_probe(limit_ns, static_cast<cudaStream_t>(stream), &status, w);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe");
  if (waited_ns) {
    waited_ns[0] = (int64_t)w[0];
    waited_ns[1] = (int64_t)w[1];
  }
  if (status & sa::kDeviceErrTimeout)
    return fail(SA_ERR_DEVICE_TIMEOUT, "device wait expired after %llu ns (as designed)",
                (unsigned long long)w[0]);
  return SA_OK;
}

namespace {
sa_status validate_gdn_config(const sa_gdn_config* cfg) {
  if (!cfg) return fail(SA_ERR_INVALID_ARG, "config is NULL");
  if (cfg->batch < 1 || cfg->batch > SA_MAX_STREAMS)
    return fail(SA_ERR_INVALID_ARG, "batch must be in [1, %d], got %d", SA_MAX_STREAMS, cfg->batch);
  if (cfg->heads < 1 || cfg->heads > 65535)
    return fail(SA_ERR_INVALID_ARG, "heads must be in [1, 65535], got %d", cfg->heads);
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return fail(SA_ERR_INVALID_ARG, "head_dim must be 64 or 128, got %d", cfg->head_dim);
  if (cfg->dtype != SA_F32 && cfg->dtype != SA_BF16)
    return fail(SA_ERR_INVALID_ARG, "dtype must be SA_F32 or SA_BF16");
  if (cfg->tokens < 0) return fail(SA_ERR_INVALID_ARG, "tokens must be >= 0");
  if (!(cfg->scale >= 0.f) || !std::isfinite(cfg->scale))
    return fail(SA_ERR_INVALID_ARG, "scale must be finite and >= 0 (0 = 1/sqrt(D))");
  const size_t esz = cfg->dtype == SA_F32 ? 4 : 2;
  if ((double)cfg->batch * (double)cfg->tokens * cfg->heads * cfg->head_dim * esz > 9.0e18)
    return fail(SA_ERR_UNSUPPORTED, "batch*tokens*heads*head_dim too large");
  if ((cfg->tokens + 63) / 64 > 65535)
    return fail(SA_ERR_UNSUPPORTED, "tokens must be at most 65535 * 64 per call");
  return SA_OK;
}
}  // namespace

sa_status sa_gdn_workspace_size(const sa_gdn_config* cfg, size_t* bytes) {
  sa_status st = validate_gdn_config(cfg);
  if (st != SA_OK) return st;
  if (!bytes) return fail(SA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = sa::gdn_workspace_bytes(cfg->batch, cfg->heads, cfg->head_dim, cfg->tokens);
  return SA_OK;
}

sa_status sa_gdn_chunk(const sa_gdn_config* cfg, float* state, const void* q, const void* k,
                       const void* v, const float* g, const float* beta, void* out,
                       void* workspace, size_t workspace_bytes, const uint8_t* active,
                       sa_stream_t stream) {
  sa_status vst = validate_gdn_config(cfg);
  if (vst != SA_OK) return vst;
  if (!state) return fail(SA_ERR_INVALID_ARG, "state is NULL");
  if (reinterpret_cast<uintptr_t>(state) % 16)
    return fail(SA_ERR_INVALID_ARG, "state must be 16-byte aligned");
  if (cfg->tokens > 0) {
    if (!q || !k || !v || !g || !beta || !out)
      return fail(SA_ERR_INVALID_ARG, "q, k, v, g, beta and out must be non-NULL");
    const uintptr_t ptrs[3] = {(uintptr_t)q, (uintptr_t)k, (uintptr_t)v};
    for (uintptr_t a : ptrs)
      if (a % 16) return fail(SA_ERR_INVALID_ARG, "q, k and v must be 16-byte aligned");
    if ((uintptr_t)out % 16) return fail(SA_ERR_INVALID_ARG, "out must be 16-byte aligned");
    if ((uintptr_t)g % 4 || (uintptr_t)beta % 4)
      return fail(SA_ERR_INVALID_ARG, "g and beta must be 4-byte aligned");
    const size_t need = sa::gdn_workspace_bytes(cfg->batch, cfg->heads, cfg->head_dim, cfg->tokens);
    if (!workspace || (uintptr_t)workspace % 16)
      return fail(SA_ERR_INVALID_ARG, "workspace must be non-NULL and 16-byte aligned");
    if (workspace_bytes < need)
      return fail(SA_ERR_INVALID_ARG, "workspace has %zu bytes, %zu needed (sa_gdn_workspace_size)",
                  workspace_bytes, need);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SA_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10)
    return fail(SA_ERR_UNSUPPORTED, "device %d is sm_%d; this library runs on sm_100a (B200)", dev,
                major * 10);
  sa::GdnParams p;
  memset(&p, 0, sizeof(p));
  for (int b = 0; b < cfg->batch; ++b)
    if (!active || active[b]) p.stream_of[p.n_streams++] = b;
  if (p.n_streams == 0 || cfg->tokens == 0) return SA_OK;
  p.state = state;
  p.q = q;
  p.k = k;
  p.v = v;
  p.g = g;
  p.beta = beta;
  p.out = out;
  p.workspace = static_cast<float*>(workspace);
  p.T = cfg->tokens;
  p.n_sub = (int32_t)((cfg->tokens + 63) / 64);
  p.batch = cfg->batch;
  p.H = cfg->heads;
  p.scale = cfg->scale > 0.f ? cfg->scale : (float)(1.0 / sqrt((double)cfg->head_dim));
  NvtxRange nv("sa_gdn_chunk");
  e = sa::launch_gdn(p, cfg->head_dim, cfg->dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gdn launch");
  return SA_OK;
}

sa_status sa_gdn_device_status(const void* workspace, sa_stream_t stream) {
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 16)
    return fail(SA_ERR_INVALID_ARG, "workspace must be non-NULL and 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "gdn status read");
  if (word & sa::kDeviceErrTimeout)
    return fail(SA_ERR_DEVICE_TIMEOUT, "a bounded wait of the last sa_gdn_chunk call gave up; its "
                                       "outputs and state are not valid");
  return SA_OK;
}

const char* sa_last_error_string(void) { return g_last_error.c_str(); }

sa_status sa_plan_chunk(const sa_config* cfg, int64_t frames_written, int64_t pos_base,
                        sa_chunk_plan* plan) {
  sa_status st = validate_config(cfg);
  if (st != SA_OK) return st;
  if (!plan) return fail(SA_ERR_INVALID_ARG, "plan is NULL");
  return plan_chunk(cfg, frames_written, pos_base, plan);
}

sa_status sa_refresh_delta(const sa_config* cfg, int64_t frames_written, int64_t pos_base,
                           int64_t* delta) {
  sa_status st = validate_config(cfg);
  if (st != SA_OK) return st;
  if (!delta) return fail(SA_ERR_INVALID_ARG, "delta is NULL");
  if (frames_written < 0 || frames_written % cfg->chunk_frames != 0)
    return fail(SA_ERR_STATE, "frames_written is not a multiple of the chunk size");
  *delta = refresh_delta(cfg, frames_written, pos_base);
  return SA_OK;
}

sa_status sa_cache_create(const sa_config* cfg, sa_stream_t stream, sa_cache** out) {
  if (!out) return fail(SA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  sa_status st = validate_config(cfg);
  if (st != SA_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SA_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10)
    return fail(SA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100a (B200)",
                dev, prop.major, prop.minor);

  sa_cache* h = new sa_cache();
  h->cfg = *cfg;
  h->dev = dev;
  h->num_sms = prop.multiProcessorCount;
  h->create_stream = static_cast<cudaStream_t>(stream);
  h->F = (int64_t)cfg->frame_h * cfg->frame_w;
  h->Lc = h->F * cfg->chunk_frames;
  h->R = (int64_t)cfg->window_frames + cfg->chunk_frames;
  h->sf = h->F * cfg->sink_frames;
  h->ntok = h->sf + h->R * h->F;
  h->esz = cfg->dtype == SA_F32 ? 4 : 2;
  h->cesz = cfg->dtype == SA_BF16_E4M3 ? 1 : h->esz;
  h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : (float)(1.0 / sqrt((double)cfg->head_dim));
  h->frames_written.assign(cfg->batch, 0);
  h->pos_base.assign(cfg->batch, 0);
  const int64_t B = cfg->batch, H = cfg->heads, D = cfg->head_dim;
  const size_t cache_bytes = (size_t)(B * H * h->ntok * D) * h->cesz;
  const size_t raw_bytes = (size_t)(B * H * std::max<int64_t>(h->sf, 1) * D) * h->esz;
  const size_t ws_bytes = (size_t)(B * H * h->Lc * D) * h->cesz;
  const int dh2 = cfg->rope_dims[1] / 2, dw2 = cfg->rope_dims[2] / 2;
  cudaStream_t cs = h->create_stream;
  h->fault = fault_from_env();
  if (h->fault == FAULT_ALLOC) {
    free_all(h);
    delete h;
    return cuda_fail(cudaErrorMemoryAllocation, "cudaMalloc (injected by SA_FAULT=alloc)");
  }
  struct Alloc { void** p; size_t n; } allocs[] = {
      {&h->k_cache, cache_bytes}, {&h->v_cache, cache_bytes}, {&h->k_raw, raw_bytes},
      {&h->q_ws, ws_bytes},
      {reinterpret_cast<void**>(&h->htab), sizeof(float2) * (size_t)std::max(1, cfg->frame_h * dh2)},
      {reinterpret_cast<void**>(&h->wtab), sizeof(float2) * (size_t)std::max(1, cfg->frame_w * dw2)},
      {reinterpret_cast<void**>(&h->d_status), 256}};
  for (auto& a : allocs) {
    e = cudaMalloc(a.p, a.n);
    if (e != cudaSuccess) {
      free_all(h);
      delete h;
      return cuda_fail(e, "cudaMalloc");
    }
    e = cudaMemsetAsync(*a.p, 0, a.n, cs);
    if (e != cudaSuccess) {
      free_all(h);
      delete h;
      return cuda_fail(e, "cudaMemsetAsync");
    }
  }
  // spatial RoPE tables: fp64 on the host, stored fp32
  std::vector<float2> ht((size_t)std::max(1, cfg->frame_h * dh2)), wt((size_t)std::max(1, cfg->frame_w * dw2));
  for (int y = 0; y < cfg->frame_h; ++y)
    for (int j = 0; j < dh2; ++j) {
      const double ang = (double)y * theta(cfg, 1, j);
      ht[(size_t)y * dh2 + j] = make_float2((float)cos(ang), (float)sin(ang));
    }
  for (int x = 0; x < cfg->frame_w; ++x)
    for (int j = 0; j < dw2; ++j) {
      const double ang = (double)x * theta(cfg, 2, j);
      wt[(size_t)x * dw2 + j] = make_float2((float)cos(ang), (float)sin(ang));
    }
  e = cudaMemcpyAsync(h->htab, ht.data(), sizeof(float2) * ht.size(), cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->wtab, wt.data(), sizeof(float2) * wt.size(), cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);  // the host tables go out of scope
  if (e != cudaSuccess) {
    free_all(h);
    delete h;
    return cuda_fail(e, "table upload");
  }
  if (cfg->dtype == SA_BF16_E4M3) {  // per-head scales, all 1 until set
    h->fp8_scale.assign((size_t)(3 * H), 1.f);
    e = cudaMalloc(&h->d_fp8_scale, sizeof(float) * h->fp8_scale.size());
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(h->d_fp8_scale, h->fp8_scale.data(), sizeof(float) * h->fp8_scale.size(),
                          cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) {
      free_all(h);
      delete h;
      return cuda_fail(e, "fp8 scales");
    }
  }
  if (cfg->dtype != SA_F32) {
    const int64_t max_units = B * H * ((h->Lc + 255) / 256);
    h->partials_bytes = sa::attend_partials_bytes((int)D, h->num_sms, max_units);
    e = cudaMalloc(&h->partials, h->partials_bytes);
    if (e == cudaSuccess) {  // the split-unit arrival counters start at zero
      e = cudaMemsetAsync(h->partials, 0, h->partials_bytes, cs);
      if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
      if (e != cudaSuccess) {
        cudaFree(h->partials);
        h->partials = nullptr;
        free_all(h);
        delete h;
        return cuda_fail(e, "partials init");
      }
    }
    if (e != cudaSuccess) {
      h->partials = nullptr;
      free_all(h);
      delete h;
      return cuda_fail(e, "cudaMalloc(partials)");
    }
    const bool f8 = cfg->dtype == SA_BF16_E4M3;
    if (!make_map(&h->tm_q, h->q_ws, D, h->Lc, B * H, f8) ||
        !make_map(&h->tm_k, h->k_cache, D, h->ntok, B * H, f8) ||
        !make_map(&h->tm_v, h->v_cache, D, h->ntok, B * H, f8)) {
      free_all(h);
      delete h;
      return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    }
  }
  *out = h;
  return SA_OK;
}

sa_status sa_cache_destroy(sa_cache* h) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  cudaStreamSynchronize(h->create_stream);
  free_all(h);
  delete h;
  return SA_OK;
}

sa_status sa_cache_reset(sa_cache* h, const uint8_t* streams) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  for (int b = 0; b < h->cfg.batch; ++b)
    if (!streams || streams[b]) {
      h->frames_written[b] = 0;
      h->pos_base[b] = 0;
    }
  return SA_OK;
}

namespace {
// RoPE + append of the next chunk, then attention; `commit` advances the
// streams' frame counts (sa_append_attend), otherwise the chunk's rows are
// rewritten by the next call (sa_attend).
sa_status append_attend(sa_cache* h, const void* q, const void* k, const void* v, void* out,
                        const uint8_t* active, sa_stream_t stream, bool commit) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (!q || !k || !v || !out) return fail(SA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  const sa_config& c = h->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<int> act;
  active_list(h, active, act);
  if (act.empty()) return SA_OK;

  // plans for every active stream (validated before anything is launched)
  std::vector<sa_chunk_plan> plans(act.size());
  for (size_t i = 0; i < act.size(); ++i) {
    sa_status s = plan_chunk(&c, h->frames_written[act[i]], h->pos_base[act[i]], &plans[i]);
    if (s != SA_OK) return s;
  }
  const int C = c.chunk_frames, dt2 = c.rope_dims[0] / 2;
  if (h->fault == FAULT_LAUNCH || h->fault == FAULT_LAUNCH_ONCE) {
    if (h->fault == FAULT_LAUNCH_ONCE) h->fault = FAULT_NONE;
    return cuda_fail(cudaErrorLaunchFailure, "append launch (injected by SA_FAULT)");
  }
  // ---- K1: fused RoPE + append, up to kMaxEntries (stream, frame) entries per launch
  const int per_launch = std::max(1, sa::kMaxEntries / C);
  for (size_t s0 = 0; s0 < act.size(); s0 += per_launch) {
    sa::AppendParams p;
    memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v;
    p.q_ws = h->q_ws; p.k_cache = h->k_cache; p.v_cache = h->v_cache; p.k_raw = h->k_raw;
    p.fp8_scale = h->d_fp8_scale;
    p.htab = h->htab; p.wtab = h->wtab;
    p.H = c.heads; p.D = c.head_dim; p.fw = c.frame_w; p.F = (int32_t)h->F; p.C = C;
    p.Lc = (int32_t)h->Lc; p.ntok = h->ntok; p.sf = h->sf;
    p.dt2 = dt2; p.dh2 = c.rope_dims[1] / 2; p.dw2 = c.rope_dims[2] / 2;
    const size_t n = std::min(act.size() - s0, (size_t)per_launch);
    p.n_streams = (int32_t)n;
    p.batch = c.batch;
    for (size_t a = 0; a < n; ++a) {
      const sa_chunk_plan& pl = plans[s0 + a];
      p.stream_of[a] = act[s0 + a];
      for (int i = 0; i < C; ++i) {
        const int e = (int)a * C + i;
        p.dest_row[e] = pl.dest_row[i];
        p.raw_row[e] = pl.is_sink[i] ? pl.dest_row[i] : -1;
        for (int j = 0; j < dt2; ++j) {
          const double ang = (double)pl.t_pos[i] * theta(&c, 0, j);
          p.tcs[e][j] = make_float2((float)cos(ang), (float)sin(ang));
        }
      }
    }
    NvtxRange nv("sa.append");
    prof_before(h, st, KIND_APPEND);
    cudaError_t e = sa::launch_append(p, c.dtype, h->num_sms, st);
    prof_after(h, st);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    h->kernels += 1;
  }
  // ---- K2: attention, streams ordered by decreasing key count
  std::vector<int> order(act.size());
  for (size_t i = 0; i < act.size(); ++i) order[i] = (int)i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int x, int y) { return plans[x].n_keys > plans[y].n_keys; });
  sa::AttnParams ap;
  memset(&ap, 0, sizeof(ap));
  ap.H = c.heads; ap.Lc = (int32_t)h->Lc; ap.ntok = h->ntok;
  ap.n_q_tiles = (int32_t)((h->Lc + 127) / 128);
  ap.n_streams = (int32_t)act.size();
  ap.batch = c.batch;
  ap.scale_log2 = (float)((double)h->scale * 1.4426950408889634);
  ap.out = out; ap.q_ws = h->q_ws; ap.k_cache = h->k_cache; ap.v_cache = h->v_cache;
  ap.status = h->d_status;
  ap.fp8 = c.dtype == SA_BF16_E4M3;
  if (ap.fp8)
    for (int hh = 0; hh < c.heads; ++hh) {
      ap.inv_qk[hh] = 1.f / (h->fp8_scale[hh] * h->fp8_scale[c.heads + hh]);
      ap.inv_v[hh] = 1.f / h->fp8_scale[2 * c.heads + hh];
    }
  for (size_t i = 0; i < act.size(); ++i) {
    ap.stream_of[i] = act[order[i]];
    ap.n_keys[i] = (int32_t)plans[order[i]].n_keys;
  }
  NvtxRange nv("sa.attend");
  prof_before(h, st, KIND_ATTEND);
  int n_att = 1;
  cudaError_t e = c.dtype != SA_F32
                      ? sa::launch_attend_tc_bf16(ap, c.head_dim, &h->tm_q, &h->tm_k, &h->tm_v,
                                                  h->partials, h->partials_bytes, h->num_sms, st,
                                                  &n_att)
                      : sa::launch_attend_simt_f32(ap, c.head_dim, st);
  prof_after(h, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  h->kernels += n_att;
  if (commit)
    for (int b : act) h->frames_written[b] += C;
  return SA_OK;
}
}  // namespace

sa_status sa_append_attend(sa_cache* h, const void* q, const void* k, const void* v, void* out,
                           const uint8_t* active, sa_stream_t stream) {
  return append_attend(h, q, k, v, out, active, stream, true);
}

sa_status sa_attend(sa_cache* h, const void* q, const void* k, const void* v, void* out,
                    const uint8_t* active, sa_stream_t stream) {
  return append_attend(h, q, k, v, out, active, stream, false);
}

sa_status sa_rope_refresh(sa_cache* h, const uint8_t* active, sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  const sa_config& c = h->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<int> act, todo;
  active_list(h, active, act);
  for (int b : act)
    if (h->frames_written[b] > 0) todo.push_back(b);
  if (todo.empty()) return SA_OK;
  const int S = c.sink_frames, dt2 = c.rope_dims[0] / 2;
  int per_launch = sa::kMaxRefresh;
  if (S > 0) per_launch = std::max(1, std::min(per_launch, sa::kMaxRefresh / S));
  if (S > sa::kMaxRefresh)
    return fail(SA_ERR_UNSUPPORTED, "refresh supports at most %d sink frames", sa::kMaxRefresh);
  std::vector<int64_t> deltas(todo.size());
  for (size_t i = 0; i < todo.size(); ++i)
    deltas[i] = refresh_delta(&c, h->frames_written[todo[i]], h->pos_base[todo[i]]);
  for (size_t s0 = 0; s0 < todo.size(); s0 += per_launch) {
    sa::RefreshParams p;
    memset(&p, 0, sizeof(p));
    p.k_cache = h->k_cache; p.k_raw = h->k_raw; p.htab = h->htab; p.wtab = h->wtab;
    p.fp8_scale = h->d_fp8_scale; p.v_cache = h->v_cache;
    p.H = c.heads; p.D = c.head_dim; p.fw = c.frame_w; p.F = (int32_t)h->F; p.S = S;
    p.ntok = h->ntok; p.sf = h->sf;
    p.dt2 = dt2; p.dh2 = c.rope_dims[1] / 2; p.dw2 = c.rope_dims[2] / 2;
    const size_t n = std::min(todo.size() - s0, (size_t)per_launch);
    p.n_streams = (int32_t)n;
    p.batch = c.batch;
    for (size_t a = 0; a < n; ++a) {
      const int b = todo[s0 + a];
      const int64_t fw_ = h->frames_written[b];
      const int64_t new_base = h->pos_base[b] + deltas[s0 + a];
      p.stream_of[a] = b;
      p.sink_rows[a] = std::min<int64_t>(S, fw_) * h->F;
      p.ring_rows[a] = std::min<int64_t>(std::max<int64_t>(0, fw_ - S), h->R) * h->F;
      for (int j = 0; j < dt2; ++j) {
        const double ang = -(double)deltas[s0 + a] * theta(&c, 0, j);
        p.dcs[a][j] = make_float2((float)cos(ang), (float)sin(ang));
      }
      const int64_t sb = sink_base(h, new_base);
      for (int s = 0; s < S; ++s)
        for (int j = 0; j < dt2; ++j) {
          const double ang = (double)(s - sb) * theta(&c, 0, j);
          p.scs[a * S + s][j] = make_float2((float)cos(ang), (float)sin(ang));
        }
    }
    NvtxRange nv("sa.refresh");
    prof_before(h, st, KIND_REFRESH);
    cudaError_t e = sa::launch_refresh(p, c.dtype, h->num_sms, st);
    prof_after(h, st);
    if (e != cudaSuccess) return cuda_fail(e, "refresh launch");
    h->kernels += 1;
  }
  for (size_t i = 0; i < todo.size(); ++i) h->pos_base[todo[i]] += deltas[i];
  return SA_OK;
}

sa_status sa_cache_set_fp8_scales(sa_cache* h, const float* q_scale, const float* k_scale,
                                  const float* v_scale) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (h->cfg.dtype != SA_BF16_E4M3)
    return fail(SA_ERR_INVALID_ARG, "per-head fp8 scales need dtype SA_BF16_E4M3");
  for (int b = 0; b < h->cfg.batch; ++b)
    if (h->frames_written[b] > 0)
      return fail(SA_ERR_STATE, "scales must be set before any stream holds a frame");
  const int H = h->cfg.heads;
  std::vector<float> sc((size_t)(3 * H), 1.f);
  const float* src[3] = {q_scale, k_scale, v_scale};
  for (int t = 0; t < 3; ++t)
    for (int i = 0; i < H && src[t]; ++i) {
      if (!(src[t][i] > 0.f) || !isfinite(src[t][i]))
        return fail(SA_ERR_INVALID_ARG, "scale %d of tensor %d is not positive and finite", i, t);
      sc[(size_t)t * H + i] = src[t][i];
    }
  cudaError_t e = cudaMemcpyAsync(h->d_fp8_scale, sc.data(), sizeof(float) * sc.size(),
                                  cudaMemcpyHostToDevice, h->create_stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(h->create_stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp8 scale upload");
  h->fp8_scale = sc;
  return SA_OK;
}

sa_status sa_cache_get_fp8_scales(const sa_cache* h, float* q_scale, float* k_scale,
                                  float* v_scale) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (h->cfg.dtype != SA_BF16_E4M3)
    return fail(SA_ERR_INVALID_ARG, "per-head fp8 scales need dtype SA_BF16_E4M3");
  float* dst[3] = {q_scale, k_scale, v_scale};
  const size_t H = (size_t)h->cfg.heads;
  for (int t = 0; t < 3; ++t)
    if (dst[t]) memcpy(dst[t], h->fp8_scale.data() + t * H, sizeof(float) * H);
  return SA_OK;
}

sa_status sa_cache_set_sink_mode(sa_cache* h, int32_t mode) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (mode != SA_SINK_SHIFT && mode != SA_SINK_REPIN)
    return fail(SA_ERR_INVALID_ARG, "sink mode %d is not SA_SINK_SHIFT or SA_SINK_REPIN", mode);
  h->sink_mode = mode;
  return SA_OK;
}

sa_status sa_sink_update(sa_cache* h, const void* k_new, const void* v_new, float alpha,
                         const uint8_t* active, sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  const sa_config& c = h->cfg;
  const int S = c.sink_frames, dt2 = c.rope_dims[0] / 2;
  if (S <= 0) return fail(SA_ERR_INVALID_ARG, "the cache has no sink (sink_frames = 0)");
  if (!k_new || !v_new) return fail(SA_ERR_INVALID_ARG, "k_new and v_new must be non-NULL");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(SA_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  if (!(alpha >= 0.f && alpha <= 1.f)) return fail(SA_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (S > sa::kMaxRefresh)
    return fail(SA_ERR_UNSUPPORTED, "sink update supports at most %d sink frames", sa::kMaxRefresh);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<int> act;
  active_list(h, active, act);
  for (int b : act)
    if (h->frames_written[b] < S)
      return fail(SA_ERR_STATE, "stream %d: the sink is not complete (%lld of %d frames)", b,
                  (long long)h->frames_written[b], S);
  if (act.empty()) return SA_OK;
  const int per_launch = std::max(1, sa::kMaxRefresh / S);
  for (size_t s0 = 0; s0 < act.size(); s0 += per_launch) {
    sa::RefreshParams p;
    memset(&p, 0, sizeof(p));
    p.k_cache = h->k_cache; p.k_raw = h->k_raw; p.htab = h->htab; p.wtab = h->wtab;
    p.fp8_scale = h->d_fp8_scale; p.v_cache = h->v_cache;
    p.v_cache = h->v_cache; p.k_new = k_new; p.v_new = v_new; p.alpha = alpha; p.update = 1;
    p.H = c.heads; p.D = c.head_dim; p.fw = c.frame_w; p.F = (int32_t)h->F; p.S = S;
    p.ntok = h->ntok; p.sf = h->sf;
    p.dt2 = dt2; p.dh2 = c.rope_dims[1] / 2; p.dw2 = c.rope_dims[2] / 2;
    const size_t n = std::min(act.size() - s0, (size_t)per_launch);
    p.n_streams = (int32_t)n;
    p.batch = c.batch;
    for (size_t a = 0; a < n; ++a) {
      const int b = act[s0 + a];
      p.stream_of[a] = b;
      p.sink_rows[a] = (int64_t)S * h->F;
      p.ring_rows[a] = 0;
      const int64_t sb = sink_base(h, h->pos_base[b]);
      for (int s = 0; s < S; ++s)
        for (int j = 0; j < dt2; ++j) {
          const double ang = (double)(s - sb) * theta(&c, 0, j);
          p.scs[a * S + s][j] = make_float2((float)cos(ang), (float)sin(ang));
        }
    }
    NvtxRange nv("sa.sink_update");
    prof_before(h, st, KIND_REFRESH);
    cudaError_t e = sa::launch_refresh(p, c.dtype, h->num_sms, st);
    prof_after(h, st);
    if (e != cudaSuccess) return cuda_fail(e, "sink update launch");
    h->kernels += 1;
  }
  return SA_OK;
}

sa_status sa_append_attend_host(sa_cache* h, const void* q, const void* k, const void* v,
                                void* out, const uint8_t* active, sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (!q || !k || !v || !out) return fail(SA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t per = (size_t)(h->Lc * h->cfg.heads * h->cfg.head_dim) * h->esz;
  const size_t total = per * (size_t)h->cfg.batch;
  for (int i = 0; i < 4; ++i) {
    if (!h->stage[i]) {
      cudaError_t e = cudaMalloc(&h->stage[i], total);
      if (e != cudaSuccess) return cuda_fail(e, "staging cudaMalloc");
    }
  }
  std::vector<int> act;
  active_list(h, active, act);
  const void* src[3] = {q, k, v};
  for (int t = 0; t < 3; ++t)
    for (int b : act) {
      cudaError_t e = cudaMemcpyAsync(static_cast<char*>(h->stage[t]) + per * b,
                                      static_cast<const char*>(src[t]) + per * b, per,
                                      cudaMemcpyHostToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    }
  sa_status s = sa_append_attend(h, h->stage[0], h->stage[1], h->stage[2], h->stage[3], active, stream);
  if (s != SA_OK) return s;
  for (int b : act) {
    cudaError_t e = cudaMemcpyAsync(static_cast<char*>(out) + per * b,
                                    static_cast<const char*>(h->stage[3]) + per * b, per,
                                    cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  }
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  return SA_OK;
}

sa_status sa_append_attend_host_async(sa_cache* h, const void* q, const void* k, const void* v,
                                      void* out, const uint8_t* active, sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (!q || !k || !v || !out) return fail(SA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t per = (size_t)(h->Lc * h->cfg.heads * h->cfg.head_dim) * h->esz;
  const size_t total = per * (size_t)h->cfg.batch;
  cudaError_t e = cudaSuccess;
  if (!h->copy_in) {  // first call: streams, events and staging slots
    e = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking);
    for (int s = 0; s < sa_cache::kSlots && e == cudaSuccess; ++s) {
      for (cudaEvent_t* ev : {&h->in_done[s], &h->comp_done[s], &h->out_done[s]})
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
      for (int t = 0; t < 4 && e == cudaSuccess; ++t) e = cudaMalloc(&h->slot_buf[s][t], total);
    }
    if (e != cudaSuccess) return cuda_fail(e, "host pipeline setup");
  }
  std::vector<int> act;
  active_list(h, active, act);
  if (act.empty()) return SA_OK;
  // validate the chunk plans before any copy is queued
  for (int b : act) {
    sa_chunk_plan pl;
    sa_status s = plan_chunk(&h->cfg, h->frames_written[b], h->pos_base[b], &pl);
    if (s != SA_OK) return s;
  }
  const int slot = (int)(h->async_calls % sa_cache::kSlots);
  void** buf = h->slot_buf[slot];
  // copy-in: the slot's inputs are free once its previous compute finished
  e = cudaStreamWaitEvent(h->copy_in, h->comp_done[slot], 0);
  const void* src[3] = {q, k, v};
  for (int t = 0; t < 3 && e == cudaSuccess; ++t)
    for (int b : act) {
      e = cudaMemcpyAsync(static_cast<char*>(buf[t]) + per * b,
                          static_cast<const char*>(src[t]) + per * b, per,
                          cudaMemcpyHostToDevice, h->copy_in);
      if (e != cudaSuccess) break;
    }
  if (e == cudaSuccess) e = cudaEventRecord(h->in_done[slot], h->copy_in);
  // compute on the caller's stream after the inputs landed and after the
  // slot's previous output left the device
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, h->in_done[slot], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, h->out_done[slot], 0);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline copy-in");
  sa_status s = sa_append_attend(h, buf[0], buf[1], buf[2], buf[3], active, stream);
  if (s != SA_OK) return s;
  e = cudaEventRecord(h->comp_done[slot], st);
  // copy-out once the chunk is computed
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_out, h->comp_done[slot], 0);
  for (int b : act) {
    if (e != cudaSuccess) break;
    e = cudaMemcpyAsync(static_cast<char*>(out) + per * b,
                        static_cast<const char*>(buf[3]) + per * b, per,
                        cudaMemcpyDeviceToHost, h->copy_out);
  }
  if (e == cudaSuccess) e = cudaEventRecord(h->out_done[slot], h->copy_out);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline copy-out");
  ++h->async_calls;
  return SA_OK;
}

sa_status sa_host_wait(sa_cache* h) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  cudaError_t e = cudaSuccess;
  if (h->copy_in) e = cudaStreamSynchronize(h->copy_in);
  if (e == cudaSuccess && h->copy_out) e = cudaStreamSynchronize(h->copy_out);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline wait");
  return SA_OK;
}

namespace {
// Checkpoint header; followed by frames_written[B], pos_base[B] (int64),
// the e4m3 scales [3H] (float, e4m3 caches only), then K', V, raw sink keys.
struct CkptHeader {
  char magic[8];  // "SACKPT01"
  int32_t abi;
  int32_t sink_mode;
  sa_config cfg;
  uint64_t cache_bytes, raw_bytes, total_bytes;
};

void ckpt_sizes(const sa_cache* h, size_t& meta, size_t& cache, size_t& raw, size_t& total) {
  const sa_config& c = h->cfg;
  cache = (size_t)(c.batch * (int64_t)c.heads * h->ntok * c.head_dim) * h->cesz;
  raw = (size_t)(c.batch * (int64_t)c.heads * std::max<int64_t>(h->sf, 1) * c.head_dim) * h->esz;
  meta = sizeof(CkptHeader) + 2 * sizeof(int64_t) * (size_t)c.batch +
         (c.dtype == SA_BF16_E4M3 ? sizeof(float) * 3 * (size_t)c.heads : 0);
  meta = (meta + 255) & ~(size_t)255;
  total = meta + 2 * cache + raw;
}
}  // namespace

sa_status sa_cache_export_size(const sa_cache* h, size_t* bytes) {
  if (!h || !bytes) return fail(SA_ERR_INVALID_ARG, "handle and bytes must be non-NULL");
  size_t meta, cache, raw, total;
  ckpt_sizes(h, meta, cache, raw, total);
  *bytes = total;
  return SA_OK;
}

sa_status sa_cache_export(const sa_cache* h, void* dst, size_t cap, sa_stream_t stream) {
  if (!h || !dst) return fail(SA_ERR_INVALID_ARG, "handle and dst must be non-NULL");
  size_t meta, cache, raw, total;
  ckpt_sizes(h, meta, cache, raw, total);
  if (cap < total) return fail(SA_ERR_INVALID_ARG, "checkpoint needs %zu bytes, got %zu", total, cap);
  char* out = static_cast<char*>(dst);
  memset(out, 0, meta);
  CkptHeader hd;
  memset(&hd, 0, sizeof(hd));
  memcpy(hd.magic, "SACKPT01", 8);
  hd.abi = SA_ABI_VERSION;
  hd.sink_mode = h->sink_mode;
  hd.cfg = h->cfg;
  hd.cache_bytes = cache;
  hd.raw_bytes = raw;
  hd.total_bytes = total;
  memcpy(out, &hd, sizeof(hd));
  const size_t B = (size_t)h->cfg.batch;
  memcpy(out + sizeof(hd), h->frames_written.data(), sizeof(int64_t) * B);
  memcpy(out + sizeof(hd) + sizeof(int64_t) * B, h->pos_base.data(), sizeof(int64_t) * B);
  if (h->cfg.dtype == SA_BF16_E4M3)
    memcpy(out + sizeof(hd) + 2 * sizeof(int64_t) * B, h->fp8_scale.data(),
           sizeof(float) * h->fp8_scale.size());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(out + meta, h->k_cache, cache, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out + meta + cache, h->v_cache, cache, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out + meta + 2 * cache, h->k_raw, raw, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "checkpoint export");
  return SA_OK;
}

sa_status sa_cache_import(sa_cache* h, const void* src, size_t size, sa_stream_t stream) {
  if (!h || !src) return fail(SA_ERR_INVALID_ARG, "handle and src must be non-NULL");
  size_t meta, cache, raw, total;
  ckpt_sizes(h, meta, cache, raw, total);
  if (size != total) return fail(SA_ERR_INVALID_ARG, "checkpoint of %zu bytes, expected %zu", size, total);
  const char* in = static_cast<const char*>(src);
  CkptHeader hd;
  memcpy(&hd, in, sizeof(hd));
  if (memcmp(hd.magic, "SACKPT01", 8) != 0 || hd.abi != SA_ABI_VERSION)
    return fail(SA_ERR_INVALID_ARG, "not a checkpoint of this library version");
  if (memcmp(&hd.cfg, &h->cfg, sizeof(sa_config)) != 0 || hd.cache_bytes != cache ||
      hd.raw_bytes != raw || hd.total_bytes != total)
    return fail(SA_ERR_INVALID_ARG, "checkpoint of another configuration");
  if (hd.sink_mode != SA_SINK_SHIFT && hd.sink_mode != SA_SINK_REPIN)
    return fail(SA_ERR_INVALID_ARG, "damaged checkpoint header");
  const size_t B = (size_t)h->cfg.batch;
  std::vector<int64_t> fw(B), pb(B);
  memcpy(fw.data(), in + sizeof(hd), sizeof(int64_t) * B);
  memcpy(pb.data(), in + sizeof(hd) + sizeof(int64_t) * B, sizeof(int64_t) * B);
  for (size_t b = 0; b < B; ++b)
    if (fw[b] < 0 || fw[b] % h->cfg.chunk_frames != 0 || pb[b] < 0 || pb[b] > fw[b])
      return fail(SA_ERR_INVALID_ARG, "damaged checkpoint stream state");
  std::vector<float> sc = h->fp8_scale;
  if (h->cfg.dtype == SA_BF16_E4M3)
    memcpy(sc.data(), in + sizeof(hd) + 2 * sizeof(int64_t) * B, sizeof(float) * sc.size());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(h->k_cache, in + meta, cache, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->v_cache, in + meta + cache, cache, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->k_raw, in + meta + 2 * cache, raw, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && h->cfg.dtype == SA_BF16_E4M3)
    e = cudaMemcpyAsync(h->d_fp8_scale, sc.data(), sizeof(float) * sc.size(),
                        cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "checkpoint import");
  h->frames_written = fw;
  h->pos_base = pb;
  h->sink_mode = hd.sink_mode;
  h->fp8_scale = sc;
  return SA_OK;
}

sa_status sa_stream_state(const sa_cache* h, int32_t b, int64_t* frames_written,
                          int64_t* pos_base) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (b < 0 || b >= h->cfg.batch) return fail(SA_ERR_INVALID_ARG, "stream index out of range");
  if (frames_written) *frames_written = h->frames_written[b];
  if (pos_base) *pos_base = h->pos_base[b];
  return SA_OK;
}

sa_status sa_cache_copy_out(const sa_cache* h, int32_t b, void* host_k, void* host_v,
                            sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (b < 0 || b >= h->cfg.batch) return fail(SA_ERR_INVALID_ARG, "stream index out of range");
  if (!host_k || !host_v) return fail(SA_ERR_INVALID_ARG, "host buffers must be non-NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)(h->cfg.heads * h->ntok * h->cfg.head_dim) * h->cesz;
  cudaError_t e = cudaMemcpyAsync(host_k, static_cast<const char*>(h->k_cache) + n * b, n,
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(host_v, static_cast<const char*>(h->v_cache) + n * b, n,
                        cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cache copy-out");
  return SA_OK;
}

sa_status sa_get_device_status(sa_cache* h, sa_stream_t stream) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, h->d_status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->d_status, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "device status read");
  if (word & sa::kDeviceErrTimeout)
    return fail(SA_ERR_DEVICE_TIMEOUT, "a kernel abandoned a bounded wait");
  return SA_OK;
}

sa_status sa_debug_bounds_status(sa_stream_t stream) {
#ifdef SA_DEBUG_BOUNDS
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  struct {
    const char* file;
    cudaError_t (*read)(unsigned int*, cudaStream_t);
  } words[] = {{"attend_tc", sa::bounds_word_attend_tc},
               {"attend_simt", sa::bounds_word_attend_simt},
               {"rope_append", sa::bounds_word_rope_append},
               {"gdn", sa::bounds_word_gdn}};
  std::string bad;
  for (const auto& w : words) {
    unsigned int word = 0;
    cudaError_t e = w.read(&word, st);
    if (e != cudaSuccess) return cuda_fail(e, "bounds word read");
    if (word) {
      char buf[96];
      snprintf(buf, sizeof(buf), "%s%s sites 0x%08x", bad.empty() ? "" : ", ", w.file, word);
      bad += buf;
    }
  }
  if (!bad.empty())
    return fail(SA_ERR_DEVICE_BOUNDS, "index checks failed in kernels: %s", bad.c_str());
  return SA_OK;
#else
  (void)stream;
  return fail(SA_ERR_UNSUPPORTED, "not a debug build (libsa_debug.so has the index checks)");
#endif
}

sa_status sa_debug_bounds_selftest(sa_stream_t stream) {
#ifdef SA_DEBUG_BOUNDS
  cudaError_t e = sa::bounds_selftest(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return SA_OK;
#else
  (void)stream;
  return fail(SA_ERR_UNSUPPORTED, "not a debug build (libsa_debug.so has the index checks)");
#endif
}

sa_status sa_profile_begin(sa_cache* h) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  if (h->ev.empty()) {
    h->ev.resize(2 * 8192);
    h->ev_kind.resize(8192);
    for (auto& e : h->ev) {
      cudaError_t r = cudaEventCreate(&e);
      if (r != cudaSuccess) return cuda_fail(r, "cudaEventCreate");
    }
  }
  h->ev_used = 0;
  h->kernels = 0;
  h->profiling = true;
  return SA_OK;
}

sa_status sa_profile_launches(const sa_cache* h, int64_t* launches) {
  if (!h || !launches) return fail(SA_ERR_INVALID_ARG, "handle and launches must be non-NULL");
  *launches = h->kernels;
  return SA_OK;
}

sa_status sa_profile_end(sa_cache* h, double* append_ms, int32_t* n_append, double* attend_ms,
                         int32_t* n_attend, double* refresh_ms, int32_t* n_refresh) {
  if (!h) return fail(SA_ERR_INVALID_ARG, "handle is NULL");
  double ms[3] = {0, 0, 0};
  int32_t cnt[3] = {0, 0, 0};
  for (size_t i = 0; i + 1 < h->ev_used + 1 && i < h->ev_used; i += 2) {
    cudaError_t e = cudaEventSynchronize(h->ev[i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float t = 0.f;
    cudaEventElapsedTime(&t, h->ev[i], h->ev[i + 1]);
    const int kind = h->ev_kind[i / 2];
    ms[kind] += t;
    cnt[kind] += 1;
  }
  h->profiling = false;
  h->ev_used = 0;
  if (append_ms) *append_ms = ms[KIND_APPEND];
  if (n_append) *n_append = cnt[KIND_APPEND];
  if (attend_ms) *attend_ms = ms[KIND_ATTEND];
  if (n_attend) *n_attend = cnt[KIND_ATTEND];
  if (refresh_ms) *refresh_ms = ms[KIND_REFRESH];
  if (n_refresh) *n_refresh = cnt[KIND_REFRESH];
  return SA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of sa_append_attend.
//
// For callers that may not call the CUDA allocator at all: engines and plugin
// hosts that own every byte of device memory through their own pool, and
// real-time frame loops that cannot afford cudaMalloc/cudaFree (they may
// synchronise the whole device). The caller passes the cache buffers and the
// stream state; the one scratch buffer the path needs (the rotated-query
// workspace, the spatial RoPE tables and a device status word) lives in the
// static array below, 16 MiB, which every GPU that loads this library holds
// until the process exits. The first call on a device looks its address up
// (cudaGetSymbolAddress with that device current), so that first call should
// come before any stream capture. All calls share the array and it keeps the
// last call's contents: the status word is sticky (a call whose bounded wait
// gave up sets it; only sa_noalloc_device_status reads and clears it), and
// calls whose work overlaps on the GPU race.
// ---------------------------------------------------------------------------
#include <mutex>

#define SA_NOALLOC_SCRATCH_BYTES (16u << 20)

static __device__ __align__(256) unsigned char g_sa_noalloc_scratch[SA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};

// Device address of the static scratch on the current device. Looked up once
// per device (with that device current) and remembered.
sa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoallocMaxDevices)
    return fail(SA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kNoallocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sa_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SA_OK;
}

// Spatial RoPE tables, (cos, sin) of y * base^(-2j/d_h) and x * base^(-2j/d_w),
// evaluated in fp64 and stored as fp32.
__global__ void noalloc_tables_kernel(float2* htab, float2* wtab, int fh, int fw, int dh2,
                                      int dw2, int dh, int dw, double base) {
  const int nh = fh * dh2, nw = fw * dw2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nh + nw; i += gridDim.x * blockDim.x) {
    if (i < nh) {
      const int y = i / dh2, j = i % dh2;
      const double ang = (double)y * pow(base, -2.0 * (double)j / (double)dh);
      htab[i] = make_float2((float)cos(ang), (float)sin(ang));
    } else {
      const int k = i - nh, x = k / dw2, j = k % dw2;
      const double ang = (double)x * pow(base, -2.0 * (double)j / (double)dw);
      wtab[k] = make_float2((float)cos(ang), (float)sin(ang));
    }
  }
}

}  // namespace

extern "C" sa_status sa_append_attend_noalloc(const sa_config* cfg, void* k_cache, void* v_cache,
                                              void* k_raw, int64_t* frames_written,
                                              const int64_t* pos_base, const void* q,
                                              const void* k, const void* v, void* out,
                                              const uint8_t* active, sa_stream_t stream) {
  sa_status st = validate_config(cfg);
  if (st != SA_OK) return st;
  if (cfg->dtype == SA_BF16_E4M3)
    return fail(SA_ERR_UNSUPPORTED, "the allocation-free entry runs SA_F32 and SA_BF16 caches");
  if (!k_cache || !v_cache || !frames_written || !pos_base || !q || !k || !v || !out)
    return fail(SA_ERR_INVALID_ARG, "cache buffers, stream state, q, k, v and out must be non-NULL");
  if (cfg->sink_frames > 0 && !k_raw)
    return fail(SA_ERR_INVALID_ARG, "k_raw must be non-NULL when sink_frames > 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (k_raw && !aligned16(k_raw)))
    return fail(SA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  const sa_config& c = *cfg;
  const int64_t B = c.batch, H = c.heads, D = c.head_dim;
  const int64_t F = (int64_t)c.frame_h * c.frame_w, Lc = F * c.chunk_frames;
  const int64_t R = (int64_t)c.window_frames + c.chunk_frames, sf = F * c.sink_frames;
  const int64_t ntok = sf + R * F;
  const size_t esz = c.dtype == SA_BF16 ? 2 : 4;
  const int dt2 = c.rope_dims[0] / 2, dh2 = c.rope_dims[1] / 2, dw2 = c.rope_dims[2] / 2;
  // scratch layout: [0,256) status word | tables | (1024-aligned) Q' workspace
  const size_t tab_bytes = sizeof(float2) * (size_t)(c.frame_h * dh2 + c.frame_w * dw2);
  const size_t q_off = (256 + tab_bytes + 1023) & ~(size_t)1023;
  const size_t q_bytes = (size_t)(B * H * Lc * D) * esz;
  if (q_off + q_bytes > SA_NOALLOC_SCRATCH_BYTES)
    return fail(SA_ERR_UNSUPPORTED,
                "sa_append_attend_noalloc: needs %zu bytes of scratch (rotated queries "
                "B*H*C*F*D plus RoPE tables) but the static scratch holds %u bytes",
                q_off + q_bytes, (unsigned)SA_NOALLOC_SCRATCH_BYTES);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SA_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  int major = 0, nsm = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10)
    return fail(SA_ERR_UNSUPPORTED, "device %d is not compute capability 10.x (B200)", dev);
  std::vector<int> act;
  for (int b = 0; b < c.batch; ++b)
    if (!active || active[b]) act.push_back(b);
  if (act.empty()) return SA_OK;
  std::vector<sa_chunk_plan> plans(act.size());
  for (size_t i = 0; i < act.size(); ++i) {
    st = plan_chunk(&c, frames_written[act[i]], pos_base[act[i]], &plans[i]);
    if (st != SA_OK) return st;
  }
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != SA_OK) return st;
  char* sbase = static_cast<char*>(scratch);
  int* d_status = reinterpret_cast<int*>(sbase);
  float2* htab = reinterpret_cast<float2*>(sbase + 256);
  float2* wtab = htab + c.frame_h * dh2;
  void* q_ws = sbase + q_off;
  CUtensorMap tm_q, tm_k, tm_v;
  if (c.dtype == SA_BF16) {
    if (!make_map(&tm_q, q_ws, D, Lc, B * H) || !make_map(&tm_k, k_cache, D, ntok, B * H) ||
        !make_map(&tm_v, v_cache, D, ntok, B * H))
      return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word starts at zero (static storage) and is cleared only by
  // sa_noalloc_device_status, so an expired wait stays visible until read
  if (c.frame_h * dh2 + c.frame_w * dw2 > 0) {
    noalloc_tables_kernel<<<std::max(1, nsm), 256, 0, s>>>(
        htab, wtab, c.frame_h, c.frame_w, dh2, dw2, c.rope_dims[1], c.rope_dims[2],
        (double)c.rope_base);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "RoPE table launch");
  }
  const int C = c.chunk_frames;
  const int per_launch = std::max(1, sa::kMaxEntries / C);
  for (size_t s0 = 0; s0 < act.size(); s0 += per_launch) {
    sa::AppendParams p;
    memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v;
    p.q_ws = q_ws; p.k_cache = k_cache; p.v_cache = v_cache; p.k_raw = k_raw;
    p.htab = htab; p.wtab = wtab;
    p.H = c.heads; p.D = c.head_dim; p.fw = c.frame_w; p.F = (int32_t)F; p.C = C;
    p.Lc = (int32_t)Lc; p.ntok = ntok; p.sf = sf;
    p.dt2 = dt2; p.dh2 = dh2; p.dw2 = dw2;
    const size_t n = std::min(act.size() - s0, (size_t)per_launch);
    p.n_streams = (int32_t)n;
    p.batch = c.batch;
    for (size_t a = 0; a < n; ++a) {
      const sa_chunk_plan& pl = plans[s0 + a];
      p.stream_of[a] = act[s0 + a];
      for (int i = 0; i < C; ++i) {
        const int en = (int)a * C + i;
        p.dest_row[en] = pl.dest_row[i];
        p.raw_row[en] = pl.is_sink[i] ? pl.dest_row[i] : -1;
        for (int j = 0; j < dt2; ++j) {
          const double ang = (double)pl.t_pos[i] * theta(&c, 0, j);
          p.tcs[en][j] = make_float2((float)cos(ang), (float)sin(ang));
        }
      }
    }
    e = sa::launch_append(p, c.dtype, nsm, s);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
  }
  std::vector<int> order(act.size());
  for (size_t i = 0; i < act.size(); ++i) order[i] = (int)i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int x, int y) { return plans[x].n_keys > plans[y].n_keys; });
  sa::AttnParams ap;
  memset(&ap, 0, sizeof(ap));
  ap.H = c.heads; ap.Lc = (int32_t)Lc; ap.ntok = ntok;
  ap.n_q_tiles = (int32_t)((Lc + 127) / 128);
  ap.n_streams = (int32_t)act.size();
  ap.batch = c.batch;
  const double scale = c.softmax_scale > 0.f ? (double)c.softmax_scale : 1.0 / sqrt((double)D);
  ap.scale_log2 = (float)((double)(float)scale * 1.4426950408889634);
  ap.out = out; ap.q_ws = q_ws; ap.k_cache = k_cache; ap.v_cache = v_cache;
  ap.status = d_status;
  for (size_t i = 0; i < act.size(); ++i) {
    ap.stream_of[i] = act[order[i]];
    ap.n_keys[i] = (int32_t)plans[order[i]].n_keys;
  }
  e = c.dtype == SA_BF16 ? sa::launch_attend_tc_bf16(ap, c.head_dim, &tm_q, &tm_k, &tm_v, nullptr,
                                                     0, nsm, s, nullptr)
                         : sa::launch_attend_simt_f32(ap, c.head_dim, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  for (int b : act) frames_written[b] += C;
  return SA_OK;
}

extern "C" sa_status sa_noalloc_device_status(sa_stream_t stream) {
  void* scratch = nullptr;
  sa_status st = noalloc_scratch(&scratch);
  if (st != SA_OK) return st;
  int* d_status = static_cast<int*>(scratch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, d_status, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word != 0) {
    e = cudaMemsetAsync(d_status, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    return fail(SA_ERR_DEVICE_TIMEOUT,
                "a bounded device wait of an allocation-free call gave up (status %d); the "
                "outputs and caches those calls wrote are not valid", word);
  }
  return SA_OK;
}
