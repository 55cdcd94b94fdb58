/*
 * sa.h -- C ABI of libsa.so: per-chunk block-causal attention over a rolling
 * (sink + sliding window) KV cache with 3D RoPE, for streaming video
 * diffusion transformers, on NVIDIA B200 (sm_100a).
 *
 * What the calls compute (the pages print no formula; the plain reading):
 *  - StreamDiffusionV2 (technical summary, section 2.A.2): sink tokens keep
 *    the stream anchored; RoPE offsets are reset at block boundaries so
 *    positions stay bounded over unbounded streams -> sa_rope_refresh.
 *  - SANA-Streaming (section "hybrid diffusion transformer"): softmax blocks
 *    attend to a sliding local window plus a persistent sink chunk, a bounded
 *    context with constant memory -> the cache layout of sa_cache_create and
 *    the attention of sa_append_attend.
 *  - StreamDiT (abstract): window attention over a moving buffer of frames.
 *
 * Per stream b, frames are numbered from 0 and chunk c holds frames
 * [cC, (c+1)C). sa_append_attend appends the stream's next chunk: it rotates
 * q and k with 3D RoPE at position (t, y, x), t = frame - pos_base, stores
 * the rotated k and the raw v in the cache (the first S frames in a pinned
 * sink, later frames in a ring of R = W + C frames, slot (f - S) mod R, which
 * evicts the frame written R frames before), and lets every query of the
 * chunk attend, with softmax scale `softmax_scale`, over
 *     [ sink | the W frames before the chunk | the whole chunk ]
 * (the chunk itself bidirectionally). RoPE: the head dim splits into bands
 * (d_t | d_h | d_w); inside a band of width d, dims (2j, 2j+1) rotate by
 * pos * base^(-2j/d) as (a, b) -> (a cos - b sin, a sin + b cos).
 *
 * Conventions for every call:
 *  - Device pointers are CUDA device addresses in the current context;
 *    `stream` is a cudaStream_t passed as void*. Calls enqueue work on that
 *    stream and return without synchronising, except where noted.
 *  - Validation happens before any launch: on an error nothing is enqueued
 *    and no stream state changes. No exception crosses the ABI. The reason of
 *    the last error of the calling thread is in sa_last_error_string().
 *  - Inputs are borrowed only until the enqueued work completes. A handle is
 *    not thread-safe; use it from one host thread and one CUDA stream.
 *  - Devices other than compute capability 10.x (B200 class) are refused with
 *    SA_ERR_UNSUPPORTED. There is no CPU fallback.
 */
#ifndef SA_H
#define SA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SA_ABI_VERSION 1
#define SA_MAX_CHUNK_FRAMES 32 /* C <= 32 */
#define SA_MAX_SINK_FRAMES 32  /* S <= 32 */
#define SA_MAX_STREAMS 64      /* B <= 64 */

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,    /* a pointer, size or configuration is invalid */
  SA_ERR_UNSUPPORTED = 2,    /* no B200-class device, or a shape the library does not run */
  SA_ERR_OOM = 3,            /* device or pinned-host allocation failed */
  SA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  SA_ERR_STATE = 5,          /* call not valid in the handle's current state */
  SA_ERR_DEVICE_TIMEOUT = 6, /* a kernel gave up on a bounded wait (see sa_get_device_status) */
  SA_ERR_DEVICE_BOUNDS = 7   /* debug build: a kernel's index check failed (sa_debug_bounds_status) */
} sa_status;

/* SA_F32, SA_BF16: q, k, v, out and the cache in that type.
 * SA_BF16_E4M3: q, k, v, out in bf16; the rotated keys and values in the
 * cache, the rotated queries and the attention's P in e4m3 (OCP FP8 E4M3,
 * round to nearest even, saturating to +-448) with per-head scales
 * (sa_cache_set_fp8_scales): a value x of head h is stored as
 * e4m3(x * s[h]); both attention products run on the tensor cores in fp8
 * with fp32 accumulation. Raw sink keys stay bf16. head_dim must be 128.
 * (SANA-Streaming, system co-design: mixed-precision policy that keeps
 * sensitive layers in BF16/FP8; here applied to the cache.) */
typedef enum { SA_F32 = 0, SA_BF16 = 1, SA_BF16_E4M3 = 2 } sa_dtype;

typedef void* sa_stream_t; /* a cudaStream_t */

typedef struct {
  int32_t batch;          /* B independent streams, 1..SA_MAX_STREAMS */
  int32_t heads;          /* H */
  int32_t head_dim;       /* D: 64 or 128 */
  int32_t frame_h;        /* latent frame rows (fh) */
  int32_t frame_w;        /* latent frame columns (fw); F = fh * fw tokens per frame */
  int32_t chunk_frames;   /* C >= 1: frames appended per call */
  int32_t sink_frames;    /* S >= 0: first frames pinned forever */
  int32_t window_frames;  /* W >= 0: earlier frames each chunk also sees */
  int32_t rope_dims[3];   /* (d_t, d_h, d_w): even, sum = D, d_t <= 128 */
  float rope_base;        /* theta base (> 0), e.g. 10000 */
  float softmax_scale;    /* 0 means 1/sqrt(D) */
  int32_t dtype;          /* sa_dtype: of q, k, v, out and the cache */
} sa_config;

typedef struct sa_cache sa_cache; /* opaque */

/* Plan of one stream's next chunk (host-side bookkeeping, exposed for tests). */
typedef struct {
  int64_t chunk;        /* local chunk index c = frames_written / C */
  int64_t sink_len;     /* visible sink key tokens after the append */
  int64_t ring_len;     /* visible ring key tokens after the append */
  int64_t n_keys;       /* sink_len + ring_len: keys are cache rows [0, n_keys) */
  int32_t n_frames;     /* C */
  int32_t pad_;
  int64_t dest_row[SA_MAX_CHUNK_FRAMES]; /* cache row of each frame's first token */
  int64_t t_pos[SA_MAX_CHUNK_FRAMES];    /* temporal RoPE position of each frame */
  int32_t is_sink[SA_MAX_CHUNK_FRAMES];  /* 1 if the frame lands in the sink */
} sa_chunk_plan;

/*
 * Creates a cache for cfg->batch streams on the current device and zeroes it.
 * Device memory owned by the handle (freed by sa_cache_destroy):
 *   K' and V cache, [B][H][(S+R)F][D] each (per (b, h): S*F sink rows, then
 *   R*F ring rows); the raw (unrotated) sink keys, [B][H][S*F][D]; a rotated-
 *   query workspace, [B][H][C*F][D]; the spatial cos/sin tables (fp64 on the
 *   host, stored fp32). All streams start empty (frames_written = 0,
 *   pos_base = 0). The zeroing runs on `stream`.
 * Errors: SA_ERR_INVALID_ARG (cfg invalid or out == NULL), SA_ERR_UNSUPPORTED
 * (no compute capability 10.x device), SA_ERR_OOM, SA_ERR_CUDA.
 */
sa_status sa_cache_create(const sa_config* cfg, sa_stream_t stream, sa_cache** out);

/*
 * The hot path: appends the next chunk of every active stream and attends.
 *   q, k, v : device, [B][C*F][H][D] in cfg dtype, contiguous, 16-byte aligned.
 *   out     : device, [B][C*F][H][D] in cfg dtype; rows of inactive streams
 *             are not written.
 *   active  : host, B bytes (nonzero = active) or NULL for all streams.
 * Launches the fused RoPE + append kernel, then the attention kernel, on
 * `stream`; advances frames_written of each active stream by C afterwards.
 * Never synchronises (capturable in a CUDA graph).
 */
sa_status sa_append_attend(sa_cache* h, const void* q, const void* k, const void* v, void* out,
                           const uint8_t* active, sa_stream_t stream);

/*
 * Attention of the next chunk without committing it (StreamDiffusionV2,
 * section 2.B.2 "Stream-Batch": a chunk is denoised over several steps, and
 * each step is a forward pass over the same cached context with that step's
 * latents; section 3 reports 1-step and 4-step runs). Same arguments, layouts
 * and output as sa_append_attend: the chunk's queries attend to the cached
 * context plus the chunk's own keys and values. The chunk's rotated keys and
 * values are written into the cache rows the chunk will occupy -- ring rows
 * whose frames no chunk from this one on can see (or empty sink rows) -- but
 * frames_written and pos_base do not advance, so the next sa_attend or
 * sa_append_attend on the handle processes the same chunk again, overwriting
 * those rows; the final step of a chunk calls sa_append_attend, which commits.
 * Never synchronises (capturable in a CUDA graph). Errors as sa_append_attend.
 */
sa_status sa_attend(sa_cache* h, const void* q, const void* k, const void* v, void* out,
                    const uint8_t* active, sa_stream_t stream);

/*
 * RoPE refresh of the active streams (StreamDiffusionV2, section 2.A.2):
 * before stream b's next chunk c, every cached position is rebased by
 *   Delta = max(S, cC - W) - pos_base,
 * so the oldest non-sink frame that chunk c will see sits at t = 0 and all
 * relative offsets (hence, exactly, all scores) are kept. Ring keys have
 * their temporal band re-rotated by -Delta in place; sink keys are
 * re-derived from their raw copy at the new position (one rounding, no drift
 * over many refreshes). pos_base += Delta. Streams with no frames are skipped.
 * The caller chooses when to refresh (e.g. when c > 0 and c % period == 0).
 */
sa_status sa_rope_refresh(sa_cache* h, const uint8_t* active, sa_stream_t stream);

/* Empties the selected streams (NULL = all): frames_written = pos_base = 0.
 * Host bookkeeping only; cache contents are overwritten by later appends. */
sa_status sa_cache_reset(sa_cache* h, const uint8_t* streams);

/* Synchronises the stream given at create, frees all memory of the handle. */
sa_status sa_cache_destroy(sa_cache* h);

/*
 * Host-buffer variant of sa_append_attend: q, k, v are HOST pointers
 * ([B][C*F][H][D]); they are copied to device staging buffers owned by the
 * handle, the chunk is processed, and the result is copied back to the host
 * pointer `out` before the call returns (the call synchronises `stream`).
 * Page-locked host memory gives asynchronous copies. The staging buffers are
 * allocated by the first call on a handle.
 */
sa_status sa_append_attend_host(sa_cache* h, const void* q, const void* k, const void* v,
                                void* out, const uint8_t* active, sa_stream_t stream);

/*
 * Pipelined host-buffer variant: the same work as sa_append_attend_host, but
 * the call returns once the work is queued, so consecutive calls overlap the
 * host-to-device copies of one chunk, the computation of another and the
 * device-to-host copy of a third. The handle owns three staging slots (q, k,
 * v, out; allocated by the first call) and two copy streams; events order
 * copy-in -> compute (on `stream`) -> copy-out per slot, and a slot is reused
 * only after its previous chunk's computation and copy-out completed.
 * Ownership: q, k, v are read until their copies complete; `out` is written
 * when the copy-out completes. Call sa_host_wait before reading `out` or
 * reusing the input buffers. Page-locked host memory is needed for copies to
 * overlap (pageable memory works but serialises). Refreshes on `stream` are
 * ordered with the computations. Errors as sa_append_attend (validated before
 * any copy is queued), SA_ERR_CUDA on a copy or setup failure.
 */
sa_status sa_append_attend_host_async(sa_cache* h, const void* q, const void* k, const void* v,
                                      void* out, const uint8_t* active, sa_stream_t stream);

/* Blocks until every copy queued by sa_append_attend_host_async on the handle
 * has completed (and with them the computations they follow). */
sa_status sa_host_wait(sa_cache* h);

/* ---- checkpoint / resume ---- */

/* Bytes of a handle's checkpoint: a header (configuration, per-stream
 * frames_written and pos_base, sink mode, e4m3 scales) followed by the K' and
 * V cache and the raw sink keys. */
sa_status sa_cache_export_size(const sa_cache* h, size_t* bytes);

/* Writes the checkpoint into the host buffer dst (cap >= export size;
 * SA_ERR_INVALID_ARG otherwise). Copies on `stream` after the work queued
 * before it, then synchronises `stream`. The rotated-query workspace and the
 * attention's split-unit counters are not part of it (rewritten by every
 * call; zero between calls). A stream's continuation from an imported
 * checkpoint is bit-identical to the original's. */
sa_status sa_cache_export(const sa_cache* h, void* dst, size_t cap, sa_stream_t stream);

/* Restores a checkpoint written by sa_cache_export into a handle created
 * with the same configuration (SA_ERR_INVALID_ARG for another configuration,
 * a wrong size or a damaged header; nothing changes then). Copies on
 * `stream` and synchronises it. */
sa_status sa_cache_import(sa_cache* h, const void* src, size_t size, sa_stream_t stream);

/* ---- introspection (tests, benchmarks) ---- */

/* frames_written and pos_base of stream b (host bookkeeping; no sync). */
sa_status sa_stream_state(const sa_cache* h, int32_t b, int64_t* frames_written,
                          int64_t* pos_base);

/* Copies stream b's cache to host: host_k and host_v receive [H][(S+R)F][D]
 * each in the cache's element type (SA_BF16_E4M3: e4m3 bytes, scaled by the
 * head's k or v scale); rows of never-written slots are zero. Synchronous. */
sa_status sa_cache_copy_out(const sa_cache* h, int32_t b, void* host_k, void* host_v,
                            sa_stream_t stream);

/* Synchronises `stream`, reads and clears the device error word. Returns
 * SA_ERR_DEVICE_TIMEOUT if a kernel abandoned a bounded wait since the last
 * call, else SA_OK. */
sa_status sa_get_device_status(sa_cache* h, sa_stream_t stream);

/* Plan of the next chunk of a stream in state (frames_written, pos_base);
 * pure host computation, needs no device. frames_written must be a multiple
 * of C. */
sa_status sa_plan_chunk(const sa_config* cfg, int64_t frames_written, int64_t pos_base,
                        sa_chunk_plan* plan);

/* Refresh offset Delta for a stream in state (frames_written, pos_base);
 * pure host computation. */
sa_status sa_refresh_delta(const sa_config* cfg, int64_t frames_written, int64_t pos_base,
                           int64_t* delta);

/* Kernel timing with CUDA events recorded around each launch on the launch
 * stream (as external records, so launches captured into a CUDA graph keep
 * their timing: the events then hold the last replay's times).
 * sa_profile_begin clears the counters and starts recording (up to 8192
 * launches); sa_profile_end synchronises and returns the summed device times
 * in milliseconds and the launch counts, then stops recording. Any output
 * pointer may be NULL. */
sa_status sa_profile_begin(sa_cache* h);
sa_status sa_profile_end(sa_cache* h, double* append_ms, int32_t* n_append, double* attend_ms,
                         int32_t* n_attend, double* refresh_ms, int32_t* n_refresh);

/*
 * Allocation-free form of sa_append_attend. The pages have no counterpart:
 * this entry exists for callers that must not call the CUDA allocator at all
 * -- engines and plugin hosts that own every byte of device memory through
 * their own pool and do not let a library allocate, and real-time frame
 * loops that cannot afford cudaMalloc/cudaFree, which may synchronise the
 * whole device and stall the loop past its per-frame deadline. Such callers
 * cannot create a cache handle (sa_cache_create allocates); here they pass
 * the cache memory themselves.
 *   cfg            : as for sa_cache_create.
 *   k_cache, v_cache, k_raw : caller-owned device buffers with the layouts
 *                    sa_cache_create documents ([B][H][(S+R)F][D] and
 *                    [B][H][S*F][D]); zero them before a stream's first
 *                    chunk. k_raw may be NULL when S = 0.
 *   frames_written : host array [B], read and advanced by C per active stream.
 *   pos_base       : host array [B], the streams' RoPE position bases (read).
 *                    There is no allocation-free RoPE refresh: the keys
 *                    already stored keep the positions they were written
 *                    with, so a stream's pos_base must stay the value it had
 *                    at its first chunk (0 for a new stream). Changing it
 *                    between calls shifts new keys against stored ones and
 *                    silently changes every score; streams that need periodic
 *                    refreshes must use a cache handle (sa_rope_refresh).
 *   q, k, v, out, active, stream : as for sa_append_attend.
 * Scratch: a file-scope static device array of 16 MiB (rotated queries
 * B*H*C*F*D elements, the spatial RoPE tables and a status word), present on
 * every GPU that loads the library until the process exits. Configurations
 * that need more return SA_ERR_UNSUPPORTED with the sizes in the error text.
 * The first call on a device looks up the scratch address on that device;
 * make that first call before any stream capture. Every call shares the one
 * scratch array, which keeps the last call's contents: calls whose work
 * overlaps on the GPU (other streams, other host threads) race and must be
 * serialised by the caller. Enqueues work on `stream` and never synchronises;
 * calls no allocator. A bounded-wait expiry is not returned by the call (it
 * happens later, on the GPU): it sets a sticky status word in the scratch,
 * which sa_noalloc_device_status reports and clears.
 */
sa_status sa_append_attend_noalloc(const sa_config* cfg, void* k_cache, void* v_cache,
                                   void* k_raw, int64_t* frames_written, const int64_t* pos_base,
                                   const void* q, const void* k, const void* v, void* out,
                                   const uint8_t* active, sa_stream_t stream);

/* Device status of the allocation-free entry on the current device (no
 * counterpart on the pages; the analogue of sa_get_device_status for callers
 * without a handle). Synchronises `stream`, reads the status word in the
 * static scratch and clears it. Returns SA_ERR_DEVICE_TIMEOUT if a bounded
 * wait of any sa_append_attend_noalloc call on this device gave up since the
 * last read (the outputs and cache rows of those calls are not valid),
 * SA_OK otherwise, SA_ERR_CUDA on a CUDA error. Allocates nothing. */
sa_status sa_noalloc_device_status(sa_stream_t stream);

/*
 * Debug build (libsa_debug.so, compiled with -DSA_DEBUG_BOUNDS; no passage on
 * the pages: robustness of this implementation, the in-kernel stand-in for a
 * memory checker). Every index a kernel computes into a buffer -- cache rows
 * of appended frames, raw-sink rows, ring and sink rows of a refresh, query
 * and key/value tile coordinates, partial-result slots and arrival counters
 * of split attention units, GDN workspace blocks and state slices -- is
 * range-checked before the access. A failed check skips the access (a load
 * reads zero, a tile coordinate is clamped to 0) and sets a bit in a device
 * word of the kernel's source file; no trap, no fault, the kernel ends.
 * sa_debug_bounds_status synchronises `stream`, reads and clears those words
 * on the current device, and returns SA_ERR_DEVICE_BOUNDS (the words in the
 * error text: file and site bits) if any bit was set, SA_OK otherwise. In the
 * normal build (libsa.so) the checks are compiled out and both calls return
 * SA_ERR_UNSUPPORTED. sa_debug_bounds_selftest enqueues one kernel on
 * `stream` that records a failed check at site 31 of the attention file's
 * word without any memory access, so a test can see the recording path work.
 */
sa_status sa_debug_bounds_status(sa_stream_t stream);
sa_status sa_debug_bounds_selftest(sa_stream_t stream);

/* Number of kernels the handle launched since sa_profile_begin (host count). */
sa_status sa_profile_launches(const sa_cache* h, int64_t* launches);

/*
 * Per-head scales of an SA_BF16_E4M3 cache: q_scale, k_scale, v_scale are
 * host arrays of H positive finite floats (NULL = all 1). A rotated query,
 * rotated key or value x of head h is stored as e4m3(x * scale[h]); scores
 * are divided by q_scale[h] * k_scale[h] and outputs by v_scale[h], so the
 * scales choose where in the e4m3 range (2^-9 .. 448) each head's values
 * fall. Call before any stream holds a frame (SA_ERR_STATE otherwise);
 * SA_ERR_INVALID_ARG for another dtype or a non-positive scale. Copies the
 * scales to the device (synchronous on the handle's create stream).
 */
sa_status sa_cache_set_fp8_scales(sa_cache* h, const float* q_scale, const float* k_scale,
                                  const float* v_scale);

/* Copies the handle's per-head scales of an SA_BF16_E4M3 cache to host arrays
 * of H floats each (any may be NULL); SA_ERR_INVALID_ARG for another dtype.
 * Host only. */
sa_status sa_cache_get_fp8_scales(const sa_cache* h, float* q_scale, float* k_scale,
                                  float* v_scale);

/* Sink position modes (sa_cache_set_sink_mode). */
#define SA_SINK_SHIFT 0 /* a refresh rebases the sink with every other position: scores invariant */
#define SA_SINK_REPIN 1 /* after a refresh the sink sits right before the oldest window frame */

/*
 * How the sink's temporal positions follow a RoPE refresh (StreamDiffusionV2,
 * section 2.A.2: RoPE offsets are reset at block boundaries; sink tokens
 * anchor the stream). SA_SINK_SHIFT (the default): sink frame f is at
 * t = f - pos_base, like every other key, so a refresh leaves every score
 * unchanged. SA_SINK_REPIN: sink frame f is at t = f - min(pos_base, S): a
 * refresh (which sets pos_base >= S and puts the oldest visible window frame
 * at t = 0) places the sink immediately before the window, instead of ever
 * farther in the past; scores involving the sink change at each refresh.
 * Takes effect at the next sa_rope_refresh or sa_sink_update (stored keys are
 * not touched by this call). Host only; never fails for a valid handle and
 * mode (SA_ERR_INVALID_ARG otherwise). sa_append_attend_noalloc always shifts.
 */
sa_status sa_cache_set_sink_mode(sa_cache* h, int32_t mode);

/*
 * Adaptive sink update (StreamDiffusionV2, section 2.A.2: sink tokens are
 * updated dynamically from the prompt's semantics and the recent visual
 * context). For every active stream, the sink's raw (unrotated) keys and its
 * values become (1 - alpha) * old + alpha * new, computed in fp32 and rounded
 * to the cache dtype; the stored sink keys are then re-derived from the new
 * raw keys at the sink's current positions (sa_cache_set_sink_mode).
 *   k_new, v_new : device, [B][S*F][H][D] in cfg dtype (the sink frames'
 *                  tokens in frame, row, column order), contiguous, 16-byte
 *                  aligned; rows of inactive streams are not read. Borrowed
 *                  until the stream-ordered work completes.
 *   alpha        : in [0, 1]; 1 replaces the sink, 0 leaves it unchanged.
 *   active       : host, B bytes or NULL for all streams.
 * One kernel on `stream`; never synchronises. Errors: SA_ERR_INVALID_ARG
 * (no sink, NULL or unaligned buffers, alpha outside [0, 1]), SA_ERR_STATE
 * (an active stream's sink frames are not all written yet), SA_ERR_UNSUPPORTED
 * (more than 16 sink frames), SA_ERR_CUDA; nothing is launched on error.
 */
sa_status sa_sink_update(sa_cache* h, const void* k_new, const void* v_new, float alpha,
                         const uint8_t* active, sa_stream_t stream);

/* Check of the bounded device waits that every kernel of the library relies
 * on (no reference passage: robustness of this implementation). Launches one
 * CTA on `stream` whose two warps wait on a shared-memory barrier that
 * nothing completes: warp 0 gives up after limit_ns nanoseconds, raises the
 * CTA's abort flag and records SA_ERR_DEVICE_TIMEOUT in a device status
 * word; warp 1 waits with a 20x longer limit but leaves as soon as it sees
 * the abort flag. Synchronises `stream`, then stores the two warps' waiting
 * times (ns) to waited_ns[0..1] (host array, may be NULL) and returns
 * SA_ERR_DEVICE_TIMEOUT when the wait expired as designed (the CUDA context
 * stays usable), SA_OK if the barrier completed, SA_ERR_INVALID_ARG for
 * limit_ns outside [1e5, 1e10] (0.1 ms .. 10 s), SA_ERR_CUDA on a CUDA
 * error. No fault, trap or unbounded wait is involved. */
sa_status sa_wait_probe(uint64_t limit_ns, int64_t* waited_ns, sa_stream_t stream);

/* Thread-local text of the last error; never NULL. */
/*
 * Gated DeltaNet (GDN) block: the linear-attention half of a hybrid streaming
 * transformer (SANA-Streaming, sections "hybrid diffusion transformer" and
 * "system co-design": most blocks keep a fixed-size recurrent state per head,
 * updated as frames arrive, and cache only that state between chunks; a fused
 * kernel keeps the state on chip). The pages give no recurrence; this call
 * runs the published gated delta rule (Yang, Kautz and Hatamizadeh, "Gated
 * Delta Networks", ICLR 2025) with L2-normalised q and k, token by token in
 * the order given, per stream b and head h:
 *     S <- exp(g_t) S (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale S q_t
 * (k_t, q_t divided by their norms; a zero vector stays zero). S is D x D:
 * row i = value dim, column j = key dim.
 */
typedef struct {
  int32_t batch;     /* B streams, 1..SA_MAX_STREAMS */
  int32_t heads;     /* H, 1..65535 */
  int32_t head_dim;  /* D: 64 or 128 (query, key and value dims) */
  int32_t dtype;     /* SA_F32 or SA_BF16: element type of q, k, v and out */
  int64_t tokens;    /* T tokens of every active stream in this call, >= 0 */
  float scale;       /* output scale, >= 0; 0 means 1/sqrt(D) */
  int32_t pad_;
} sa_gdn_config;

/*
 * Advances the state of every active stream over its next T tokens and
 * writes their outputs. Device pointers, all owned by the caller:
 *   state  [B][H][D][D] fp32, 16-byte aligned, read and written in place (the
 *          block's whole memory between calls; zero it to start a stream);
 *   q, k, v, out [B][T][H][D] in cfg->dtype (out may not alias the inputs;
 *          all four 16-byte aligned);
 *   g      [B][T][H] fp32, log decay of each token (<= 0; exp(g) multiplies S);
 *   beta   [B][T][H] fp32, write strength of each token (in [0, 1] for a
 *          contracting update; other values are computed as given);
 *   workspace  scratch of workspace_bytes >= sa_gdn_workspace_size(cfg),
 *          16-byte aligned; contents need not be kept between calls. Its
 *          first 1 KiB holds the call's device status word
 *          (sa_gdn_device_status). The call runs two kernels: one computes,
 *          for every 64-token block and all blocks in parallel, the normalised
 *          keys and queries, the triangular inverse T of the chunkwise form
 *          and M = scale P T (P the decay-masked q.k matrix) into the
 *          workspace; the other walks the blocks in order and updates the
 *          state. With D = 128 the kernels are chained by programmatic
 *          dependent launches (the pass sets up while its prep finishes), and
 *          a call of at least 8 blocks whose pass leaves half of the SMs idle
 *          runs in two pieces of its blocks (3/8 and 5/8), the second piece's
 *          prep beside the first piece's pass. A later kernel on `stream`
 *          starts after all of them (one that the caller launches as a
 *          programmatic dependent must execute griddepcontrol.wait before it
 *          reads the outputs or the state).
 * Precision. The sequential pass runs its contractions (K S^T, Q S^T, T and
 * M times the right-hand side, the state update), and the first kernel its
 * Gram matrices, on the tensor cores as three-term split products of bf16
 * operands (x = hi + lo, a.b ~ a_hi.b_hi + a_hi.b_lo + a_lo.b_hi, fp32
 * accumulation: about 2^-16 relative per product, within 1e-4 of the fp64
 * recurrence on the outputs and the state), with the state in tensor memory
 * for the whole call; everything else is fp32. D = 64 runs through the same
 * kernels with the key dims padded to 128 with zeros.
 * active: host array of B flags, NULL = all; an inactive stream's state and
 * out rows are untouched. The state is fp32; outputs are rounded once to
 * cfg->dtype. Asynchronous on `stream`, graph-capturable.
 * Errors: SA_ERR_INVALID_ARG (cfg, a NULL pointer with tokens > 0, alignment,
 * a workspace smaller than sa_gdn_workspace_size), SA_ERR_UNSUPPORTED (no
 * compute capability 10.x device, or a size that does not fit), SA_ERR_CUDA
 * (the launch failed).
 */
sa_status sa_gdn_chunk(const sa_gdn_config* cfg, float* state, const void* q, const void* k,
                       const void* v, const float* g, const float* beta, void* out,
                       void* workspace, size_t workspace_bytes, const uint8_t* active,
                       sa_stream_t stream);

/*
 * Bytes of the device workspace sa_gdn_chunk needs for cfg: a 1 KiB header
 * plus, per (stream, head, started 64-token block of the call), 96 KiB for
 * D = 128 (the operand images of the tensor-core pass) or 32 KiB for D = 64,
 * i.e. 1024 + batch * heads * ceil(tokens / 64) * (98304 or 32768).
 * Errors: SA_ERR_INVALID_ARG (cfg invalid or bytes NULL), SA_ERR_UNSUPPORTED.
 */
sa_status sa_gdn_workspace_size(const sa_gdn_config* cfg, size_t* bytes);

/*
 * Device status of the last sa_gdn_chunk call that used `workspace` (no
 * passage on the pages: robustness of this implementation). Synchronises
 * `stream` and reads the status word the call's kernels keep in the
 * workspace header (cleared by each call's first kernel). Returns
 * SA_ERR_DEVICE_TIMEOUT if a bounded wait of the tensor-core pass gave up
 * (the call's outputs and state are not valid), SA_OK otherwise,
 * SA_ERR_INVALID_ARG for a NULL or unaligned workspace, SA_ERR_CUDA.
 */
sa_status sa_gdn_device_status(const void* workspace, sa_stream_t stream);

const char* sa_last_error_string(void);

int32_t sa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_H */
