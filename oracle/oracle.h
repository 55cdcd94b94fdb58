/*
 * oracle.h -- plain, slow, fp64 CPU oracle of per-chunk block-causal attention
 * over a rolling (sink + sliding window) KV cache with 3D RoPE and refresh,
 * and of the gated delta rule of the hybrid model's GDN blocks (orc_gdn_chunk).
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code with
 * the CUDA path: the only common dependency is the seeded input generator
 * (inputgen/sa_inputgen.h), which holds none of the method's arithmetic.
 *
 * Sources of the definition:
 *  - StreamDiffusionV2 (technical summary, section 2.A.2 "adaptive sink tokens
 *    and RoPE refresh"): sink tokens anchor the stream; RoPE offsets are reset
 *    at block boundaries so positions do not drift over long horizons.
 *  - SANA-Streaming (section "hybrid diffusion transformer"): softmax blocks
 *    attend to a sliding local window plus a persistent sink chunk, i.e. a
 *    bounded context with constant memory.
 *  - StreamDiT (abstract): window attention over a moving buffer of frames.
 *  - SANA-Streaming (sections "hybrid diffusion transformer", "system
 *    co-design"): the GDN blocks' recurrent state (see orc_gdn_chunk).
 * The pages print no formula; the numeric definition below (ring geometry,
 * 3D RoPE bands, rebase offset, dtype rounding) is the reading stated beside
 * each function.
 *
 * Notation: H heads, D head dim, F = fh*fw tokens per frame, C frames per
 * chunk, S sink frames, W window frames, R = W + C ring frames. Frames are
 * numbered per stream from 0; chunk c holds frames [cC, (c+1)C); token order
 * within a chunk is frame, then row y, then column x. Input blocks are
 * [tok][head][d] (see sa_inputgen.h).
 */
#ifndef SA_ORACLE_H
#define SA_ORACLE_H

#include <stdint.h>
#include "../inputgen/sa_inputgen.h"

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_EXACT = 0, ORC_STORE_F32 = 1, ORC_STORE_BF16 = 2, ORC_STORE_E4M3 = 3 };

typedef struct {
  int32_t H, D, fh, fw;
  int32_t C, S, W;
  int32_t rope_dims[3];   /* (d_t, d_h, d_w), even, sum D */
  double rope_base;       /* theta base, e.g. 10000 */
  double scale;           /* softmax scale; 0 means 1/sqrt(D) */
  int64_t refresh_period; /* refresh before chunk c when c>0 and c % period == 0; 0 = never */
  int32_t store;          /* ORC_EXACT, ORC_STORE_F32 or ORC_STORE_BF16 */
  int32_t in_dtype;       /* IG_F32 or IG_BF16: how the generated inputs are stored */
  int32_t sink_repin;     /* 0: the sink's positions rebase with the rest (shift);
                             1: after a refresh the sink sits right before the
                             oldest window frame (t = f - S) */
  int32_t pad_;
  int64_t sink_update_period; /* sink update before chunk u when u > 0, u % period == 0
                                 and the sink is complete (uC >= S); 0 = never */
  double sink_alpha;      /* weight of the new sink data in the update (1 = replace) */
  const double* fp8_scale; /* ORC_STORE_E4M3: [3][H] per-head scales of q, k, v; a value x
                              is stored as round_e4m3(x * s) / s; NULL = all 1 */
} orc_cfg;

double orc_round_store(int32_t store, double x);
double orc_theta(const orc_cfg* cfg, int32_t band, int32_t j);
void orc_rope_vec(const orc_cfg* cfg, const double* x, double t, double y, double w,
                  double* out);
void orc_rope_tband(const orc_cfg* cfg, const double* x, double t, double* out);

int32_t orc_refresh_due(const orc_cfg* cfg, int64_t c);
int64_t orc_refresh_delta(const orc_cfg* cfg, int64_t c, int64_t base);
int64_t orc_base_at(const orc_cfg* cfg, int64_t c);

int32_t orc_visible(const orc_cfg* cfg, int64_t c, int64_t f);
int64_t orc_frame_slot(const orc_cfg* cfg, int64_t f);
void orc_slot_frames(const orc_cfg* cfg, int64_t c, int64_t* slot_frame);
int64_t orc_n_keys(const orc_cfg* cfg, int64_t c);

int32_t orc_input_block(const orc_cfg* cfg, const ig_spec* sp, int64_t stream, int64_t chunk,
                        int32_t tensor, double* out);
double orc_sink_pos(const orc_cfg* cfg, int64_t f, int64_t c);
int32_t orc_sink_raw(const orc_cfg* cfg, const ig_spec* sp, int64_t stream, int64_t f,
                     int64_t c, int32_t tensor, double* out);
int32_t orc_stored_key_frame(const orc_cfg* cfg, const ig_spec* sp, int64_t stream,
                             int64_t f, int64_t c, double* out);
int32_t orc_query_rot(const orc_cfg* cfg, const ig_spec* sp, int64_t stream, int64_t c,
                      double* out);
int32_t orc_cache_contents(const orc_cfg* cfg, const ig_spec* sp, int64_t stream, int64_t c,
                           double* k_out, double* v_out, int64_t* slot_frame);
int32_t orc_attend_rows(const orc_cfg* cfg, const ig_spec* sp, int64_t stream, int64_t c,
                        int32_t n_rows, const int32_t* toks, const int32_t* heads,
                        double* out);
int32_t orc_attend_rows_uncommitted(const orc_cfg* cfg, const ig_spec* sp_cache,
                                    const ig_spec* sp_chunk, int64_t stream, int64_t c,
                                    int32_t n_rows, const int32_t* toks, const int32_t* heads,
                                    double* out);
int32_t orc_bruteforce_rows(const orc_cfg* cfg, const ig_spec* sp, int64_t stream,
                            int64_t c, int32_t n_rows, const int32_t* toks,
                            const int32_t* heads, double* out);
/* Gated DeltaNet block, one call over T tokens of one stream, all heads (see
 * oracle.c): state [H][D][D] (row i = value dim, column j = key dim) is read
 * and updated in place; q, k, v, out [T][H][D]; g (log decay) and beta
 * [T][H]. Returns 0, or -1 on a bad argument. */
int32_t orc_gdn_chunk(int32_t H, int32_t D, int64_t T, double scale, double* state,
                      const double* q, const double* k, const double* v, const double* g,
                      const double* beta, double* out);
int32_t orc_num_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_ORACLE_H */
