/*
 * oracle.c -- fp64 CPU oracle (see oracle.h). TEST INFRASTRUCTURE ONLY.
 *
 * Plain loops in fp64. OpenMP only splits independent output rows / tokens
 * across threads; it never changes the order of any sum.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int32_t orc_num_threads(void) {
#ifdef _OPENMP
  return (int32_t)omp_get_max_threads();
#else
  return 1;
#endif
}

static int64_t frame_tokens(const orc_cfg* g) { return (int64_t)g->fh * g->fw; }
static int64_t ring_frames(const orc_cfg* g) { return (int64_t)g->W + g->C; }
static double softmax_scale(const orc_cfg* g) {
  return g->scale > 0.0 ? g->scale : 1.0 / sqrt((double)g->D);
}

/* ---------------------------------------------------------------------------
 * Storage rounding. The method keeps rotated queries and keys in the cache's
 * element type, so the storage-faithful mode rounds each stored value once,
 * to nearest, ties to even. bf16 keeps 8 significant bits.
 * ------------------------------------------------------------------------- */
static double round_to_bits(double x, int bits) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  double m = frexp(x, &e);            /* x = m * 2^e, 0.5 <= |m| < 1 */
  double scaled = ldexp(m, bits);     /* |scaled| in [2^(bits-1), 2^bits) */
  double r = nearbyint(scaled);       /* default rounding mode: to nearest even */
  return ldexp(r, e - bits);
}

/* e4m3 (OCP FP8 E4M3, no infinities): 1 sign, 4 exponent bits (bias 7), 3
 * mantissa bits; normal numbers 2^-6 .. 448, subnormals in steps of 2^-9.
 * Round to nearest, ties to even, on that grid; magnitudes beyond 448
 * saturate to 448 (a conversion with saturation to the largest finite). */
static double round_e4m3(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  const double a = fabs(x);
  int e;
  frexp(a, &e);                       /* a in [2^(e-1), 2^e) */
  int k = e - 1;
  if (k < -6) k = -6;                 /* subnormal range keeps the 2^-9 step */
  const double q = ldexp(1.0, k - 3); /* grid step: 3 mantissa bits */
  double r = nearbyint(a / q) * q;
  if (r > 448.0) r = 448.0;
  return copysign(r, x);
}

double orc_round_store(int32_t store, double x) {
  if (store == ORC_STORE_F32) return (double)(float)x;
  if (store == ORC_STORE_BF16) return round_to_bits(x, 8);
  if (store == ORC_STORE_E4M3) return round_e4m3(x);
  return x;
}

/* Stored value of a rotated query (which = 0), rotated key (1) or value (2)
 * of head h: the storage rounding, with the head's scale in e4m3 mode. */
static double round_head(const orc_cfg* g, int which, int h, double x) {
  if (g->store != ORC_STORE_E4M3) return orc_round_store(g->store, x);
  const double s = g->fp8_scale ? g->fp8_scale[which * g->H + h] : 1.0;
  return round_e4m3(x * s) / s;
}

/* Precision of the raw (unrotated) sink keys: the cache type, except in
 * e4m3 mode where the raw sink keeps the bf16 input precision. */
static int32_t raw_store(const orc_cfg* g) {
  return g->store == ORC_STORE_E4M3 ? ORC_STORE_BF16 : g->store;
}

/* ---------------------------------------------------------------------------
 * 3D rotary embedding. The head dimension is split into three bands
 * (t | h | w) of widths rope_dims. Inside a band of width d, the pair of
 * adjacent dims (2j, 2j+1) is rotated by the angle pos * theta_j with
 * theta_j = base^(-2j/d), pos being the frame's temporal position t, the
 * token's row y or its column x. Rotation sense: (a, b) -> (a cos - b sin,
 * a sin + b cos), i.e. multiplication of a + ib by e^{i phi}.
 * ------------------------------------------------------------------------- */
double orc_theta(const orc_cfg* g, int32_t band, int32_t j) {
  const double d = (double)g->rope_dims[band];
  return pow(g->rope_base, -2.0 * (double)j / d);
}

static void rotate_band(const orc_cfg* g, int band, int off, double pos, const double* x,
                        double* out) {
  const int d = g->rope_dims[band];
  for (int j = 0; j < d / 2; ++j) {
    const double phi = pos * orc_theta(g, band, j);
    const double c = cos(phi), s = sin(phi);
    const double a = x[off + 2 * j], b = x[off + 2 * j + 1];
    out[off + 2 * j] = a * c - b * s;
    out[off + 2 * j + 1] = a * s + b * c;
  }
}

void orc_rope_vec(const orc_cfg* g, const double* x, double t, double y, double w,
                  double* out) {
  const double pos[3] = {t, y, w};
  int off = 0;
  for (int band = 0; band < 3; ++band) {
    rotate_band(g, band, off, pos[band], x, out);
    off += g->rope_dims[band];
  }
}

/* Rotates only the temporal band by t; the spatial bands are copied. */
void orc_rope_tband(const orc_cfg* g, const double* x, double t, double* out) {
  for (int d = 0; d < g->D; ++d) out[d] = x[d];
  rotate_band(g, 0, 0, t, x, out);
}

/* ---------------------------------------------------------------------------
 * RoPE refresh (StreamDiffusionV2 2.A.2: offsets reset at block boundaries).
 * Reading: a refresh runs before chunk c when c > 0 and c % period == 0. It
 * rebases every cached position of the stream by the same Delta, so relative
 * offsets (and, in exact arithmetic, all scores) are unchanged. Delta makes
 * the oldest non-sink frame chunk c will see start at t = 0:
 *   Delta = max(S, cC - W) - base.
 * A frame f then has temporal position t = f - base.
 * ------------------------------------------------------------------------- */
int32_t orc_refresh_due(const orc_cfg* g, int64_t c) {
  return g->refresh_period > 0 && c > 0 && (c % g->refresh_period) == 0;
}

int64_t orc_refresh_delta(const orc_cfg* g, int64_t c, int64_t base) {
  int64_t first = c * g->C - g->W;
  if (first < g->S) first = g->S;
  return first - base;
}

/* Base in effect while chunk c is processed (after a refresh due at c). */
int64_t orc_base_at(const orc_cfg* g, int64_t c) {
  int64_t base = 0;
  if (g->refresh_period <= 0) return 0;
  for (int64_t r = g->refresh_period; r <= c; r += g->refresh_period)
    base += orc_refresh_delta(g, r, base);
  return base;
}

/* ---------------------------------------------------------------------------
 * Visibility (SANA-Streaming: sliding local window + persistent sink chunk;
 * current chunk bidirectional). Queries of chunk c see frame f iff
 *   0 <= f < (c+1)C  and  (f < S  or  f >= cC - W).
 * ------------------------------------------------------------------------- */
int32_t orc_visible(const orc_cfg* g, int64_t c, int64_t f) {
  if (f < 0 || f >= (c + 1) * g->C) return 0;
  return f < g->S || f >= c * g->C - g->W;
}

/* Cache slot of frame f: sink frames keep slot f forever; later frames go to
 * the ring of R = W + C frames at slot S + (f - S) mod R, overwriting the
 * frame written R frames earlier. */
int64_t orc_frame_slot(const orc_cfg* g, int64_t f) {
  if (f < g->S) return f;
  return g->S + (f - g->S) % ring_frames(g);
}

/* Frame held by each of the S + R slots after chunk c is appended (-1 = never
 * written), in closed form: the newest frame f < (c+1)C mapped to the slot. */
void orc_slot_frames(const orc_cfg* g, int64_t c, int64_t* slot_frame) {
  const int64_t R = ring_frames(g);
  const int64_t written = (c + 1) * g->C;
  for (int64_t s = 0; s < g->S; ++s) slot_frame[s] = s < written ? s : -1;
  const int64_t n = written - g->S; /* non-sink frames written */
  for (int64_t r = 0; r < R; ++r) {
    int64_t f = -1;
    if (n > r) {
      const int64_t last = n - 1;
      const int64_t i = last - ((last - r) % R);
      f = g->S + i;
    }
    slot_frame[g->S + r] = f;
  }
}

/* Number of visible key tokens for chunk c. */
int64_t orc_n_keys(const orc_cfg* g, int64_t c) {
  int64_t n = 0;
  for (int64_t f = 0; f < (c + 1) * g->C; ++f) n += orc_visible(g, c, f);
  return n * frame_tokens(g);
}

/* ---------------------------------------------------------------------------
 * Inputs. Tokens [tok0, tok0+ntok) of tensor `tensor` of chunk `chunk`, as the
 * stored input values (generator value rounded to the input dtype).
 * ------------------------------------------------------------------------- */
static void gen_tokens(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t chunk,
                       int32_t tensor, int64_t tok0, int64_t ntok, double* out) {
  const uint64_t key = ig_key(sp->seed, stream, chunk, tensor);
  const uint64_t okey = ig_key(sp->seed, stream, chunk, IG_OUTLIER);
  const uint64_t thr = tensor == IG_K ? ig_outlier_threshold(sp->outlier_frac) : 0;
  const int64_t n = ntok * (int64_t)g->H * g->D;
  const uint64_t base = (uint64_t)tok0 * (uint64_t)g->H * (uint64_t)g->D;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    float x = ig_value_keyed(sp->dist[tensor], key, okey, thr, tensor == IG_K,
                             base + (uint64_t)i, g->D, sp->outlier_scale);
    if (g->in_dtype == IG_BF16) x = ig_bf16_to_f32(ig_f32_to_bf16_rne(x));
    out[i] = (double)x;
  }
}

int32_t orc_input_block(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t chunk,
                        int32_t tensor, double* out) {
  if (!g || !sp || !out || tensor < 0 || tensor > 2) return -1;
  gen_tokens(g, sp, stream, chunk, tensor, 0, (int64_t)g->C * frame_tokens(g), out);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Sink (StreamDiffusionV2, technical summary, section 2.A.2: sink tokens are
 * updated adaptively; RoPE offsets are reset at block boundaries).
 * Temporal position of sink frame f while chunk c is processed:
 *   shift : f - base(c)  (the sink moves with every rebase; scores invariant)
 *   repin : f - min(base(c), S)  -- before the first refresh base(c) = 0 and
 *           the sink is at its own frame index; a refresh sets base >= S and
 *           the sink then sits immediately before the oldest window frame,
 *           which the refresh puts at t = 0.
 * ------------------------------------------------------------------------- */
double orc_sink_pos(const orc_cfg* g, int64_t f, int64_t c) {
  int64_t base = orc_base_at(g, c);
  if (g->sink_repin && base > g->S) base = g->S;
  return (double)(f - base);
}

static int sink_update_due(const orc_cfg* g, int64_t u) {
  return g->sink_update_period > 0 && u > 0 && u % g->sink_update_period == 0 &&
         u * g->C >= g->S;
}

/* Raw (unrotated) key (IG_K) or value (IG_V) of sink frame f, [F][H][D], as
 * held while chunk c is processed: the frame's input, then for every update
 * before a chunk u in (0, c] in order
 *   raw <- round((1 - alpha) * raw + alpha * new),
 * new = frame f's rows of the update block drawn at chunk coordinate
 * IG_SINK_UPDATE_CHUNK0 + u (rounding to the storage type; none when exact). */
int32_t orc_sink_raw(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t f,
                     int64_t c, int32_t tensor, double* out) {
  if (!g || !sp || !out || f < 0 || f >= g->S || (tensor != IG_K && tensor != IG_V)) return -1;
  const int64_t F = frame_tokens(g), n = F * (int64_t)g->H * g->D;
  gen_tokens(g, sp, stream, f / g->C, tensor, (f % g->C) * F, F, out);
  /* values are kept as stored (e4m3 mode: the cache's own rounding, per
   * head); raw keys at raw_store precision */
  const int v_stored = tensor == IG_V && g->store == ORC_STORE_E4M3;
#define SINK_ROUND(i, x) \
  (v_stored ? round_head(g, 2, (int)(((i) / g->D) % g->H), (x)) : orc_round_store(raw_store(g), (x)))
  for (int64_t i = 0; i < n; ++i) out[i] = SINK_ROUND(i, out[i]);
  if (g->sink_update_period <= 0) return 0;
  double* nw = (double*)malloc(sizeof(double) * (size_t)n);
  if (!nw) return -2;
  const double a = g->sink_alpha;
  for (int64_t u = g->sink_update_period; u <= c; u += g->sink_update_period) {
    if (!sink_update_due(g, u)) continue;
    gen_tokens(g, sp, stream, IG_SINK_UPDATE_CHUNK0 + u, tensor, f * F, F, nw);
    for (int64_t i = 0; i < n; ++i) out[i] = SINK_ROUND(i, (1.0 - a) * out[i] + a * nw[i]);
  }
#undef SINK_ROUND
  free(nw);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Stored key of frame f ([F][H][D]) as the cache holds it while chunk c is
 * processed (f must be visible at c).
 *  exact mode : R(f - base(c), y, x) k, no rounding.
 *  storage    : a sink frame is re-derived from its raw key at every refresh,
 *               so it is round(R(f - base(c), y, x) k). A ring frame is
 *               rotated once when written (chunk cw = f / C, base(cw)) and
 *               rounded; each refresh r in (cw, c] then re-rotates its
 *               temporal band by -Delta_r and rounds again.
 * ------------------------------------------------------------------------- */
int32_t orc_stored_key_frame(const orc_cfg* g, const ig_spec* sp, int64_t stream,
                             int64_t f, int64_t c, double* out) {
  if (!g || !sp || !out || f < 0) return -1;
  const int64_t F = frame_tokens(g);
  const int H = g->H, D = g->D;
  const int64_t cw = f / g->C;
  double* raw = (double*)malloc(sizeof(double) * (size_t)(F * H * D));
  if (!raw) return -2;
  const int exact = g->store == ORC_EXACT;
  const int is_sink = f < g->S;
  if (is_sink) {
    if (orc_sink_raw(g, sp, stream, f, c, IG_K, raw) != 0) { free(raw); return -2; }
  } else {
    gen_tokens(g, sp, stream, cw, IG_K, (f % g->C) * F, F, raw);
  }
  const double pos = is_sink ? orc_sink_pos(g, f, c)
                             : (double)(f - (exact ? orc_base_at(g, c) : orc_base_at(g, cw)));
  /* refreshes that re-rotate this stored ring key: r in (cw, c] */
  int64_t deltas[4096];
  int n_ref = 0;
  if (!exact && !is_sink && g->refresh_period > 0) {
    for (int64_t r = (cw / g->refresh_period + 1) * g->refresh_period; r <= c && n_ref < 4096;
         r += g->refresh_period)
      deltas[n_ref++] = orc_refresh_delta(g, r, orc_base_at(g, r - 1));
  }

#pragma omp parallel for schedule(static)
  for (int64_t th = 0; th < F * H; ++th) {
    const int64_t j = th / H;
    const double y = (double)(j / g->fw), x = (double)(j % g->fw);
    const double* kin = raw + th * D;
    double* ko = out + th * D;
    double tmp[512];
    const int h = (int)(th % H);
    orc_rope_vec(g, kin, pos, y, x, tmp);
    for (int d = 0; d < D; ++d) ko[d] = round_head(g, 1, h, tmp[d]);
    for (int i = 0; i < n_ref; ++i) {
      orc_rope_tband(g, ko, -(double)deltas[i], tmp);
      for (int d = 0; d < D; ++d) ko[d] = round_head(g, 1, h, tmp[d]);
    }
  }
  free(raw);
  return 0;
}

/* Rotated queries of chunk c ([Lc][H][D]): round(R(f - base(c), y, x) q). */
int32_t orc_query_rot(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t c,
                      double* out) {
  if (!g || !sp || !out) return -1;
  const int64_t F = frame_tokens(g), Lc = (int64_t)g->C * F;
  const int H = g->H, D = g->D;
  double* raw = (double*)malloc(sizeof(double) * (size_t)(Lc * H * D));
  if (!raw) return -2;
  gen_tokens(g, sp, stream, c, IG_Q, 0, Lc, raw);
  const int64_t base = orc_base_at(g, c);
#pragma omp parallel for schedule(static)
  for (int64_t th = 0; th < Lc * H; ++th) {
    const int64_t tok = th / H;
    const int64_t f = c * g->C + tok / F;
    const int64_t j = tok % F;
    double tmp[512];
    orc_rope_vec(g, raw + th * D, (double)(f - base), (double)(j / g->fw),
                 (double)(j % g->fw), tmp);
    for (int d = 0; d < D; ++d) out[th * D + d] = round_head(g, 0, (int)(th % H), tmp[d]);
  }
  free(raw);
  return 0;
}

/* Cache contents after chunk c's append: K' and V per slot, [H][(S+R)F][D]. */
int32_t orc_cache_contents(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t c,
                           double* k_out, double* v_out, int64_t* slot_frame) {
  if (!g || !sp || !k_out || !v_out || !slot_frame) return -1;
  const int64_t F = frame_tokens(g), nslot = g->S + ring_frames(g);
  const int H = g->H, D = g->D;
  const int64_t rows = nslot * F;
  memset(k_out, 0, sizeof(double) * (size_t)(H * rows * D));
  memset(v_out, 0, sizeof(double) * (size_t)(H * rows * D));
  orc_slot_frames(g, c, slot_frame);
  double* kf = (double*)malloc(sizeof(double) * (size_t)(F * H * D));
  double* vf = (double*)malloc(sizeof(double) * (size_t)(F * H * D));
  if (!kf || !vf) { free(kf); free(vf); return -2; }
  for (int64_t s = 0; s < nslot; ++s) {
    const int64_t f = slot_frame[s];
    if (f < 0) continue;
    orc_stored_key_frame(g, sp, stream, f, c, kf);
    if (f < g->S) {
      orc_sink_raw(g, sp, stream, f, c, IG_V, vf);
    } else {
      gen_tokens(g, sp, stream, f / g->C, IG_V, (f % g->C) * F, F, vf);
      if (g->store == ORC_STORE_E4M3)
        for (int64_t i = 0; i < F * H * D; ++i) vf[i] = round_head(g, 2, (int)((i / D) % H), vf[i]);
    }
    for (int64_t j = 0; j < F; ++j)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          const int64_t dst = ((int64_t)h * rows + s * F + j) * D + d;
          k_out[dst] = kf[(j * H + h) * D + d];
          v_out[dst] = vf[(j * H + h) * D + d];
        }
  }
  free(kf);
  free(vf);
  return 0;
}

/* Softmax attention of one query row over n keys (row-major [n][D] with a
 * key stride), fp64, max-subtracted, two passes. */
static void attend_one(const double* q, const double* keys, const double* vals, int64_t n,
                       int64_t stride, int D, double scale, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += q[d] * keys[j * stride + d];
    s[j] = acc * scale;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    const double p = exp(s[j] - m);
    l += p;
    for (int d = 0; d < D; ++d) out[d] += p * vals[j * stride + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
  free(s);
}

/* ---------------------------------------------------------------------------
 * Cache-path attention: output rows (tok, head) of chunk c. Keys and values
 * are the visible frames as stored in the cache (sink, then window, then the
 * current chunk); queries are rotated with the same base.
 * ------------------------------------------------------------------------- */
/* Rows of the cache-path attention of chunk c. Frames before the chunk are
 * stored keys / values drawn from sp_past; the chunk's own frames (keys,
 * values) and its queries are drawn from sp_chunk. With sp_past == sp_chunk
 * this is the committed path; otherwise the chunk is attended with inputs
 * that the cache never keeps. */
static int32_t attend_rows_two(const orc_cfg* g, const ig_spec* sp_past, const ig_spec* sp_chunk,
                               int64_t stream, int64_t c, int32_t n_rows, const int32_t* toks,
                               const int32_t* heads, double* out) {
  if (!g || !sp_past || !sp_chunk || !out || n_rows < 0 || (n_rows > 0 && (!toks || !heads)))
    return -1;
  const int64_t F = frame_tokens(g), Lc = (int64_t)g->C * F;
  const int H = g->H, D = g->D;
  if (D > 512) return -1;
  for (int32_t r = 0; r < n_rows; ++r)
    if (toks[r] < 0 || toks[r] >= Lc || heads[r] < 0 || heads[r] >= H) return -1;

  int64_t nvis = 0;
  for (int64_t f = 0; f < (c + 1) * g->C; ++f) nvis += orc_visible(g, c, f);
  const int64_t nk = nvis * F;
  /* keys/values laid out [head][key][D] */
  double* K = (double*)malloc(sizeof(double) * (size_t)(H * nk * D));
  double* V = (double*)malloc(sizeof(double) * (size_t)(H * nk * D));
  double* kf = (double*)malloc(sizeof(double) * (size_t)(F * H * D));
  double* vf = (double*)malloc(sizeof(double) * (size_t)(F * H * D));
  double* qr = (double*)malloc(sizeof(double) * (size_t)(Lc * H * D));
  if (!K || !V || !kf || !vf || !qr) {
    free(K); free(V); free(kf); free(vf); free(qr);
    return -2;
  }
  int64_t kpos = 0;
  for (int64_t f = 0; f < (c + 1) * g->C; ++f) {
    if (!orc_visible(g, c, f)) continue;
    const ig_spec* sp = f < c * g->C ? sp_past : sp_chunk;
    orc_stored_key_frame(g, sp, stream, f, c, kf);
    if (f < g->S) {
      orc_sink_raw(g, sp, stream, f, c, IG_V, vf);
    } else {
      gen_tokens(g, sp, stream, f / g->C, IG_V, (f % g->C) * F, F, vf);
      if (g->store == ORC_STORE_E4M3)
        for (int64_t i = 0; i < F * H * D; ++i) vf[i] = round_head(g, 2, (int)((i / D) % H), vf[i]);
    }
    for (int64_t j = 0; j < F; ++j)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          K[((int64_t)h * nk + kpos + j) * D + d] = kf[(j * H + h) * D + d];
          V[((int64_t)h * nk + kpos + j) * D + d] = vf[(j * H + h) * D + d];
        }
    kpos += F;
  }
  orc_query_rot(g, sp_chunk, stream, c, qr);
  const double scale = softmax_scale(g);
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t r = 0; r < n_rows; ++r) {
    const int h = heads[r];
    attend_one(qr + ((int64_t)toks[r] * H + h) * D, K + (int64_t)h * nk * D,
               V + (int64_t)h * nk * D, nk, D, D, scale, out + (int64_t)r * D);
  }
  free(K); free(V); free(kf); free(vf); free(qr);
  return 0;
}

int32_t orc_attend_rows(const orc_cfg* g, const ig_spec* sp, int64_t stream, int64_t c,
                        int32_t n_rows, const int32_t* toks, const int32_t* heads,
                        double* out) {
  return attend_rows_two(g, sp, sp, stream, c, n_rows, toks, heads, out);
}

/* Attention of chunk c over the committed context (frames before the chunk,
 * drawn from sp_cache) and an uncommitted chunk (queries, keys and values of
 * the chunk's frames drawn from sp_chunk). StreamDiffusionV2 (technical
 * summary, section 2.B.2 "Stream-Batch"): every denoising step of a chunk is
 * a forward pass over the same cached context with that step's latents;
 * only the final step's keys and values are kept. */
int32_t orc_attend_rows_uncommitted(const orc_cfg* g, const ig_spec* sp_cache,
                                    const ig_spec* sp_chunk, int64_t stream, int64_t c,
                                    int32_t n_rows, const int32_t* toks, const int32_t* heads,
                                    double* out) {
  return attend_rows_two(g, sp_cache, sp_chunk, stream, c, n_rows, toks, heads, out);
}

/* ---------------------------------------------------------------------------
 * Brute-force definition for tiny inputs: exact fp64, absolute positions
 * (t = f, never rebased), every frame 0..(c+1)C-1 as a key, and the explicit
 * sink + window + block-causal mask M(fq, fk) applied as -inf scores.
 * ------------------------------------------------------------------------- */
int32_t orc_bruteforce_rows(const orc_cfg* g, const ig_spec* sp, int64_t stream,
                            int64_t c, int32_t n_rows, const int32_t* toks,
                            const int32_t* heads, double* out) {
  if (!g || !sp || !out || n_rows < 0 || (n_rows > 0 && (!toks || !heads))) return -1;
  const int64_t F = frame_tokens(g), Lc = (int64_t)g->C * F;
  const int H = g->H, D = g->D;
  if (D > 512) return -1;
  const int64_t nf = (c + 1) * g->C;
  const int64_t nk = nf * F;
  double* Kr = (double*)malloc(sizeof(double) * (size_t)(nk * H * D)); /* [key][h][d] */
  double* Vr = (double*)malloc(sizeof(double) * (size_t)(nk * H * D));
  double* Qr = (double*)malloc(sizeof(double) * (size_t)(Lc * H * D));
  if (!Kr || !Vr || !Qr) { free(Kr); free(Vr); free(Qr); return -2; }
  for (int64_t ch = 0; ch <= c; ++ch) {
    gen_tokens(g, sp, stream, ch, IG_K, 0, Lc, Kr + ch * Lc * H * D);
    gen_tokens(g, sp, stream, ch, IG_V, 0, Lc, Vr + ch * Lc * H * D);
  }
  gen_tokens(g, sp, stream, c, IG_Q, 0, Lc, Qr);
  const double scale = softmax_scale(g);
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t r = 0; r < n_rows; ++r) {
    const int h = heads[r];
    const int64_t tq = toks[r];
    const int64_t fq = c * g->C + tq / F;
    const int64_t cq = fq / g->C;
    double q[512], k[512];
    orc_rope_vec(g, Qr + (tq * H + h) * D, (double)fq, (double)((tq % F) / g->fw),
                 (double)((tq % F) % g->fw), q);
    double* s = (double*)malloc(sizeof(double) * (size_t)nk);
    double m = -INFINITY;
    for (int64_t key = 0; key < nk; ++key) {
      const int64_t fk = key / F;
      const int allowed = fk < (cq + 1) * g->C && (fk < g->S || fk >= cq * g->C - g->W);
      if (!allowed) { s[key] = -INFINITY; continue; }
      orc_rope_vec(g, Kr + (key * H + h) * D, (double)fk, (double)((key % F) / g->fw),
                   (double)((key % F) % g->fw), k);
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += q[d] * k[d];
      s[key] = acc * scale;
      if (s[key] > m) m = s[key];
    }
    double l = 0.0;
    double* o = out + (int64_t)r * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t key = 0; key < nk; ++key) {
      const double p = exp(s[key] - m); /* exp(-inf) = 0 for masked keys */
      l += p;
      for (int d = 0; d < D; ++d) o[d] += p * Vr[(key * H + h) * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    free(s);
  }
  free(Kr); free(Vr); free(Qr);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Gated DeltaNet (GDN) block. SANA-Streaming, section "hybrid diffusion
 * transformer": most blocks of that model use GDN linear attention, which
 * folds the stream's history into a recurrent state of fixed size, updated
 * as frames arrive; a GDN block keeps only its latest state between chunks.
 * Section "system co-design": a fused kernel keeps that state on chip.
 *
 * The pages give neither the recurrence nor its gating or normalisation.
 * Reading: the published gated delta rule (Yang, Kautz and Hatamizadeh,
 * "Gated Delta Networks: Improving Mamba2 with Delta Rule", ICLR 2025) with
 * its L2-normalised queries and keys, taken token by token in stream order
 * (frame, row, column), per head:
 *   k^ = k/|k|,  q^ = q/|q|                (a zero vector stays zero)
 *   S  <- exp(g_t) S                        decay, g_t <= 0
 *   S  <- S + beta_t (v_t - S k^_t) k^_t^T  delta-rule write
 *   o_t = scale * S q^_t
 * S has D rows (value dims) and D columns (key dims). Row i of S only ever
 * meets v_t[i], so rows evolve independently.
 * ------------------------------------------------------------------------- */
static void l2_normalised(const double* x, int32_t D, double* out) {
  double s = 0.0;
  for (int32_t d = 0; d < D; ++d) s += x[d] * x[d];
  const double inv = s > 0.0 ? 1.0 / sqrt(s) : 0.0;
  for (int32_t d = 0; d < D; ++d) out[d] = x[d] * inv;
}

int32_t orc_gdn_chunk(int32_t H, int32_t D, int64_t T, double scale, double* state,
                      const double* q, const double* k, const double* v, const double* g,
                      const double* beta, double* out) {
  if (H <= 0 || D <= 0 || T < 0 || !state) return -1;
  if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return -1;
  int32_t err = 0;
#pragma omp parallel for schedule(dynamic)
  for (int32_t h = 0; h < H; ++h) {
    double* S = state + (size_t)h * D * D;
    double* kh = (double*)malloc(sizeof(double) * (size_t)D * 2);
    if (!kh) {
#pragma omp atomic write
      err = -1;
      continue;
    }
    double* qh = kh + D;
    for (int64_t t = 0; t < T; ++t) {
      const size_t row = ((size_t)t * H + h) * D;
      const size_t gi = (size_t)t * H + h;
      l2_normalised(k + row, D, kh);
      l2_normalised(q + row, D, qh);
      const double alpha = exp(g[gi]);
      for (size_t e = 0; e < (size_t)D * D; ++e) S[e] *= alpha;
      for (int32_t i = 0; i < D; ++i) {
        double* Si = S + (size_t)i * D;
        double pred = 0.0;
        for (int32_t j = 0; j < D; ++j) pred += Si[j] * kh[j];
        const double u = beta[gi] * (v[row + i] - pred);
        for (int32_t j = 0; j < D; ++j) Si[j] += u * kh[j];
      }
      for (int32_t i = 0; i < D; ++i) {
        const double* Si = S + (size_t)i * D;
        double o = 0.0;
        for (int32_t j = 0; j < D; ++j) o += Si[j] * qh[j];
        out[row + i] = scale * o;
      }
    }
    free(kh);
  }
  return err;
}
