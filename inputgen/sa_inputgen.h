/*
 * sa_inputgen.h -- seeded, counter-based synthetic inputs for the rolling
 * KV-cache attention workloads.
 *
 * This module is shared by the fp64 CPU oracle (host side) and by the GPU
 * test/bench harness (device side). It holds NO arithmetic of the attention
 * method itself: it only turns (seed, stream, chunk, tensor, element index)
 * into a number, identically on the host and on the device, so that the
 * oracle can regenerate any chunk of any stream without copying data back
 * from the GPU.
 *
 * Generator: the splitmix64 output function (G. Steele, D. Lea, C. Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014) applied to a
 * counter. Every value is a pure function of its coordinates.
 *
 * Distributions (all exact in fp32, so host and device agree bit for bit):
 *   IG_NORMAL  : Irwin-Hall sum of 12 uniform 16-bit integers, centred and
 *                scaled to unit variance -- the classical "sum of twelve
 *                uniforms" approximation of N(0,1); support [-6, 6].
 *   IG_UNIFORM : U(-1,1) on the 2^23-point midpoint grid (2i+1)/2^23 - 1.
 *   IG_ZERO, IG_ONES : the constants 0 and 1 (degenerate test inputs).
 * Gate inputs of the Gated DeltaNet block (one value per token and head):
 *   IG_GATE    : log decay g = g_scale * (u - 1) / 2 in (-g_scale, 0);
 *   IG_BETA    : write strength beta = (u + 1) / 2 in (0, 1);
 *                u the IG_UNIFORM draw; exact in fp32 up to the product with
 *                g_scale.
 * Optional row outliers (K only): a (token, head) row is selected with
 * probability `outlier_frac` by its own hash and multiplied by
 * `outlier_scale` in fp32 before the storage rounding.
 * bf16 storage uses round-to-nearest-even on the fp32 bit pattern.
 */
#ifndef SA_INPUTGEN_H
#define SA_INPUTGEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define IG_FN __host__ __device__ __forceinline__
#else
#define IG_FN static inline
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum { IG_NORMAL = 0, IG_UNIFORM = 1, IG_ZERO = 2, IG_ONES = 3 };
enum { IG_Q = 0, IG_K = 1, IG_V = 2, IG_OUTLIER = 3, IG_GATE = 4, IG_BETA = 5 };
enum { IG_F32 = 0, IG_BF16 = 1 };

typedef struct {
  uint64_t seed;
  int32_t dist[3];        /* per tensor Q, K, V: IG_NORMAL or IG_UNIFORM */
  double outlier_frac;    /* fraction of K rows that are scaled (0 = none) */
  float outlier_scale;    /* factor applied to selected K rows */
  int32_t pad_;
} ig_spec;

#define IG_GOLDEN 0x9E3779B97F4A7C15ULL

/* Chunk coordinate of the sink-update blocks: the [S*F][H][D] keys (IG_K) and
 * values (IG_V) of the sink update applied before chunk u are drawn at chunk
 * coordinate IG_SINK_UPDATE_CHUNK0 + u, far from every real chunk index. */
#define IG_SINK_UPDATE_CHUNK0 (1LL << 40)

IG_FN uint64_t ig_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of one (seed, stream, chunk, tensor) block of values. */
IG_FN uint64_t ig_key(uint64_t seed, int64_t stream, int64_t chunk, int32_t tensor) {
  uint64_t k = ig_mix64(seed + IG_GOLDEN);
  k = ig_mix64(k + (uint64_t)stream * IG_GOLDEN + (uint64_t)(uint32_t)tensor);
  k = ig_mix64(k ^ ((uint64_t)chunk * 0xD1B54A32D192ED03ULL));
  return k;
}

/* j-th 64-bit draw for element idx of a block. */
IG_FN uint64_t ig_draw(uint64_t key, uint64_t idx, uint32_t j) {
  return ig_mix64(key + (idx * 4u + j + 1u) * IG_GOLDEN);
}

IG_FN float ig_normal(uint64_t key, uint64_t idx) {
  int32_t s = 0;
  for (uint32_t j = 0; j < 3; ++j) {
    uint64_t z = ig_draw(key, idx, j);
    s += (int32_t)(z & 0xFFFF) + (int32_t)((z >> 16) & 0xFFFF) +
         (int32_t)((z >> 32) & 0xFFFF) + (int32_t)(z >> 48);
  }
  /* 2*s - 12*65535 is an integer of magnitude < 2^20; /2^17 is exact. */
  return (float)(2 * s - 12 * 65535) * (1.0f / 131072.0f);
}

IG_FN float ig_uniform(uint64_t key, uint64_t idx) {
  uint64_t z = ig_draw(key, idx, 0);
  uint32_t i = (uint32_t)(z >> 41); /* 23 bits */
  return (float)(2u * i + 1u) * (1.0f / 8388608.0f) - 1.0f;
}

/* Gate values of element idx = tok*H + h of an IG_GATE / IG_BETA block. */
IG_FN float ig_gate_log_decay(uint64_t key, uint64_t idx, float g_scale) {
  return g_scale * ((ig_uniform(key, idx) - 1.0f) * 0.5f);
}

IG_FN float ig_gate_beta(uint64_t key, uint64_t idx) {
  return (ig_uniform(key, idx) + 1.0f) * 0.5f;
}

/* Selection threshold for a row-outlier fraction: frac * 2^64, saturated. */
IG_FN uint64_t ig_outlier_threshold(double frac) {
  if (!(frac > 0.0)) return 0;
  double t = frac * 18446744073709551616.0;
  return t >= 18446744073709551615.0 ? ~0ULL : (uint64_t)t;
}

IG_FN int ig_row_is_outlier(uint64_t okey, uint64_t row, uint64_t thr) {
  return thr != 0 && ig_mix64(okey + (row + 1u) * IG_GOLDEN) < thr;
}

IG_FN uint16_t ig_f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } cv;
  cv.f = f;
  uint32_t u = cv.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

IG_FN float ig_bf16_to_f32(uint16_t h) {
  union { float f; uint32_t u; } cv;
  cv.u = ((uint32_t)h) << 16;
  return cv.f;
}

/*
 * Value (fp32, before storage rounding) of element idx = (tok*H + h)*D + d of
 * one block. key = ig_key(seed, stream, chunk, tensor); okey = the block's
 * IG_OUTLIER key (used only for K when thr != 0).
 */
IG_FN float ig_value_keyed(int32_t dist, uint64_t key, uint64_t okey, uint64_t thr,
                           int32_t is_k, uint64_t idx, int32_t D, float outlier_scale) {
  float x;
  if (dist == IG_ZERO) x = 0.0f;
  else if (dist == IG_ONES) x = 1.0f;
  else x = dist == IG_UNIFORM ? ig_uniform(key, idx) : ig_normal(key, idx);
  if (is_k && ig_row_is_outlier(okey, idx / (uint64_t)D, thr)) x = x * outlier_scale;
  return x;
}

/* Convenience form of ig_value_keyed that derives the keys (slower). */
IG_FN float ig_value(const ig_spec* sp, int64_t stream, int64_t chunk, int32_t tensor,
                     uint64_t idx, int32_t D) {
  uint64_t key = ig_key(sp->seed, stream, chunk, tensor);
  uint64_t okey = ig_key(sp->seed, stream, chunk, IG_OUTLIER);
  uint64_t thr = tensor == IG_K ? ig_outlier_threshold(sp->outlier_frac) : 0;
  return ig_value_keyed(sp->dist[tensor], key, okey, thr, tensor == IG_K, idx, D,
                        sp->outlier_scale);
}

#ifdef __cplusplus
}
#endif

#endif /* SA_INPUTGEN_H */
