// rope_append.cu -- K1: fused 3D RoPE + rolling-cache append; K3: RoPE refresh.
//
// Both are HBM-bound streaming kernels: every thread moves one 16-byte vector
// per tensor (8 bf16 or 4 fp32 elements = 4 or 2 rotation pairs), loads and
// stores are 16-byte and coalesced (consecutive threads cover consecutive
// 16-byte pieces of a head row), grids are a multiple of the SM count with a
// grid-stride loop.
//
// 3D RoPE (the rotary embedding StreamDiffusionV2 refreshes, technical
// summary section 2.A.2): the head dim splits into bands (d_t | d_h | d_w);
// pair (2j, 2j+1) of a band turns by pos * theta_j as
// (a, b) -> (a cos - b sin, a sin + b cos). The (cos, sin) values come from
// the host, computed in fp64: per launch for the temporal band, per cache for
// the row and column bands.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

// debug build: the bounds word of this file (sites: 0 input vector, 1 cache
// row of an appended frame, 2 raw-sink row, 3 rotated-query row, 4 ring row of
// a refresh, 5 sink row of a refresh or sink update)
SA_DEFINE_BOUNDS_WORD(bounds_word_rope_append)

namespace {

template <typename T>
struct Vec16;

template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const void* p, float (&x)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ __forceinline__ static void load_cache(const void* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ __forceinline__ static void store(void* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __device__ __forceinline__ static void copy(void* dst, const void* src) {
    *reinterpret_cast<float4*>(dst) = __ldg(reinterpret_cast<const float4*>(src));
  }
  __device__ __forceinline__ static void round(float (&)[4]) {}
};

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4 v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ __forceinline__ static void load(const void* p, float (&x)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), x);
  }
  __device__ __forceinline__ static void load_cache(const void* p, float (&x)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), x);
  }
  __device__ __forceinline__ static void store(void* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h2);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ __forceinline__ static void copy(void* dst, const void* src) {
    *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
  }
  // the value a store followed by a load gives (round to nearest even)
  __device__ __forceinline__ static void round(float (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
  }
};

__device__ __forceinline__ void rotate(float& a, float& b, const float2 cs) {
  const float na = a * cs.x - b * cs.y;
  const float nb = a * cs.y + b * cs.x;
  a = na;
  b = nb;
}

// (cos, sin) of global pair index pi of a token at row y, column x.
__device__ __forceinline__ float2 pair_cs(int pi, int y, int x, const float2* tband, int dt2,
                                          int dh2, int dw2, const float2* htab,
                                          const float2* wtab) {
  if (pi < dt2) return tband[pi];
  if (pi < dt2 + dh2) return __ldg(&htab[y * dh2 + (pi - dt2)]);
  return __ldg(&wtab[x * dw2 + (pi - dt2 - dh2)]);
}

template <typename T>
__global__ void __launch_bounds__(256) append_rope_kernel(const __grid_constant__ AppendParams p) {
  using V = Vec16<T>;
  constexpr int N = V::N;
  const uint32_t nvec = (uint32_t)p.D / N;
  const uint32_t per_tok = (uint32_t)p.H * nvec;
  const uint32_t per_stream = (uint32_t)p.Lc * per_tok;
  const uint32_t total = per_stream * (uint32_t)p.n_streams;
  const size_t esz = sizeof(T);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += gridDim.x * blockDim.x) {
    const uint32_t a = i / per_stream;
    const uint32_t r = i - a * per_stream;
    const uint32_t tok = r / per_tok;
    const uint32_t r2 = r - tok * per_tok;
    const uint32_t h = r2 / nvec;
    const uint32_t vc = r2 - h * nvec;
    const int b = p.stream_of[a];
    const int fi = (int)(tok / (uint32_t)p.F);
    const int j = (int)(tok - (uint32_t)fi * (uint32_t)p.F);
    const int y = j / p.fw, x = j - (j / p.fw) * p.fw;
    const int e = (int)a * p.C + fi;

    const int64_t in_off = (((int64_t)b * p.Lc + tok) * p.H + h) * p.D + (int64_t)vc * N;
    const int64_t bh = (int64_t)b * p.H + h;
    if (!SA_BOUNDS(b >= 0 && b < p.batch && e < kMaxEntries, 0) ||
        !SA_BOUNDS(tok < (uint32_t)p.Lc && a < (uint32_t)p.n_streams, 3))
      continue;
    const int64_t row = p.dest_row[e] + j;
    if (!SA_BOUNDS(row >= 0 && row < p.ntok, 1) ||
        !SA_BOUNDS(p.raw_row[e] < 0 || p.raw_row[e] + j < p.sf, 2))
      continue;
    float q[N], k[N];
    V::load(static_cast<const char*>(p.q) + in_off * esz, q);
    V::load(static_cast<const char*>(p.k) + in_off * esz, k);
    const int64_t cache_off = (bh * p.ntok + row) * p.D + (int64_t)vc * N;
    V::copy(static_cast<char*>(p.v_cache) + cache_off * esz,
            static_cast<const char*>(p.v) + in_off * esz);
    if (p.raw_row[e] >= 0) {
      const int64_t raw_off = (bh * p.sf + p.raw_row[e] + j) * p.D + (int64_t)vc * N;
      V::store(static_cast<char*>(p.k_raw) + raw_off * esz, k);
    }
#pragma unroll
    for (int pp = 0; pp < N / 2; ++pp) {
      const int pi = (int)vc * (N / 2) + pp;
      const float2 cs = pair_cs(pi, y, x, p.tcs[e], p.dt2, p.dh2, p.dw2, p.htab, p.wtab);
      rotate(q[2 * pp], q[2 * pp + 1], cs);
      rotate(k[2 * pp], k[2 * pp + 1], cs);
    }
    const int64_t q_off = (bh * p.Lc + tok) * p.D + (int64_t)vc * N;
    V::store(static_cast<char*>(p.q_ws) + q_off * esz, q);
    V::store(static_cast<char*>(p.k_cache) + cache_off * esz, k);
  }
}

// grid.y = stream of the launch. Ring part: only the vectors that hold
// temporal-band pairs are read and written. Sink part: every vector of the
// valid sink rows is re-derived from the raw keys; in update mode the raw
// keys and the sink values are first blended with the new sink data
// (StreamDiffusionV2, section 2.A.2: adaptive sink tokens).
template <typename T>
__global__ void __launch_bounds__(256) refresh_kernel(const __grid_constant__ RefreshParams p) {
  using V = Vec16<T>;
  constexpr int N = V::N;
  const int a = blockIdx.y;
  const int b = p.stream_of[a];
  const size_t esz = sizeof(T);
  const int64_t nvec = p.D / N;
  const int64_t nvt = (2 * p.dt2 + N - 1) / N;  // vectors touching the temporal band
  const int64_t ring_work = (int64_t)p.H * p.ring_rows[a] * nvt;
  const int64_t sink_work = (int64_t)p.H * p.sink_rows[a] * nvec;
  const int64_t total = ring_work + sink_work;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < ring_work) {
      const int64_t per_h = p.ring_rows[a] * nvt;
      const int64_t h = i / per_h;
      const int64_t rr = (i - h * per_h) / nvt;
      const int64_t vc = i - h * per_h - rr * nvt;
      if (!SA_BOUNDS(b >= 0 && b < p.batch && p.sf + rr < p.ntok && vc < nvec, 4)) continue;
      const int64_t off = (((int64_t)b * p.H + h) * p.ntok + p.sf + rr) * p.D + vc * N;
      char* ptr = static_cast<char*>(p.k_cache) + off * esz;
      float k[N];
      V::load_cache(ptr, k);
#pragma unroll
      for (int pp = 0; pp < N / 2; ++pp) {
        const int pi = (int)vc * (N / 2) + pp;
        if (pi < p.dt2) rotate(k[2 * pp], k[2 * pp + 1], p.dcs[a][pi]);
      }
      V::store(ptr, k);
    } else {
      const int64_t ii = i - ring_work;
      const int64_t per_h = p.sink_rows[a] * nvec;
      const int64_t h = ii / per_h;
      const int64_t rr = (ii - h * per_h) / nvec;
      const int64_t vc = ii - h * per_h - rr * nvec;
      const int64_t bh = (int64_t)b * p.H + h;
      const int s = (int)(rr / p.F);
      const int j = (int)(rr - (int64_t)s * p.F);
      const int y = j / p.fw, x = j - (j / p.fw) * p.fw;
      if (!SA_BOUNDS(b >= 0 && b < p.batch && rr < p.sf && s < p.S, 5)) continue;
      float k[N];
      char* raw = static_cast<char*>(p.k_raw) + ((bh * p.sf + rr) * p.D + vc * N) * esz;
      V::load_cache(raw, k);
      if (p.update) {
        // adaptive sink update: blend raw keys and values, round to storage
        const int64_t in_off = (((int64_t)b * p.S * p.F + rr) * p.H + h) * p.D + vc * N;
        char* vp = static_cast<char*>(p.v_cache) + ((bh * p.ntok + rr) * p.D + vc * N) * esz;
        float kn[N], v[N], vn[N];
        V::load(static_cast<const char*>(p.k_new) + in_off * esz, kn);
        V::load_cache(vp, v);
        V::load(static_cast<const char*>(p.v_new) + in_off * esz, vn);
        const float a = p.alpha, am = 1.f - p.alpha;
#pragma unroll
        for (int e = 0; e < N; ++e) {
          k[e] = am * k[e] + a * kn[e];
          v[e] = am * v[e] + a * vn[e];
        }
        V::store(raw, k);
        V::store(vp, v);
        V::round(k);  // the rotation starts from the stored raw key
      }
#pragma unroll
      for (int pp = 0; pp < N / 2; ++pp) {
        const int pi = (int)vc * (N / 2) + pp;
        const float2 cs =
            pair_cs(pi, y, x, p.scs[a * p.S + s], p.dt2, p.dh2, p.dw2, p.htab, p.wtab);
        rotate(k[2 * pp], k[2 * pp + 1], cs);
      }
      V::store(static_cast<char*>(p.k_cache) + ((bh * p.ntok + rr) * p.D + vc * N) * esz, k);
    }
  }
}

// ---------------------------------------------------------------- e4m3 cache
// bf16 inputs; rotated queries, rotated keys and values stored as e4m3 of the
// value times the head's scale (q, k, v scales: fp8_scale[0..2][h]); raw sink
// keys stay bf16. One thread per 8-element vector: 16-byte input loads,
// 8-byte e4m3 stores.
__device__ __forceinline__ uint2 to_e4m3x8(const float (&x)[8], float s) {
  return make_uint2(ptx::pack_e4m3x4(x[0] * s, x[1] * s, x[2] * s, x[3] * s),
                    ptx::pack_e4m3x4(x[4] * s, x[5] * s, x[6] * s, x[7] * s));
}

__device__ __forceinline__ void from_e4m3x8(const uint2 v, float inv_s, float (&x)[8]) {
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 a = ptx::unpack_e4m3x2(w[i] & 0xFFFFu), b = ptx::unpack_e4m3x2(w[i] >> 16);
    x[4 * i + 0] = a.x * inv_s;
    x[4 * i + 1] = a.y * inv_s;
    x[4 * i + 2] = b.x * inv_s;
    x[4 * i + 3] = b.y * inv_s;
  }
}

__global__ void __launch_bounds__(256) append_rope_e4m3_kernel(const __grid_constant__ AppendParams p) {
  using V = Vec16<__nv_bfloat16>;
  constexpr int N = 8;
  const uint32_t nvec = (uint32_t)p.D / N;
  const uint32_t per_tok = (uint32_t)p.H * nvec;
  const uint32_t per_stream = (uint32_t)p.Lc * per_tok;
  const uint32_t total = per_stream * (uint32_t)p.n_streams;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += gridDim.x * blockDim.x) {
    const uint32_t a = i / per_stream;
    const uint32_t r = i - a * per_stream;
    const uint32_t tok = r / per_tok;
    const uint32_t r2 = r - tok * per_tok;
    const uint32_t h = r2 / nvec;
    const uint32_t vc = r2 - h * nvec;
    const int b = p.stream_of[a];
    const int fi = (int)(tok / (uint32_t)p.F);
    const int j = (int)(tok - (uint32_t)fi * (uint32_t)p.F);
    const int y = j / p.fw, x = j - (j / p.fw) * p.fw;
    const int e = (int)a * p.C + fi;
    const int64_t in_off = (((int64_t)b * p.Lc + tok) * p.H + h) * p.D + (int64_t)vc * N;
    const int64_t bh = (int64_t)b * p.H + h;
    if (!SA_BOUNDS(b >= 0 && b < p.batch && e < kMaxEntries, 0) ||
        !SA_BOUNDS(tok < (uint32_t)p.Lc && a < (uint32_t)p.n_streams, 3))
      continue;
    const int64_t row = p.dest_row[e] + j;
    if (!SA_BOUNDS(row >= 0 && row < p.ntok, 1) ||
        !SA_BOUNDS(p.raw_row[e] < 0 || p.raw_row[e] + j < p.sf, 2))
      continue;
    float q[N], k[N], v[N];
    V::load(static_cast<const char*>(p.q) + in_off * 2, q);
    V::load(static_cast<const char*>(p.k) + in_off * 2, k);
    V::load(static_cast<const char*>(p.v) + in_off * 2, v);
    const int64_t cache_off = (bh * p.ntok + row) * p.D + (int64_t)vc * N;
    const float sq = __ldg(&p.fp8_scale[h]), sk = __ldg(&p.fp8_scale[p.H + h]),
                sv = __ldg(&p.fp8_scale[2 * p.H + h]);
    *reinterpret_cast<uint2*>(static_cast<char*>(p.v_cache) + cache_off) = to_e4m3x8(v, sv);
    if (p.raw_row[e] >= 0) {
      const int64_t raw_off = (bh * p.sf + p.raw_row[e] + j) * p.D + (int64_t)vc * N;
      V::store(static_cast<char*>(p.k_raw) + raw_off * 2, k);
    }
#pragma unroll
    for (int pp = 0; pp < N / 2; ++pp) {
      const int pi = (int)vc * (N / 2) + pp;
      const float2 cs = pair_cs(pi, y, x, p.tcs[e], p.dt2, p.dh2, p.dw2, p.htab, p.wtab);
      rotate(q[2 * pp], q[2 * pp + 1], cs);
      rotate(k[2 * pp], k[2 * pp + 1], cs);
    }
    const int64_t q_off = (bh * p.Lc + tok) * p.D + (int64_t)vc * N;
    *reinterpret_cast<uint2*>(static_cast<char*>(p.q_ws) + q_off) = to_e4m3x8(q, sq);
    *reinterpret_cast<uint2*>(static_cast<char*>(p.k_cache) + cache_off) = to_e4m3x8(k, sk);
  }
}

// Refresh / sink update of an e4m3 cache: ring keys' temporal band is
// dequantised, rotated by -Delta and requantised; sink keys are re-derived
// from the bf16 raw keys; in update mode the raw keys (bf16) and the stored
// sink values (e4m3) are first blended with the new data.
__global__ void __launch_bounds__(256) refresh_e4m3_kernel(const __grid_constant__ RefreshParams p) {
  using V = Vec16<__nv_bfloat16>;
  constexpr int N = 8;
  const int a = blockIdx.y;
  const int b = p.stream_of[a];
  const int64_t nvec = p.D / N;
  const int64_t nvt = (2 * p.dt2 + N - 1) / N;
  const int64_t ring_work = (int64_t)p.H * p.ring_rows[a] * nvt;
  const int64_t sink_work = (int64_t)p.H * p.sink_rows[a] * nvec;
  const int64_t total = ring_work + sink_work;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < ring_work) {
      const int64_t per_h = p.ring_rows[a] * nvt;
      const int64_t h = i / per_h;
      const int64_t rr = (i - h * per_h) / nvt;
      const int64_t vc = i - h * per_h - rr * nvt;
      if (!SA_BOUNDS(b >= 0 && b < p.batch && p.sf + rr < p.ntok && vc < nvec, 4)) continue;
      const int64_t off = (((int64_t)b * p.H + h) * p.ntok + p.sf + rr) * p.D + vc * N;
      uint2* ptr = reinterpret_cast<uint2*>(static_cast<char*>(p.k_cache) + off);
      const float sk = __ldg(&p.fp8_scale[p.H + h]);
      float k[N];
      from_e4m3x8(*ptr, 1.f / sk, k);
#pragma unroll
      for (int pp = 0; pp < N / 2; ++pp) {
        const int pi = (int)vc * (N / 2) + pp;
        if (pi < p.dt2) rotate(k[2 * pp], k[2 * pp + 1], p.dcs[a][pi]);
      }
      *ptr = to_e4m3x8(k, sk);
    } else {
      const int64_t ii = i - ring_work;
      const int64_t per_h = p.sink_rows[a] * nvec;
      const int64_t h = ii / per_h;
      const int64_t rr = (ii - h * per_h) / nvec;
      const int64_t vc = ii - h * per_h - rr * nvec;
      const int64_t bh = (int64_t)b * p.H + h;
      const int s = (int)(rr / p.F);
      const int j = (int)(rr - (int64_t)s * p.F);
      const int y = j / p.fw, x = j - (j / p.fw) * p.fw;
      if (!SA_BOUNDS(b >= 0 && b < p.batch && rr < p.sf && s < p.S, 5)) continue;
      const float sk = __ldg(&p.fp8_scale[p.H + h]);
      float k[N];
      char* raw = static_cast<char*>(p.k_raw) + ((bh * p.sf + rr) * p.D + vc * N) * 2;
      V::load_cache(raw, k);
      if (p.update) {
        const int64_t in_off = (((int64_t)b * p.S * p.F + rr) * p.H + h) * p.D + vc * N;
        uint2* vp = reinterpret_cast<uint2*>(static_cast<char*>(p.v_cache) +
                                             (bh * p.ntok + rr) * p.D + vc * N);
        const float sv = __ldg(&p.fp8_scale[2 * p.H + h]);
        float kn[N], v[N], vn[N];
        V::load(static_cast<const char*>(p.k_new) + in_off * 2, kn);
        from_e4m3x8(*vp, 1.f / sv, v);
        V::load(static_cast<const char*>(p.v_new) + in_off * 2, vn);
        const float al = p.alpha, am = 1.f - p.alpha;
#pragma unroll
        for (int e = 0; e < N; ++e) {
          k[e] = am * k[e] + al * kn[e];
          v[e] = am * v[e] + al * vn[e];
        }
        V::store(raw, k);
        *vp = to_e4m3x8(v, sv);
        V::round(k);  // the rotation starts from the stored raw key
      }
#pragma unroll
      for (int pp = 0; pp < N / 2; ++pp) {
        const int pi = (int)vc * (N / 2) + pp;
        const float2 cs =
            pair_cs(pi, y, x, p.scs[a * p.S + s], p.dt2, p.dh2, p.dw2, p.htab, p.wtab);
        rotate(k[2 * pp], k[2 * pp + 1], cs);
      }
      *reinterpret_cast<uint2*>(static_cast<char*>(p.k_cache) + (bh * p.ntok + rr) * p.D + vc * N) =
          to_e4m3x8(k, sk);
    }
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, int dtype, int num_sms, cudaStream_t st) {
  const int64_t vec = dtype == SA_F32 ? 4 : 8;
  const int64_t total = (int64_t)p.n_streams * p.Lc * p.H * (p.D / vec);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (dtype == SA_BF16_E4M3)
    append_rope_e4m3_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
  else if (dtype == SA_BF16)
    append_rope_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(p);
  else
    append_rope_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_refresh(const RefreshParams& p, int dtype, int num_sms, cudaStream_t st) {
  const int per_stream = (num_sms * 8 + p.n_streams - 1) / p.n_streams;
  dim3 grid((unsigned)(per_stream > 0 ? per_stream : 1), (unsigned)p.n_streams);
  if (dtype == SA_BF16_E4M3)
    refresh_e4m3_kernel<<<grid, 256, 0, st>>>(p);
  else if (dtype == SA_BF16)
    refresh_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
  else
    refresh_kernel<float><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
