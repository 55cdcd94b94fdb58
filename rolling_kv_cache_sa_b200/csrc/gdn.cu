// gdn.cu -- Gated DeltaNet (GDN) block: one call advances every active
// stream's recurrent state over T tokens and writes the block's outputs.
//
// SANA-Streaming (section "hybrid diffusion transformer"): most blocks of
// that model use GDN linear attention, a recurrent state of fixed size per
// head that is updated as frames arrive and is the only thing a GDN block
// keeps between chunks; section "system co-design": the fused kernel keeps
// that state on chip. The recurrence is the published gated delta rule
// (Yang, Kautz and Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with
// Delta Rule", ICLR 2025) with L2-normalised queries and keys, per head:
//     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//     o_t = scale * S_t q_t
// with S a D x D matrix (row i = value dim i, column j = key dim j).
//
// The kernels run the chunkwise form of that recurrence (the WY form of Yang
// et al., "Parallelizing Linear Transformers with the Delta Rule over
// Sequence Length", NeurIPS 2024) on sub-chunks of 64 tokens. With S0 the
// state before a sub-chunk and G_t = g_1 + ... + g_t inside it, the
// corrected values u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t) solve
//     (I + L) U = diag(beta) (V - diag(e^G) K S0^T),
//     L_ts = beta_t e^(G_t - G_s) k_t . k_s  (s < t),
// and then
//     o_t   = scale (e^(G_t) S0 q_t + sum_{s<=t} P_ts u_s),  P_ts = e^(G_t - G_s) q_t . k_s
//     S_end = e^(G_last) S0 + sum_s e^(G_last - G_s) u_s k_s^T.
// (I + L)^-1 is unit lower triangular: its 16 x 16 diagonal blocks come from
// forward substitution, and two merges use
//     [A 0; C B]^-1 = [A^-1 0; -B^-1 C A^-1  B^-1].
//
// Two kernels per call:
//  * the prep kernel: one CTA per (stream, head, sub-chunk), all independent.
//    It computes what depends only on K, Q, g and beta -- T = (I + L)^-1 and
//    M = scale P T. With U = T RHS, the intra-chunk part of the outputs is
//    P U = M RHS, so the sequential pass gets U and the outputs from one
//    sweep over RHS.
//  * the sequential pass: one CTA per (stream, head, slice of value rows of
//    the state). Rows of S evolve independently, so a CTA owns its slice of
//    the state for the whole call and walks the sub-chunks in order.
// D = 128 runs on the tensor core: gdn_prep_tc_kernel forms the Gram
// matrices with tcgen05 MMAs and writes bf16 hi/lo operand images of K^, Q^,
// T and M; gdn_tc_kernel keeps a 64-column state slice in TMEM (both
// described where they are defined). D = 64 runs in fp32 on the CUDA cores:
// gdn_prep_kernel writes T and M (64 x 64 fp32 each) and gdn_chunk_kernel
// keeps a 32-row state slice in registers, with a copy in shared memory for
// the products that read it by rows, loading each sub-chunk's T and M one
// sub-chunk ahead.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

// debug build: the bounds word of this file (sites: 0 stream / sub-chunk of a
// prep block, 1 workspace block written, 2 workspace block read, 3 state
// slice, 4 sub-chunk token range)
SA_DEFINE_BOUNDS_WORD(bounds_word_gdn)

namespace {

constexpr int kCt = 64;         // tokens per sub-chunk
constexpr int kDvs = 32;        // state rows (value dims) per CTA
constexpr int kGdnThreads = 256;
constexpr int kLp = kCt + 4;    // row pitch of the 64 x 64 matrices (16-byte rows)
constexpr int kVp = kDvs + 4;   // row pitch of the 64 x 32 matrices (16-byte rows)
constexpr int kTpFloats = 2 * kCt * kCt;   // T and P of one sub-chunk in the workspace
// The workspace starts with a 1 KiB header holding the device status word of
// the tensor-core path (bounded waits); the per-sub-chunk blocks follow.
constexpr size_t kWsHeader = 1024;
// Tensor-core path (D = 128): per sub-chunk the prep kernel writes the
// operand images of the sequential kernel's MMAs, bf16, each value x as
// hi = bf16(x) and lo = bf16(x - hi), in the 128-byte-swizzled layout the
// tensor core reads (64-column panels; row r at r * 128 bytes of its panel,
// the 16-byte chunk c of row r stored at chunk c ^ (r mod 8)):
//   KQ: rows 0..63 the normalised keys, rows 64..127 the normalised queries,
//       128 columns (2 panels): 32 KiB for hi, 32 KiB for lo;
//   TM: rows 0..63 T = (I + L)^-1, rows 64..127 M = scale P T, 64 columns:
//       16 KiB for hi, 16 KiB for lo.
constexpr uint32_t kImgKQ = 32768, kImgTM = 16384;
constexpr uint32_t kImgBytes = 2 * kImgKQ + 2 * kImgTM;

// Byte offset of (row, 8-column chunk c) in a 128-byte-swizzled panel.
__host__ __device__ __forceinline__ uint32_t sw128_off(int row, int c) {
  return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
}

// Eight floats as bf16 hi = bf16(x) and lo = bf16(x - hi) (round to nearest
// even), each packed into 16 bytes.
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    h[i] = *reinterpret_cast<uint32_t*>(&b);
    const float r0 = x[2 * i] - __uint_as_float(h[i] << 16);
    const float r1 = x[2 * i + 1] - __uint_as_float(h[i] & 0xffff0000u);
    __nv_bfloat162 c = __floats2bfloat162_rn(r0, r1);
    l[i] = *reinterpret_cast<uint32_t*>(&c);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}
constexpr float kLog2e = 1.4426950408889634f;

// Rows of K^ and Q^ have pitch D + 4: a multiple of 4 (16-byte aligned rows)
// whose 16-byte groups step by an odd count, so float4 reads of consecutive
// rows fall in different bank groups.
template <int D>
struct GdnPrepSmem {
  static constexpr int KP = D + 4;
  static constexpr int kh = 0;                    // [64][KP] normalised keys; later T
  static constexpr int qh = kh + kCt * KP;        // [64][KP] normalised queries; later merge scratch
  static constexpr int lm = qh + kCt * KP;        // [64][68] L (strictly lower)
  static constexpr int pm = lm + kCt * kLp;       // [64][68] scale e^(G_t-G_s) q_t.k_s (s <= t)
  static constexpr int gs = pm + kCt * kLp;       // [64] in-warp prefix sums of g log2(e)
  static constexpr int bs = gs + kCt;             // [64] beta
  static constexpr int total = bs + kCt;
  static constexpr size_t bytes = (size_t)total * sizeof(float);
  static_assert(kCt * kLp <= kCt * KP, "T must fit in the key rows it replaces");
  static_assert(32 * 33 <= kCt * KP, "merge scratch must fit in the query rows");
};

// The state slice has pitch D with its 16-byte groups XOR-swizzled by
// (row / 4) mod 8, so float4 reads of rows 4x + i (x = 0..7) are conflict
// free. The staging area receives the next sub-chunk's raw q, k rows and
// value slice (input element type) by cp.async while the current one is
// computed; T and P arrive the same way.
template <int D, typename T>
struct GdnSmem {
  static constexpr int KP = D + 4;
  static constexpr int kh = 0;                    // [64][KP] normalised keys
  static constexpr int qh = kh + kCt * KP;        // [64][KP] normalised queries
  static constexpr int st = qh + kCt * KP;        // [32][D] state slice S0 (swizzled)
  static constexpr int tm = st + kDvs * D;        // [64][68] (I + L)^-1 (lower)
  static constexpr int pm = tm + kCt * kLp;       // [64][68] M = scale P T (lower)
  static constexpr int rv = pm + kCt * kLp;       // [64][36] v slice, then the right-hand side
  static constexpr int uv = rv + kCt * kVp;       // [64][36] u_t e^(G_last - G_t)
  static constexpr int gs = uv + kCt * kVp;       // [64] in-warp prefix sums of g log2(e)
  static constexpr int bs = gs + kCt;             // [64] beta
  static constexpr int ws = bs + kCt;             // [64] e^(G_last - G_t)
  static constexpr int stage = (ws + kCt + 3) / 4 * 4;   // raw staging (bytes from here)
  static constexpr int kStageK = kCt * D * (int)sizeof(T);        // bytes of 64 raw rows
  static constexpr int kStageV = kCt * kDvs * (int)sizeof(T);     // bytes of 64 value slices
  static constexpr size_t bytes = (size_t)stage * sizeof(float) + 2 * kStageK + kStageV;
};
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Four consecutive input elements (16 bytes of fp32 or 8 of bf16) as floats.
__device__ __forceinline__ float4 ld_raw4(const float* p) { return ld4(p); }
__device__ __forceinline__ float4 ld_raw4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}
// Two consecutive input elements as floats.
__device__ __forceinline__ float2 ld_raw2(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
__device__ __forceinline__ float2 ld_raw2(const __nv_bfloat16* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void st_out(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// Normalises rows r = warp + 8 i (i < 8) of K and Q into Kh and Qh (pitch
// KP): row r of the raw inputs starts at kraw + r * rs and qraw + r * rs
// (shared staging or global memory); rows past n and zero vectors give 0.
template <int D, int KP, typename T>
__device__ __forceinline__ void normalise_rows(const T* kraw, const T* qraw, size_t rs, int n,
                                               float* Kh, float* Qh, int warp, int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = warp + 8 * i;
    float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), qx = kx;
    if (r < n) {
      if constexpr (D == 128) {
        kx = ld_raw4(kraw + r * rs + 4 * lane);
        qx = ld_raw4(qraw + r * rs + 4 * lane);
      } else {
        const float2 k2 = ld_raw2(kraw + r * rs + 2 * lane);
        const float2 q2 = ld_raw2(qraw + r * rs + 2 * lane);
        kx = make_float4(k2.x, k2.y, 0.f, 0.f);
        qx = make_float4(q2.x, q2.y, 0.f, 0.f);
      }
    }
    float sk = dot4(kx, kx, 0.f), sq = dot4(qx, qx, 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sk += __shfl_xor_sync(0xffffffffu, sk, o);
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
    }
    const float ik = sk > 0.f ? rsqrtf(sk) : 0.f;
    const float iq = sq > 0.f ? rsqrtf(sq) : 0.f;
    if constexpr (D == 128) {
      st4(Kh + r * KP + 4 * lane, make_float4(kx.x * ik, kx.y * ik, kx.z * ik, kx.w * ik));
      st4(Qh + r * KP + 4 * lane, make_float4(qx.x * iq, qx.y * iq, qx.z * iq, qx.w * iq));
    } else {
      *reinterpret_cast<float2*>(Kh + r * KP + 2 * lane) = make_float2(kx.x * ik, kx.y * ik);
      *reinterpret_cast<float2*>(Qh + r * KP + 2 * lane) = make_float2(qx.x * iq, qx.y * iq);
    }
  }
}

// Inclusive prefix sums of g log2(e) over the 64 tokens of a sub-chunk, per
// warp (threads 0..63); warp 1's sums lack warp 0's total (gcum adds it).
__device__ __forceinline__ void gate_scan(float g, float beta, float* Gs, float* Bs, int tid,
                                          int lane) {
  float gl = g * kLog2e;
  Bs[tid] = beta;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, gl, o);
    if (lane >= o) gl += y;
  }
  Gs[tid] = gl;
}

// T = (I + L)^-1 of one sub-chunk: L strictly lower in Lm (pitch kLp), T
// into Tm, Xm merge scratch (32 x 33 floats); all kGdnThreads threads take
// part and the last step ends with a barrier.
__device__ __forceinline__ void unit_lower_inverse(const float* Lm, float* Tm, float* Xm, int tid,
                                                   int warp, int lane) {
  // ---- diagonal 16 x 16 blocks of (I + L)^-1: thread (blk, j) solves for
  // column j of its block
  if (tid < 64) {
    const int r0 = (tid >> 4) * 16, j = tid & 15;
    float x[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float acc = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < t; ++s2) acc = fmaf(Lm[(r0 + t) * kLp + r0 + s2], x[s2], acc);
      x[t] = t < j ? 0.f : (t == j ? 1.f : -acc);
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) Tm[(r0 + t) * kLp + r0 + j] = x[t];
  }
  __syncthreads();

  // ---- merge to 32 x 32 blocks (rows r0+16.., columns r0.., r0 = 0, 32):
  // X = L21 T11, then T21 = -T22 X
#pragma unroll
  for (int e0 = 0; e0 < 512; e0 += kGdnThreads) {
    const int e = e0 + tid;
    const int pp = e >> 8, i = (e >> 4) & 15, j = e & 15, r0 = pp * 32;
    float acc = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2)
      if (s2 >= j)
        acc = fmaf(Lm[(r0 + 16 + i) * kLp + r0 + s2], Tm[(r0 + s2) * kLp + r0 + j], acc);
    Xm[pp * 272 + i * 17 + j] = acc;
  }
  __syncthreads();
#pragma unroll
  for (int e0 = 0; e0 < 512; e0 += kGdnThreads) {
    const int e = e0 + tid;
    const int pp = e >> 8, i = (e >> 4) & 15, j = e & 15, r0 = pp * 32;
    float acc = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2)
      if (s2 <= i)
        acc = fmaf(Tm[(r0 + 16 + i) * kLp + r0 + 16 + s2], Xm[pp * 272 + s2 * 17 + j], acc);
    Tm[(r0 + 16 + i) * kLp + r0 + j] = -acc;
  }
  __syncthreads();
  // ---- merge to the full 64 x 64 inverse (rows 32.., columns 0..31): warp
  // w takes rows 4w .. 4w+3 of the 32 x 32 block, lane j its column j
  {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int j = lane;
#pragma unroll
    for (int s4 = 0; s4 < 32; s4 += 4) {
      float4 l4[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) l4[r] = ld4(Lm + (32 + warp * 4 + r) * kLp + s4);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float tv = s4 + u >= j ? Tm[(s4 + u) * kLp + j] : 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float lv = u == 0 ? l4[r].x : u == 1 ? l4[r].y : u == 2 ? l4[r].z : l4[r].w;
          acc[r] = fmaf(lv, tv, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) Xm[(warp * 4 + r) * 33 + j] = acc[r];
  }
  __syncthreads();
  {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int j = lane;
#pragma unroll
    for (int s4 = 0; s4 < 32; s4 += 4) {
      float4 t4[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) t4[r] = ld4(Tm + (32 + warp * 4 + r) * kLp + 32 + s4);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float xv = Xm[(s4 + u) * 33 + j];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float tv = u == 0 ? t4[r].x : u == 1 ? t4[r].y : u == 2 ? t4[r].z : t4[r].w;
          if (s4 + u <= warp * 4 + r) acc[r] = fmaf(tv, xv, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) Tm[(32 + warp * 4 + r) * kLp + j] = -acc[r];
  }
  __syncthreads();
}

// M = P T of one sub-chunk (both lower triangular, pitch kLp) into Mm, which
// may alias the L of unit_lower_inverse (dead by then). The outputs'
// intra-chunk part is P U = P T RHS = M RHS. Ends with a barrier.
__device__ __forceinline__ void p_times_t(const float* Pm, const float* Tm, float* Mm, int tid) {
  // thread (ty, tx) takes rows ty + 16a and columns tx + 16b, b <= a
  {
    const int ty = tid >> 4, tx = tid & 15;
    float acc[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int r = 0; r < kCt; ++r) {
      float pv[4], tv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int t = ty + 16 * a, s2 = tx + 16 * a;
        pv[a] = r <= t ? Pm[t * kLp + r] : 0.f;
        tv[a] = r >= s2 ? Tm[r * kLp + s2] : 0.f;
      }
      int i = 0;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb <= a; ++bb, ++i) acc[i] = fmaf(pv[a], tv[bb], acc[i]);
    }
    int i = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int t = ty + 16 * a, s2 = tx + 16 * bb;
        float mv = 0.f;
        if (bb <= a) {
          if (s2 <= t) mv = acc[i];
          ++i;
        }
        Mm[t * kLp + s2] = mv;
      }
  }
  __syncthreads();
}

// M = P T of one sub-chunk in 4 x 4 register blocks: Pt holds P transposed
// (Pt[s][t] = P[t][s], zero for s > t) and Tm is T with zeros above the
// diagonal; Mm (pitch kLp, may alias the dead L) gets the 136 lower blocks
// (thread i < 136 takes block i in row-major order of (bt, bs), bs <= bt).
// Block (bt, bs) needs r in [4 bs, 4 bt + 4); each warp loops over the union
// of its threads' ranges, the zeros making the extra terms vanish. Ends with
// a barrier.
__device__ __forceinline__ void p_times_t_blocked(const float* Pt, const float* Tm, float* Mm,
                                                  int tid, int warp) {
  constexpr int kBlocks = (kCt / 4) * (kCt / 4 + 1) / 2;   // 136
  if (warp * 32 < kBlocks) {
    int bt = 0, rem = tid < kBlocks ? tid : kBlocks - 1;
    while (rem > bt) rem -= ++bt;
    const int bs = rem;
    // the warp's range: its first block has the smallest bs (0 unless the
    // warp starts inside row bt), its last the largest bt
    const int first = warp * 32, last = min(first + 31, kBlocks - 1);
    int bt_f = 0, rem_f = first;
    while (rem_f > bt_f) rem_f -= ++bt_f;
    int bt_l = 0, rem_l = last;
    while (rem_l > bt_l) rem_l -= ++bt_l;
    const int r_lo = bt_f == bt_l ? 4 * rem_f : 0, r_hi = 4 * bt_l + 4;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
    for (int r = r_lo; r < r_hi; ++r) {
      const float4 pv = ld4(Pt + r * kLp + 4 * bt);
      const float4 tv = ld4(Tm + r * kLp + 4 * bs);
      const float pa[4] = {pv.x, pv.y, pv.z, pv.w}, tb[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(pa[a], tb[c], acc[a][c]);
    }
    if (tid < kBlocks) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
        st4(Mm + (4 * bt + a) * kLp + 4 * bs, make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]));
    }
  }
  __syncthreads();
}

// Prep of the CUDA-core path (D = 64): one CTA per (stream, head,
// sub-chunk), T = (I + L)^-1 and M = scale P T of the sub-chunk into the
// workspace, both [64][64] row-major, zero above the diagonal.
template <int D, typename T>
__global__ void __launch_bounds__(kGdnThreads, 2) gdn_prep_kernel(const __grid_constant__ GdnParams p) {
  using L = GdnPrepSmem<D>;
  constexpr int KP = L::KP;
  extern __shared__ __align__(16) float sm[];
  float* Kh = sm + L::kh;
  float* Qh = sm + L::qh;
  float* Lm = sm + L::lm;
  float* Pm = sm + L::pm;
  float* Gs = sm + L::gs;
  float* Bs = sm + L::bs;
  float* Tm = Kh;   // [64][68], after the Gram matrices are built
  float* Xm = Qh;   // [32][33] merge scratch, likewise

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = blockIdx.x, h = blockIdx.y, z = blockIdx.z, b = p.stream_of[z];
  const int H = p.H;
  const int64_t Tn = p.T;
  const int64_t t0 = (int64_t)j * kCt;
  const int n = (int)(Tn - t0 < kCt ? Tn - t0 : kCt);
  // (block-uniform: the whole block leaves before any barrier)
  if (!SA_BOUNDS(b >= 0 && b < p.batch && z < p.n_streams && j < p.n_sub && n > 0, 0)) return;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const size_t tok_stride = (size_t)H * D;
  const size_t row0 = ((size_t)b * (size_t)Tn + (size_t)t0) * tok_stride + (size_t)h * D;
  const size_t g0 = ((size_t)b * (size_t)Tn + (size_t)t0) * H + h;
  auto gcum = [&](int t) -> float { return Gs[t] + (t >= 32 ? Gs[31] : 0.f); };

  normalise_rows<D, KP>(k + row0, q + row0, tok_stride, n, Kh, Qh, warp, lane);
  if (tid < kCt) {
    const bool ok = tid < n;
    gate_scan(ok ? p.g[g0 + (size_t)tid * H] : 0.f, ok ? p.beta[g0 + (size_t)tid * H] : 0.f,
              Gs, Bs, tid, lane);
  }
  __syncthreads();
  // the call's device status word starts at zero (the prep kernel runs first)
  if (j == 0 && h == 0 && z == 0 && tid == 0) *reinterpret_cast<int*>(p.workspace) = 0;
  const size_t blk = ((size_t)z * H + h) * (size_t)p.n_sub + (size_t)j;

  // ---- Gram matrices on the lower triangle -> L and P. Thread (ty, tx)
  // takes rows ty + 16a and columns tx + 16b, b <= a (the pairs a < b lie
  // above the diagonal).
  {
    const int ty = tid >> 4, tx = tid & 15;
    float akk[10], aqk[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) akk[i] = aqk[i] = 0.f;
#pragma unroll 2
    for (int d = 0; d < D; d += 4) {
      float4 kr[4], qr[4], kc[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        kr[a] = ld4(Kh + (ty + 16 * a) * KP + d);
        qr[a] = ld4(Qh + (ty + 16 * a) * KP + d);
        kc[a] = ld4(Kh + (tx + 16 * a) * KP + d);
      }
      int i = 0;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb <= a; ++bb, ++i) {
          akk[i] = dot4(kr[a], kc[bb], akk[i]);
          aqk[i] = dot4(qr[a], kc[bb], aqk[i]);
        }
    }
    int i = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int t = ty + 16 * a, s = tx + 16 * bb;
        float lv = 0.f, pv = 0.f;
        if (bb <= a) {
          if (s <= t) {
            const float e = ex2f(gcum(t) - gcum(s));
            if (s < t) lv = Bs[t] * e * akk[i];
            pv = p.scale * e * aqk[i];
          }
          ++i;
        }
        Lm[t * kLp + s] = lv;
        Pm[t * kLp + s] = pv;
      }
  }
  __syncthreads();
  unit_lower_inverse(Lm, Tm, Xm, tid, warp, lane);
  p_times_t(Pm, Tm, Lm, tid);

  {
    // ---- T and M to the workspace, zero above the diagonal
    float* dst = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(p.workspace) + kWsHeader) +
                 blk * kTpFloats;
    if (!SA_BOUNDS(blk < (size_t)p.n_streams * H * (size_t)p.n_sub, 1)) return;
    for (int e = tid; e < 2 * kCt * (kCt / 4); e += kGdnThreads) {
      const int mat = e / (kCt * (kCt / 4)), row = (e / (kCt / 4)) % kCt, c4 = (e % (kCt / 4)) * 4;
      float4 x = ld4((mat ? Lm : Tm) + row * kLp + c4);
      if (c4 + 0 > row) x.x = 0.f;
      if (c4 + 1 > row) x.y = 0.f;
      if (c4 + 2 > row) x.z = 0.f;
      if (c4 + 3 > row) x.w = 0.f;
      *reinterpret_cast<float4*>(dst + mat * kCt * kCt + row * kCt + c4) = x;
    }
  }
}

// Shared memory of gdn_prep_tc_kernel (bytes from a 1024-byte-aligned base:
// the 128-byte-swizzled image needs it).
struct GdnPrepTcSmem {
  static constexpr uint32_t img = 0;                   // [hi, lo] KQ image, read by the Gram MMA
  // once the MMA has completed, the image region holds:
  static constexpr uint32_t lm = 0;                    // [64][68] f32 L, later M
  static constexpr uint32_t pm = lm + kCt * kLp * 4;   // [64][68] f32 P, transposed
  static constexpr uint32_t tm = pm + kCt * kLp * 4;   // [64][68] f32 T
  static constexpr uint32_t xm = tm + kCt * kLp * 4;   // [32][33] f32 merge scratch
  static constexpr uint32_t gs = 2 * kImgKQ;           // [64] in-warp prefix sums of g log2(e)
  static constexpr uint32_t bs = gs + kCt * 4;         // [64] beta
  static constexpr uint32_t bar = bs + kCt * 4;        // mbarrier of the Gram MMA
  static constexpr uint32_t misc = bar + 8;            // TMEM base address; a word never set
  static constexpr uint32_t bytes = misc + 8;
  static_assert(xm + 32 * 33 * 4 <= 2 * kImgKQ, "L, P, T and the merge scratch fit in the image");
};
// three CTAs per SM: 3 x 66 KB of shared memory, 3 x 64 TMEM columns
constexpr int kPrepTcCtasPerSm = 3;
constexpr uint64_t kPrepTimeoutNs = 1000000000ull;

// Four floats as bf16 hi = bf16(x) and lo = bf16(x - hi), each packed into 8 bytes.
__device__ __forceinline__ void split4(float4 x, uint2& hi, uint2& lo) {
  const float v[4] = {x.x, x.y, x.z, x.w};
  uint32_t h[2], l[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    h[i] = *reinterpret_cast<uint32_t*>(&b);
    __nv_bfloat162 c = __floats2bfloat162_rn(v[2 * i] - __uint_as_float(h[i] << 16),
                                             v[2 * i + 1] - __uint_as_float(h[i] & 0xffff0000u));
    l[i] = *reinterpret_cast<uint32_t*>(&c);
  }
  hi = make_uint2(h[0], h[1]);
  lo = make_uint2(l[0], l[1]);
}

// Prep of the tensor-core path (D = 128): one CTA per (stream, head,
// sub-chunk), computing the same T = (I + L)^-1 and M = scale P T as
// gdn_prep_kernel, with the Gram matrices on the tensor core. The normalised
// key and query rows are split into bf16 hi and lo and written once, as the
// KQ operand image, to shared memory and to the workspace; one thread issues
// [K^;Q^] K^T (128 x 64, fp32 in TMEM) as the three-term split product over
// that image (the product the sequential pass uses for its own contractions,
// about 2^-16 relative per term); the threads read it back and form L and P
// (key rows and query rows of the product). Then T, M and the TM image.
template <typename T>
__device__ __forceinline__ void prep_tc_body(const GdnParams& p) {
  constexpr int D = 128;
  using L = GdnPrepTcSmem;
  extern __shared__ __align__(1024) unsigned char smp[];
  int* status = reinterpret_cast<int*>(p.workspace);
  const uint32_t base = ptx::smem_u32(smp);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = p.j_begin + (int)blockIdx.x, h = blockIdx.y, z = blockIdx.z, b = p.stream_of[z];
  const int H = p.H;
  const int64_t Tn = p.T;
  const int64_t t0 = (int64_t)j * kCt;
  const int n = (int)(Tn - t0 < kCt ? Tn - t0 : kCt);
  // (block-uniform: the whole block leaves before any barrier)
  if (!SA_BOUNDS(b >= 0 && b < p.batch && z < p.n_streams && j < p.j_end && j < p.n_sub && n > 0,
                 0))
    return;
  // the call's device status word starts at zero (the prep kernel runs first)
  if (j == 0 && h == 0 && z == 0 && tid == 0) *status = 0;
  if (base & 1023u) {
    if (tid == 0) atomicOr(status, kDeviceErrTimeout);
    return;
  }
  float* Lm = reinterpret_cast<float*>(smp + L::lm);
  float* Pm = reinterpret_cast<float*>(smp + L::pm);
  float* Gs = reinterpret_cast<float*>(smp + L::gs);
  float* Bs = reinterpret_cast<float*>(smp + L::bs);
  float* Tm = reinterpret_cast<float*>(smp + L::tm);
  float* Xm = reinterpret_cast<float*>(smp + L::xm);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smp + L::misc);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smp + L::misc + 4);
  const uint32_t bar = base + L::bar;
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 64);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(bar, 1);
    *no_abort = 0;
    ptx::fence_mbar_init();
  }
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const size_t tok_stride = (size_t)H * D;
  const size_t row0 = ((size_t)b * (size_t)Tn + (size_t)t0) * tok_stride + (size_t)h * D;
  const size_t g0 = ((size_t)b * (size_t)Tn + (size_t)t0) * H + h;
  const size_t blk = ((size_t)z * H + h) * (size_t)p.n_sub + (size_t)j;
  const bool blk_ok = SA_BOUNDS(blk < (size_t)p.n_streams * H * (size_t)p.n_sub, 1);
  unsigned char* img_g = reinterpret_cast<unsigned char*>(p.workspace) + kWsHeader + blk * kImgBytes;
  auto gcum = [&](int t) -> float { return Gs[t] + (t >= 32 ? Gs[31] : 0.f); };

  // ---- rows: warp w normalises key and query rows w + 8i (i < 8); lane l
  // holds columns 4l .. 4l + 3, one half of the image's 16-byte chunk l / 2
  // (chunks 0..7 in panel 0, 8..15 in panel 1); rows past n are zero. All
  // loads (and the gates') are issued before any is used.
  float gv = 0.f, bv = 0.f;
  if (tid < n) {
    gv = p.g[g0 + (size_t)tid * H];
    bv = p.beta[g0 + (size_t)tid * H];
  }
  // rows in two batches of four (within the register budget of three CTAs
  // per SM)
  constexpr int kB = 4;
#pragma unroll
  for (int i0 = 0; i0 < 8; i0 += kB) {
    float4 kr[kB], qr[kB];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = warp + 8 * (i0 + i);
      kr[i] = qr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < n) {
        kr[i] = ld_raw4(k + row0 + (size_t)r * tok_stride + 4 * lane);
        qr[i] = ld_raw4(q + row0 + (size_t)r * tok_stride + 4 * lane);
      }
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = warp + 8 * (i0 + i);
      const float4 kx = kr[i], qx = qr[i];
      float sk = dot4(kx, kx, 0.f), sq = dot4(qx, qx, 0.f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float ik = sk > 0.f ? rsqrtf(sk) : 0.f;
      const float iq = sq > 0.f ? rsqrtf(sq) : 0.f;
      uint2 kh, kl, qh, ql;
      split4(make_float4(kx.x * ik, kx.y * ik, kx.z * ik, kx.w * ik), kh, kl);
      split4(make_float4(qx.x * iq, qx.y * iq, qx.z * iq, qx.w * iq), qh, ql);
      const int cc = lane >> 1;
      const uint32_t in = (uint32_t)(cc >> 3) * (kImgKQ / 2) + (uint32_t)(lane & 1) * 8;
      const uint32_t ok_ = in + sw128_off(r, cc & 7), oq = in + sw128_off(kCt + r, cc & 7);
      *reinterpret_cast<uint2*>(smp + L::img + ok_) = kh;
      *reinterpret_cast<uint2*>(smp + L::img + kImgKQ + ok_) = kl;
      *reinterpret_cast<uint2*>(smp + L::img + oq) = qh;
      *reinterpret_cast<uint2*>(smp + L::img + kImgKQ + oq) = ql;
      if (blk_ok) {
        *reinterpret_cast<uint2*>(img_g + ok_) = kh;
        *reinterpret_cast<uint2*>(img_g + kImgKQ + ok_) = kl;
        *reinterpret_cast<uint2*>(img_g + oq) = qh;
        *reinterpret_cast<uint2*>(img_g + kImgKQ + oq) = ql;
      }
    }
  }
  if (tid < kCt) gate_scan(gv, bv, Gs, Bs, tid, lane);
  ptx::fence_proxy_async_smem();   // the image, written by the threads, is read by the MMA
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- [K^;Q^] K^T: A = all 128 image rows, B = the 64 key rows, both
  // K-major (two panels of 64 key dims); terms (hi, hi), (hi, lo), (lo, hi)
  if (tid == 0) {
    constexpr uint32_t id = ptx::idesc_bf16_f32_ab(128, kCt, false, false);
    constexpr uint32_t ta[3] = {0, 0, 1}, tb[3] = {0, 1, 0};
    const uint64_t d0 = ptx::sdesc_sw128(base + L::img, 16, 1024);
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (uint32_t)(kk >> 2) * (kImgKQ / 2) + (uint32_t)(kk & 3) * 32;
        ptx::umma_ss(tmem, ptx::sdesc_add(d0, ta[i] * kImgKQ + koff),
                     ptx::sdesc_add(d0, tb[i] * kImgKQ + koff), id, (i > 0 || kk > 0) ? 1u : 0u);
      }
    ptx::umma_commit(bar);
  }
  const bool done = __syncthreads_and(ptx::mbar_wait(bar, 0, no_abort, kPrepTimeoutNs));
  ptx::tc_fence_after();
  if (done) {
    // TMEM lane 32 (w mod 4) + l is product row `row` (key rows 0..63 give
    // L, query rows 64..127 give P); warps 0-3 read columns 0..31, 4-7 32..63
    float x[32];
    ptx::tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(32 * (warp >> 2)), x);
    ptx::tmem_wait_ld();
    const int row = 32 * (warp & 3) + lane, t = row & (kCt - 1), s0 = 32 * (warp >> 2);
    const bool isq = row >= kCt;
    const float gt = gcum(t), mul = isq ? p.scale : Bs[t];
    if (!isq) {
      // L row-major
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int s = s0 + 4 * c4 + e;
          o[e] = s < t ? mul * ex2f(gt - gcum(s)) * x[4 * c4 + e] : 0.f;
        }
        st4(Lm + t * kLp + s0 + 4 * c4, make_float4(o[0], o[1], o[2], o[3]));
      }
    } else {
      // P transposed (Pm[s][t]): the lanes of a warp hold consecutive t
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int s = s0 + e;
        Pm[s * kLp + t] = s <= t ? mul * ex2f(gt - gcum(s)) * x[e] : 0.f;
      }
    }
    // T's 16 x 16 blocks above the diagonal, which the inverse leaves
    // untouched, are zero (the blocked M = P T reads whole 4 x 4 blocks)
    for (int e = tid; e < kCt * kCt; e += kGdnThreads) {
      const int r = e >> 6, c = e & (kCt - 1);
      if ((c >> 4) > (r >> 4)) Tm[r * kLp + c] = 0.f;
    }
  } else if (tid == 0) {
    atomicOr(status, kDeviceErrTimeout);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 64);
  if (!done) return;

  unit_lower_inverse(Lm, Tm, Xm, tid, warp, lane);
  p_times_t_blocked(Pm, Tm, Lm, tid, warp);

  // ---- the TM image: T rows then M rows, zero above the diagonal
  if (!blk_ok) return;
  for (int e = tid; e < 2 * kCt * (kCt / 8); e += kGdnThreads) {
    const int r = e / (kCt / 8), c = e % (kCt / 8), row = r & (kCt - 1);
    const float* src = (r < kCt ? Tm : Lm) + row * kLp + c * 8;
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = c * 8 + i <= row ? src[i] : 0.f;
    uint4 hi, lo;
    split8(x, hi, lo);
    const uint32_t off = 2 * kImgKQ + sw128_off(r, c);
    *reinterpret_cast<uint4*>(img_g + off) = hi;
    *reinterpret_cast<uint4*>(img_g + kImgTM + off) = lo;
  }
}

template <typename T>
__global__ void __launch_bounds__(kGdnThreads, kPrepTcCtasPerSm)
    gdn_prep_tc_kernel(const __grid_constant__ GdnParams p) {
  prep_tc_body<T>(p);
  // The pass that reads these images is a programmatic dependent of this
  // grid: it may be scheduled once every CTA has done its work (signalling
  // earlier would let its CTAs take whole SMs from this grid's later CTAs);
  // it runs its set-up and then waits for this grid to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // A prep piece launched while the previous pass piece still runs
  // (programmatic dependent launch) must not complete before that pass: the
  // next pass piece, which waits for this grid to complete, continues from
  // its state. One thread of the last CTA waits for the previous grid, after
  // its own work, so the other CTAs leave their slots free.
  if (p.pdl_wait && threadIdx.x == 0 && blockIdx.x == gridDim.x - 1 &&
      blockIdx.y == gridDim.y - 1 && blockIdx.z == gridDim.z - 1)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D, typename T>
__global__ void __launch_bounds__(kGdnThreads, 1) gdn_chunk_kernel(const __grid_constant__ GdnParams p) {
  using L = GdnSmem<D, T>;
  constexpr int KP = L::KP;
  constexpr int kRow16 = D * (int)sizeof(T) / 16;    // 16-byte pieces of a raw row
  constexpr int kV16 = kDvs * (int)sizeof(T) / 16;   // 16-byte pieces of a value slice
  extern __shared__ __align__(16) float sm[];
  float* Kh = sm + L::kh;
  float* Qh = sm + L::qh;
  float* St = sm + L::st;
  float* Mm = sm + L::pm;   // M = P T
  float* Tm = sm + L::tm;
  float* Rv = sm + L::rv;
  float* Uv = sm + L::uv;
  float* Gs = sm + L::gs;
  float* Bs = sm + L::bs;
  float* Ws = sm + L::ws;
  unsigned char* stg = reinterpret_cast<unsigned char*>(sm + L::stage);
  T* Kraw = reinterpret_cast<T*>(stg);                       // [64][D]
  T* Qraw = reinterpret_cast<T*>(stg + L::kStageK);          // [64][D]
  T* Vraw = reinterpret_cast<T*>(stg + 2 * L::kStageK);      // [64][32]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = blockIdx.x, h = blockIdx.y, b = p.stream_of[blockIdx.z];
  const int H = p.H;
  const int64_t Tn = p.T;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  T* out = static_cast<T*>(p.out);
  const size_t tok_stride = (size_t)H * D;
  const size_t bh0 = (size_t)b * (size_t)Tn * tok_stride + (size_t)h * D;   // (b, t=0, h, d=0)
  const size_t g0 = (size_t)b * (size_t)Tn * H + h;                           // (b, t=0, h)
  const int vcol = slice * kDvs;
  // (block-uniform: the whole block leaves before any barrier)
  if (!SA_BOUNDS(b >= 0 && b < p.batch && blockIdx.z < (unsigned)p.n_streams && vcol + kDvs <= D,
                 3))
    return;
  float* Sg = p.state + (((size_t)b * H + h) * D + vcol) * D;

  // Issues the copies of sub-chunk [t0, t0 + 64) into the staging area (rows
  // past the end are not copied; the consumer treats them as zero) and
  // returns the gates of token t0 + tid for threads tid < 64.
  auto prefetch = [&](int64_t t0, float& gl, float& bl) {
    // (the sub-chunk's T and P are fetched separately, by prefetch_tp)
    const int n = (int)(Tn - t0 < kCt ? Tn - t0 : kCt);
    for (int c = tid; c < kCt * kRow16; c += kGdnThreads) {
      const int r = c / kRow16, piece = c % kRow16;
      if (r < n) {
        const size_t off = bh0 + (size_t)(t0 + r) * tok_stride;
        cp_async16(reinterpret_cast<unsigned char*>(Kraw + r * D) + piece * 16,
                   reinterpret_cast<const unsigned char*>(k + off) + piece * 16);
        cp_async16(reinterpret_cast<unsigned char*>(Qraw + r * D) + piece * 16,
                   reinterpret_cast<const unsigned char*>(q + off) + piece * 16);
      }
    }
    for (int c = tid; c < kCt * kV16; c += kGdnThreads) {
      const int r = c / kV16, piece = c % kV16;
      if (r < n) {
        const size_t off = bh0 + (size_t)(t0 + r) * tok_stride + vcol;
        cp_async16(reinterpret_cast<unsigned char*>(Vraw + r * kDvs) + piece * 16,
                   reinterpret_cast<const unsigned char*>(v + off) + piece * 16);
      }
    }
    cp_async_commit();
    if (tid < kCt) {
      const bool ok = tid < n;
      gl = ok ? p.g[g0 + (size_t)(t0 + tid) * H] : 0.f;
      bl = ok ? p.beta[g0 + (size_t)(t0 + tid) * H] : 0.f;
    }
  };

  // Issues the copies of T and M = scale P T of sub-chunk j from the
  // workspace (written by gdn_prep_kernel) into Tm and Mm.
  const float* wsp =
      reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(p.workspace) +
                                     kWsHeader) +
      ((size_t)blockIdx.z * H + h) * (size_t)p.n_sub * kTpFloats;
  auto prefetch_tp = [&](int64_t j) {
    if (!SA_BOUNDS(j >= 0 && j < p.n_sub, 2)) j = 0;
    const float* src = wsp + (size_t)j * kTpFloats;
    for (int c = tid; c < 2 * kCt * (kCt / 4); c += kGdnThreads) {
      const int mat = c / (kCt * (kCt / 4)), row = (c / (kCt / 4)) % kCt, c4 = (c % (kCt / 4)) * 4;
      cp_async16((mat ? Mm : Tm) + row * kLp + c4, src + mat * kCt * kCt + row * kCt + c4);
    }
    cp_async_commit();
  };

  // Cumulative log2 decay through token t of the sub-chunk (warp 1's prefix
  // sums lack warp 0's total, added here).
  auto gcum = [&](int t) -> float { return Gs[t] + (t >= 32 ? Gs[31] : 0.f); };

  // Offset of (row r, column col) of the state slice: 16-byte group col / 4
  // is stored at group (col / 4) xor ((r / 4) mod 8) of row r.
  auto st_off = [](int r, int col) -> int {
    return r * D + ((((col >> 2) ^ ((r >> 2) & 7)) << 2) | (col & 3));
  };
  // State block this thread updates: rows 4 warp + i (i < 4), columns
  // NC lane .. NC lane + NC - 1 (NC = D / 32 = 4 or 2).
  constexpr int NC = D / 32;
  const int ur = warp * 4;
  const int ucol = NC * lane;
  float sreg[4][NC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      sreg[i][c] = Sg[(size_t)(ur + i) * D + ucol + c];
      St[st_off(ur + i, ucol + c)] = sreg[i][c];
    }
  // Tokens and state rows of the products with 32 state rows (right-hand
  // side, U, outputs): tokens tq + 32a (a < 2), rows cq .. cq + 3.
  const int tq = warp * 4 + (lane >> 3);
  const int cq = 4 * (lane & 7);

  float gnext = 0.f, bnext = 0.f;
  prefetch(0, gnext, bnext);
  prefetch_tp(0);

  for (int64_t t0 = 0; t0 < Tn; t0 += kCt) {
    const int n = (int)(Tn - t0 < kCt ? Tn - t0 : kCt);
    (void)SA_BOUNDS(n > 0 && t0 / kCt < p.n_sub, 4);
    cp_async_wait_all();
    if (tid < kCt) gate_scan(gnext, bnext, Gs, Bs, tid, lane);   // warps 0 and 1
    __syncthreads();

    // ---- normalised key and query rows, the value slice (rows past n are 0)
    normalise_rows<D, KP>(Kraw, Qraw, (size_t)D, n, Kh, Qh, warp, lane);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = warp + 8 * i;
      Rv[r * kVp + lane] = r < n ? to_f(Vraw[r * kDvs + lane]) : 0.f;
    }
    __syncthreads();
    // the staging area is free again: fetch the next sub-chunk behind this one
    if (t0 + kCt < Tn) prefetch(t0 + kCt, gnext, bnext);

    // ---- K^ S0^T and Q^ S0^T for this CTA's rows. The right-hand side
    // beta_t (v_t - e^(G_t) (S0 k_t)) replaces v in Rv; the inter-chunk part of
    // the output, scale e^(G_t) (S0 q_t), stays in registers.
    float oin[2][4];
    {
      float aks[2][4], aqs[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < 4; ++i) aks[a][i] = aqs[a][i] = 0.f;
#pragma unroll 2
      for (int d = 0; d < D; d += 4) {
        float4 sr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sr[i] = ld4(St + st_off(cq + i, d));
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const float4 k4 = ld4(Kh + (tq + 32 * a) * KP + d);
          const float4 q4 = ld4(Qh + (tq + 32 * a) * KP + d);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            aks[a][i] = dot4(k4, sr[i], aks[a][i]);
            aqs[a][i] = dot4(q4, sr[i], aqs[a][i]);
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int t = tq + 32 * a;
        const float gam = ex2f(gcum(t));
        const float bt = Bs[t];
        float4 r = ld4(Rv + t * kVp + cq);
        r.x = bt * (r.x - gam * aks[a][0]);
        r.y = bt * (r.y - gam * aks[a][1]);
        r.z = bt * (r.z - gam * aks[a][2]);
        r.w = bt * (r.w - gam * aks[a][3]);
        st4(Rv + t * kVp + cq, r);
#pragma unroll
        for (int i = 0; i < 4; ++i) oin[a][i] = p.scale * gam * aqs[a][i];
      }
    }
    if (tid < kCt) Ws[tid] = ex2f(gcum(kCt - 1) - gcum(tid));   // end-state weights
    __syncthreads();

    // ---- one pass over the right-hand side: U = T RHS (the corrected values)
    // and the outputs' intra-chunk part P U = M RHS. Rows of RHS past n are
    // zero, so the sums run over all 64 tokens. u_t e^(G_last - G_t) goes to
    // Uv for the state update.
    {
      float uacc[2][4], acc[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < 4; ++i) uacc[a][i] = 0.f, acc[a][i] = oin[a][i];
#pragma unroll 8
      for (int s2 = 0; s2 < kCt; ++s2) {
        const float4 r4 = ld4(Rv + s2 * kVp + cq);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int t = tq + 32 * a;
          const float tv = s2 <= t ? Tm[t * kLp + s2] : 0.f;
          const float mv = s2 <= t ? Mm[t * kLp + s2] : 0.f;
          uacc[a][0] = fmaf(tv, r4.x, uacc[a][0]);
          uacc[a][1] = fmaf(tv, r4.y, uacc[a][1]);
          uacc[a][2] = fmaf(tv, r4.z, uacc[a][2]);
          uacc[a][3] = fmaf(tv, r4.w, uacc[a][3]);
          acc[a][0] = fmaf(mv, r4.x, acc[a][0]);
          acc[a][1] = fmaf(mv, r4.y, acc[a][1]);
          acc[a][2] = fmaf(mv, r4.z, acc[a][2]);
          acc[a][3] = fmaf(mv, r4.w, acc[a][3]);
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int t = tq + 32 * a;
        const float w = Ws[t];
        st4(Uv + t * kVp + cq, make_float4(uacc[a][0] * w, uacc[a][1] * w, uacc[a][2] * w,
                                           uacc[a][3] * w));
        if (t < n) {
          const size_t o = bh0 + (size_t)(t0 + t) * tok_stride + vcol + cq;
#pragma unroll
          for (int i = 0; i < 4; ++i) st_out(out, o + i, acc[a][i]);
        }
      }
    }
    __syncthreads();
    // T and M of this sub-chunk have been read: fetch the next sub-chunk's
    if (t0 + kCt < Tn) prefetch_tp(t0 / kCt + 1);
    // ---- state: S = e^(G_last) S0 + sum_t (u_t e^(G_last - G_t)) k_t^T
    // (u and k are zero past n)
    {
      const float dec = ex2f(gcum(kCt - 1));
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < NC; ++c) sreg[i][c] *= dec;
#pragma unroll 8
      for (int t = 0; t < kCt; ++t) {
        const float4 uw = ld4(Uv + t * kVp + ur);
        float kv[NC];
        if constexpr (NC == 4) {
          const float4 k4 = ld4(Kh + t * KP + ucol);
          kv[0] = k4.x, kv[1] = k4.y, kv[2] = k4.z, kv[3] = k4.w;
        } else {
          const float2 k2 = *reinterpret_cast<const float2*>(Kh + t * KP + ucol);
          kv[0] = k2.x, kv[1] = k2.y;
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          sreg[0][c] = fmaf(uw.x, kv[c], sreg[0][c]);
          sreg[1][c] = fmaf(uw.y, kv[c], sreg[1][c]);
          sreg[2][c] = fmaf(uw.z, kv[c], sreg[2][c]);
          sreg[3][c] = fmaf(uw.w, kv[c], sreg[3][c]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < NC; ++c) St[st_off(ur + i, ucol + c)] = sreg[i][c];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < NC; ++c) Sg[(size_t)(ur + i) * D + ucol + c] = sreg[i][c];
}

// ---------------------------------------------------------------- tensor-core sequential pass
// D = 128. One CTA per (stream, head, 64 value dims of the state): 16 warps
// for the elementwise work (four threads per TMEM lane r, 16 value columns
// each) and 1 warp that issues the copies and the tcgen05 MMAs. The state slice lives in TMEM, transposed
// (lane = key dim k, column = value dim v: ST[k][v] = S[v][k]), for the whole
// call. Per 64-token sub-chunk j, with its operand images from the prep
// kernel (KQ, TM) arriving by bulk copy one or two sub-chunks ahead:
//   MMA1  D1[t][v]      = sum_k [K^;Q^][t][k] S[v][k]       (K^ S0^T and Q^ S0^T)
//   (threads) RHS[t][v] = beta_t (v_t[v] - e^{G_t} D1[t][v]); O_in = scale e^{G_t} D1[64+t][v]
//   MMA2  D2[t][v]      = sum_s [T;M][t][s] RHS[s][v]      (U = T RHS and the intra-chunk outputs)
//   (threads) U~[t][v]  = e^{G_last - G_t} D2[t][v]; out = O_in + D2[64+t]
//   MMA3  ST[k][v]     += sum_t K^[t][k] U~[t][v]            (ST was scaled by e^{G_last})
//   (threads) the S image of the new state for the next MMA1; ST *= e^{G_last} of j + 1
// Every product is the three-term split product of bf16 operands:
// x = hi + lo, a.b ~ a_hi.b_hi + a_hi.b_lo + a_lo.b_hi with fp32 accumulation
// (about 2^-16 relative per product; a plain bf16 product has 2^-8). Images
// written by the threads (S, RHS, U~) are 128-byte-swizzled rows of 64
// values, read as MN-major operands; the K^ rows of KQ serve as the MN-major
// A operand of MMA3. Every wait is bounded (about 1 s); on expiry the CTA
// records a device error in the workspace header, drains and returns.
struct GdnTcSmem {
  static constexpr uint32_t kq = 0;                         // [2 buffers][hi, lo] KQ images
  static constexpr uint32_t tm = 4 * kImgKQ;                // [hi, lo] TM image
  static constexpr uint32_t st = tm + 2 * kImgTM;           // [hi, lo] S image, 128 x 64
  static constexpr uint32_t rhs = st + 2 * 16384;           // [hi, lo] RHS image, 64 x 64
  static constexpr uint32_t uu = rhs + 2 * 8192;            // [hi, lo] U~ image, 64 x 64
  static constexpr uint32_t bars = uu + 2 * 8192;
  static constexpr int B_KQ = 0, B_TM = 2, B_S = 3, B_D1 = 4, B_RHS = 5, B_D2 = 6, B_U = 7,
                       B_D3 = 8, B_G = 9, B_DR = 10;
  static constexpr int kNumBars = 11;
  static constexpr uint32_t misc = bars + kNumBars * 8;     // TMEM base, abort flags
  static constexpr uint32_t gs = misc + 16;                 // [2][64] gate prefix sums (log2)
  static constexpr uint32_t bs = gs + 2 * kCt * 4;          // [2][64] beta
  static constexpr uint32_t bytes = bs + 2 * kCt * 4;
  static_assert(bytes <= 232448, "exceeds 227 KB of shared memory per CTA");
};
constexpr int kTcSlice = 64;
// elementwise warps: warps w, w + 4, w + 8 and w + 12 share TMEM lanes
// 32 (w % 4) .. + 31 and take 16 value columns each of those rows (the
// elementwise phases are on the sequential chain: 16 warps shorten them
// against 4 or 8)
constexpr int kTcElemWarps = 16;
constexpr int kTcCols = kTcSlice / (kTcElemWarps / 4);   // values per thread
constexpr int kTcThreads = 32 * kTcElemWarps + 32;
static_assert(kTcCols == 32 || kTcCols == 16, "two or four threads per TMEM lane");

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* x) {
  if constexpr (N == 32)
    ptx::tmem_ld32(taddr, x);
  else
    ptx::tmem_ld16(taddr, x);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float* x) {
  if constexpr (N == 32)
    ptx::tmem_st32(taddr, x);
  else
    ptx::tmem_st16u(taddr, reinterpret_cast<const uint32_t*>(x));
}
constexpr uint64_t kTcTimeoutNs = 1000000000ull;
// a call of at least this many sub-chunks runs in two pieces (launch_gdn_t)
constexpr int kGdnSplitMin = 8;

// NV floats of row `row` of a single-panel image, from 16-byte column group
// c0 on, as bf16 hi and lo.
template <int NV>
__device__ __forceinline__ void put_row(unsigned char* sm, uint32_t hi_off, uint32_t lo_off,
                                        int row, int c0, const float* x) {
#pragma unroll
  for (int c = 0; c < NV / 8; ++c) {
    uint4 h, l;
    split8(x + 8 * c, h, l);
    const uint32_t off = sw128_off(row, c0 + c);
    *reinterpret_cast<uint4*>(sm + hi_off + off) = h;
    *reinterpret_cast<uint4*>(sm + lo_off + off) = l;
  }
}

template <int NV, typename T>
__device__ __forceinline__ void load_row(const T* src, float* x) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < NV / 8; ++i) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + 8 * i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
        x[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < NV / 4; ++i) {
      const float4 u = *reinterpret_cast<const float4*>(src + 4 * i);
      x[4 * i] = u.x, x[4 * i + 1] = u.y, x[4 * i + 2] = u.z, x[4 * i + 3] = u.w;
    }
  }
}

template <int NV, typename T>
__device__ __forceinline__ void store_row(T* dst, const float* x) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < NV / 8; ++i) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(x[8 * i + 2 * k], x[8 * i + 2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&b);
      }
      *reinterpret_cast<uint4*>(dst + 8 * i) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < NV / 4; ++i)
      *reinterpret_cast<float4*>(dst + 4 * i) =
          make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kTcThreads, 1) gdn_tc_kernel(const __grid_constant__ GdnParams p) {
  constexpr int D = 128;
  using L = GdnTcSmem;
  extern __shared__ __align__(1024) unsigned char smc[];
  int* status = reinterpret_cast<int*>(p.workspace);
  const uint32_t base = ptx::smem_u32(smc);
  if (base & 1023u) {  // 128-byte-swizzled images need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(status, kDeviceErrTimeout);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x, h = blockIdx.y, z = blockIdx.z, b = p.stream_of[z];
  const int H = p.H;
  const int64_t Tn = p.T;
  const int nsub = p.n_sub;
  // sub-chunks [j0, j0 + nl) of the call; barrier parities and buffers follow
  // the local index jl = j - j0 (every barrier starts at phase 0 in a launch)
  const int j0 = p.j_begin, nl = p.j_end - p.j_begin;
  const int vcol = slice * kTcSlice;
  // the next prep piece (if any) may start on the SMs this grid leaves free
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t bar0 = base + L::bars;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smc + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smc + L::misc + 4);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smc + L::misc + 8);
  float* Gs = reinterpret_cast<float*>(smc + L::gs);
  float* Bs = reinterpret_cast<float*>(smc + L::bs);
  if (!SA_BOUNDS(b >= 0 && b < p.batch && z < p.n_streams && vcol + kTcSlice <= D && j0 >= 0 &&
                     nl > 0 && p.j_end <= nsub,
                 3))
    return;

  if (tid == 0) {
    ptx::mbar_init(bar(L::B_KQ), 1);
    ptx::mbar_init(bar(L::B_KQ + 1), 1);
    ptx::mbar_init(bar(L::B_TM), 1);
    ptx::mbar_init(bar(L::B_S), 32 * kTcElemWarps);
    ptx::mbar_init(bar(L::B_D1), 1);
    ptx::mbar_init(bar(L::B_RHS), 32 * kTcElemWarps);
    ptx::mbar_init(bar(L::B_D2), 1);
    ptx::mbar_init(bar(L::B_U), 32 * kTcElemWarps);
    ptx::mbar_init(bar(L::B_D3), 1);
    ptx::mbar_init(bar(L::B_G), 64);
    ptx::mbar_init(bar(L::B_DR), 1);
    *abort_flag = 0;
    *no_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kTcElemWarps) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_st = tmem, t_d1 = tmem + 64, t_d2 = tmem + 128;
  // launched as a programmatic dependent of the prep: nothing the prep (or,
  // through it, the previous pass piece) writes is read before this point
  asm volatile("griddepcontrol.wait;" ::: "memory");
  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(status, kDeviceErrTimeout);
  };
  const unsigned char* images = reinterpret_cast<const unsigned char*>(p.workspace) + kWsHeader +
                                ((size_t)z * H + h) * (size_t)nsub * kImgBytes;

  if (warp == kTcElemWarps) {
    // ------------------------------------------------------------ copies + MMA issue
    if (lane == 0) {
      auto load_kq = [&](int jl) {
        const uint32_t dst = base + L::kq + (uint32_t)(jl & 1) * 2 * kImgKQ;
        const unsigned char* src = images + (size_t)(j0 + jl) * kImgBytes;
        ptx::mbar_arrive_expect_tx(bar(L::B_KQ + (jl & 1)), 2 * kImgKQ);
        for (uint32_t o = 0; o < 2 * kImgKQ; o += 16384)
          ptx::bulk_g2s(dst + o, src + o, 16384, bar(L::B_KQ + (jl & 1)));
      };
      auto load_tm = [&](int jl) {
        const unsigned char* src = images + (size_t)(j0 + jl) * kImgBytes + 2 * kImgKQ;
        ptx::mbar_arrive_expect_tx(bar(L::B_TM), 2 * kImgTM);
        for (uint32_t o = 0; o < 2 * kImgTM; o += 16384)
          ptx::bulk_g2s(base + L::tm + o, src + o, 16384, bar(L::B_TM));
      };
      constexpr uint32_t id_kk = ptx::idesc_bf16_f32_ab(128, kTcSlice, false, true);
      constexpr uint32_t id_mm = ptx::idesc_bf16_f32_ab(128, kTcSlice, true, true);
      // split-product term i: (A part, B part) = (hi, hi), (hi, lo), (lo, hi)
      constexpr uint32_t ta[3] = {0, 0, 1}, tb[3] = {0, 1, 0};
      // base descriptors of the fixed operand buffers (MN-major images have
      // their 64-column panels 16 KiB apart, rows 8 x 128 bytes per core group)
      const uint64_t d_st = ptx::sdesc_sw128(base + L::st, 16384, 1024);
      const uint64_t d_tm = ptx::sdesc_sw128(base + L::tm, 16, 1024);
      const uint64_t d_rhs = ptx::sdesc_sw128(base + L::rhs, 16384, 1024);
      const uint64_t d_uu = ptx::sdesc_sw128(base + L::uu, 16384, 1024);
      int kq_issued = 0, kq_done = 0, tm_issued = 0;
      load_kq(0);
      ++kq_issued;
      if (nl > 1) {
        load_kq(1);
        ++kq_issued;
      }
      load_tm(0);
      ++tm_issued;
      bool ok = true;
      for (int jl = 0; ok && jl < nl; ++jl) {
        const uint32_t par = (uint32_t)jl & 1;
        const uint32_t kqb = base + L::kq + (uint32_t)(jl & 1) * 2 * kImgKQ;
        if (!ptx::mbar_wait(bar(L::B_KQ + (jl & 1)), (uint32_t)(jl >> 1) & 1, abort_flag, kTcTimeoutNs) ||
            !ptx::mbar_wait(bar(L::B_S), par, abort_flag, kTcTimeoutNs)) {
          ok = false;
          break;
        }
        ++kq_done;
        ptx::tc_fence_after();
        // MMA1: [K^;Q^] (K-major, 2 panels of 64 key dims) x S image (MN-major)
        const uint64_t a1 = ptx::sdesc_sw128(kqb, 16, 1024);
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            ptx::umma_ss(t_d1,
                         ptx::sdesc_add(a1, ta[i] * kImgKQ + (uint32_t)(kk >> 2) * 16384 +
                                                (uint32_t)(kk & 3) * 32),
                         ptx::sdesc_add(d_st, tb[i] * 16384 + (uint32_t)kk * 2048), id_kk,
                         (i > 0 || kk > 0) ? 1u : 0u);
        ptx::umma_commit(bar(L::B_D1));
        if (!ptx::mbar_wait(bar(L::B_TM), par, abort_flag, kTcTimeoutNs) ||
            !ptx::mbar_wait(bar(L::B_RHS), par, abort_flag, kTcTimeoutNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // MMA2: [T;M] (K-major, one panel of 64 tokens) x RHS image (MN-major)
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int kk = 0; kk < kCt / 16; ++kk)
            ptx::umma_ss(t_d2, ptx::sdesc_add(d_tm, ta[i] * kImgTM + (uint32_t)kk * 32),
                         ptx::sdesc_add(d_rhs, tb[i] * 8192 + (uint32_t)kk * 2048), id_kk,
                         (i > 0 || kk > 0) ? 1u : 0u);
        ptx::umma_commit(bar(L::B_D2));
        // the TM buffer is free once MMA2 has read it
        if (!ptx::mbar_wait(bar(L::B_D2), par, abort_flag, kTcTimeoutNs)) {
          ok = false;
          break;
        }
        if (jl + 1 < nl) {
          load_tm(jl + 1);
          ++tm_issued;
        }
        if (!ptx::mbar_wait(bar(L::B_U), par, abort_flag, kTcTimeoutNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // MMA3: ST += K^ (the key rows of KQ as the MN-major A: 2 panels of 64
        // key dims LBO apart, 64 token rows) x U~ image (MN-major)
        const uint64_t a3 = ptx::sdesc_sw128(kqb, 16384, 1024);
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int kk = 0; kk < kCt / 16; ++kk)
            ptx::umma_ss(t_st, ptx::sdesc_add(a3, ta[i] * kImgKQ + (uint32_t)kk * 2048),
                         ptx::sdesc_add(d_uu, tb[i] * 8192 + (uint32_t)kk * 2048), id_mm, 1u);
        ptx::umma_commit(bar(L::B_D3));
        // the KQ buffer of jl is free once MMA3 has read it
        if (jl + 2 < nl) {
          if (!ptx::mbar_wait(bar(L::B_D3), par, abort_flag, kTcTimeoutNs)) {
            ok = false;
            break;
          }
          load_kq(jl + 2);
          ++kq_issued;
        }
      }
      if (!ok) fail();
      // drain: the copies this thread issued have landed and its MMAs are done
      for (int jj = kq_done; jj < kq_issued; ++jj)
        ptx::mbar_wait(bar(L::B_KQ + (jj & 1)), (uint32_t)(jj >> 1) & 1, no_abort, kTcTimeoutNs);
      if (tm_issued > 0)
        ptx::mbar_wait(bar(L::B_TM), (uint32_t)(tm_issued - 1) & 1, no_abort, kTcTimeoutNs);
      ptx::umma_commit(bar(L::B_DR));
      ptx::mbar_wait(bar(L::B_DR), 0, no_abort, kTcTimeoutNs);
    }
  } else {
    // ------------------------------------------------------------ elementwise
    // TMEM lane r: 0..63 key/U rows, 64..127 query/output rows; also key dim r
    // of ST. Columns [cb, cb + 32) of the slice.
    const int r = (warp & 3) * 32 + lane;
    const int grp = warp >> 2;   // column group
    const int cb = grp * kTcCols;
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
    const T* v = static_cast<const T*>(p.v);
    T* out = static_cast<T*>(p.out);
    const size_t tok_stride = (size_t)H * D;
    const size_t bh0 = (size_t)b * (size_t)Tn * tok_stride + (size_t)h * D + vcol + cb;
    const size_t g0 = (size_t)b * (size_t)Tn * H + h;
    float* Sg = p.state + ((size_t)b * H + h) * D * D;   // [v][k]
    auto gates = [&](int jl) {
      // threads 0..63: prefix sums of g log2(e) and beta of sub-chunk j0 + jl
      if (grp == 0 && r < kCt) {
        const int64_t t = (int64_t)(j0 + jl) * kCt + r;
        const bool in = t < Tn;
        gate_scan(in ? p.g[g0 + (size_t)t * H] : 0.f, in ? p.beta[g0 + (size_t)t * H] : 0.f,
                  Gs + (jl & 1) * kCt, Bs + (jl & 1) * kCt, r, lane);
        ptx::mbar_arrive(bar(L::B_G));
      }
    };
    auto gcum = [&](int jl, int t) -> float {
      const float* G = Gs + (jl & 1) * kCt;
      return G[t] + (t >= 32 ? G[31] : 0.f);
    };
    bool ok = true;
    // prologue: the gates of sub-chunk j0, the S image of the initial state and
    // ST = e^{G_last} S
    gates(0);
    if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_G), 0, abort_flag, kTcTimeoutNs))) ok = false;
    if (ok) {
      float x[kTcCols];
#pragma unroll
      for (int i = 0; i < kTcCols; ++i) x[i] = Sg[(size_t)(vcol + cb + i) * D + r];
      put_row<kTcCols>(smc, L::st, L::st + 16384, r, cb / 8, x);
      const float dec = ptx::ex2(gcum(0, kCt - 1));
#pragma unroll
      for (int i = 0; i < kTcCols; ++i) x[i] *= dec;
      tmem_st_cols<kTcCols>(t_st + lane_off + cb, x);
      ptx::tmem_wait_st();
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_S));
    }
    for (int jl = 0; ok && jl < nl; ++jl) {
      const uint32_t par = (uint32_t)jl & 1;
      const int64_t t0 = (int64_t)(j0 + jl) * kCt;
      const int tr = r & (kCt - 1);               // token of this row
      const bool tok_in = t0 + tr < Tn;
      // values of this sub-chunk's token (key rows), loaded while MMA1 runs
      float vv[kTcCols];
      if (r < kCt) {
        if (tok_in) {
          load_row<kTcCols>(v + bh0 + (size_t)(t0 + tr) * tok_stride, vv);
        } else {
#pragma unroll
          for (int i = 0; i < kTcCols; ++i) vv[i] = 0.f;
        }
      }
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_D1), par, abort_flag, kTcTimeoutNs))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float x[kTcCols];
      tmem_ld_cols<kTcCols>(t_d1 + lane_off + cb, x);
      ptx::tmem_wait_ld();
      const float eg = ptx::ex2(gcum(jl, tr));
      if (r < kCt) {
        const float bt = Bs[(jl & 1) * kCt + tr];
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) vv[i] = bt * (vv[i] - eg * x[i]);
        put_row<kTcCols>(smc, L::rhs, L::rhs + 8192, tr, cb / 8, vv);
      } else {
        const float sc = p.scale * eg;
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) vv[i] = sc * x[i];   // (query rows: the inter-chunk output)
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_RHS));
      // the gates of the next sub-chunk, while MMA2 runs
      if (jl + 1 < nl) gates(jl + 1);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_D2), par, abort_flag, kTcTimeoutNs))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      tmem_ld_cols<kTcCols>(t_d2 + lane_off + cb, x);
      ptx::tmem_wait_ld();
      if (r < kCt) {
        const float wt = ptx::ex2(gcum(jl, kCt - 1) - gcum(jl, tr));
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) x[i] *= wt;
        put_row<kTcCols>(smc, L::uu, L::uu + 8192, tr, cb / 8, x);
      } else if (tok_in) {
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) x[i] += vv[i];
        store_row<kTcCols>(out + bh0 + (size_t)(t0 + tr) * tok_stride, x);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_U));
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_D3), par, abort_flag, kTcTimeoutNs))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // the state after sub-chunk j0 + jl (key dim r, this thread's value dims)
      tmem_ld_cols<kTcCols>(t_st + lane_off + cb, x);
      ptx::tmem_wait_ld();
      if (jl + 1 < nl) {
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_G), (uint32_t)(jl + 1) & 1, abort_flag,
                                                    kTcTimeoutNs))) {
          ok = false;
          break;
        }
        put_row<kTcCols>(smc, L::st, L::st + 16384, r, cb / 8, x);
        const float dec = ptx::ex2(gcum(jl + 1, kCt - 1));
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) x[i] *= dec;
        tmem_st_cols<kTcCols>(t_st + lane_off + cb, x);
        ptx::tmem_wait_st();
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_S));
      } else {
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) Sg[(size_t)(vcol + cb + i) * D + r] = x[i];
      }
    }
    if (!ok) fail();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kTcElemWarps) ptx::tmem_dealloc(tmem, 256);
}

// D = 128: the prep kernel writes the operand images and the tensor-core
// kernel runs the sequential pass; D = 64: fp32 T and M and the CUDA-core
// sequential kernel.
template <int D, typename T>
cudaError_t launch_gdn_t(const GdnParams& p, cudaStream_t st) {
  constexpr bool kTc = D == 128;
  constexpr size_t smem = kTc ? GdnTcSmem::bytes : GdnSmem<D, T>::bytes;
  constexpr size_t psmem = kTc ? (size_t)GdnPrepTcSmem::bytes : GdnPrepSmem<D>::bytes;
  static unsigned configured = 0;   // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e;
    if constexpr (kTc)
      e = cudaFuncSetAttribute(gdn_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    else
      e = cudaFuncSetAttribute(gdn_chunk_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (e == cudaSuccess) {
      if constexpr (kTc)
        e = cudaFuncSetAttribute(gdn_prep_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)psmem);
      else
        e = cudaFuncSetAttribute(gdn_prep_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)psmem);
    }
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  if constexpr (!kTc) {
    GdnParams q = p;
    q.j_begin = 0;
    q.j_end = p.n_sub;
    q.pdl_wait = 0;
    gdn_prep_kernel<D, T><<<dim3(p.n_sub, p.H, p.n_streams), kGdnThreads, psmem, st>>>(q);
    gdn_chunk_kernel<D, T><<<dim3(D / kDvs, p.H, p.n_streams), kGdnThreads, smem, st>>>(q);
    return cudaGetLastError();
  } else {
    // The sequential pass occupies one SM per (stream, head, value slice) and
    // leaves the others idle, while the prep of every sub-chunk must precede
    // the pass that reads it. So the call runs in two pieces of sub-chunks:
    // the second prep is launched as a programmatic dependent of the first
    // pass and runs on the idle SMs while that pass runs (it reads only the
    // inputs and writes only its own sub-chunks' images). Every pass is a
    // programmatic dependent of its prep: it runs its set-up once the prep's
    // CTAs have done their work and reads nothing before the prep grid has
    // completed, which for the second prep is after the first pass (see
    // gdn_prep_tc_kernel); so the second pass continues from the state the
    // first one stored.
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // Two pieces: each further piece adds a launch hand-off of 5-7 us
    // (measured on the 512p call, 32 sub-chunks: 0.161 ms in two halves,
    // 0.169 in four pieces, 0.186 in eight, 0.177 unsplit). The first piece
    // takes 3/8 of the sub-chunks: its prep is exposed, while the larger
    // second prep still fits beside the first pass (first pieces of 10, 12,
    // 14 and 16 of 32: 0.166, 0.158, 0.162 and 0.162 ms). Split only when the
    // pass leaves at least half of the SMs to the prep.
    const int pass_ctas = (D / kTcSlice) * p.H * p.n_streams;
    const int first = (p.n_sub >= kGdnSplitMin && 2 * pass_ctas <= sms) ? (3 * p.n_sub + 7) / 8
                                                                        : p.n_sub;
    for (int jb = 0; jb < p.n_sub;) {
      GdnParams q = p;
      q.j_begin = jb;
      q.j_end = jb == 0 ? first : p.n_sub;
      jb = q.j_end;
      q.pdl_wait = q.j_begin > 0;
      const dim3 pg((unsigned)(q.j_end - q.j_begin), (unsigned)p.H, (unsigned)p.n_streams);
      if (q.j_begin == 0) {
        gdn_prep_tc_kernel<T><<<pg, kGdnThreads, psmem, st>>>(q);
      } else {
        cudaLaunchConfig_t lc = {};
        lc.gridDim = pg;
        lc.blockDim = dim3(kGdnThreads);
        lc.dynamicSmemBytes = psmem;
        lc.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = at;
        lc.numAttrs = 1;
        e = cudaLaunchKernelEx(&lc, gdn_prep_tc_kernel<T>, q);
        if (e != cudaSuccess) return e;
      }
      {
        // the pass as a programmatic dependent of its prep: its set-up and
        // launch overlap the end of the prep (measured 0.150 against 0.157
        // ms per 512p call)
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(D / kTcSlice, p.H, p.n_streams);
        lc.blockDim = dim3(kTcThreads);
        lc.dynamicSmemBytes = smem;
        lc.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = at;
        lc.numAttrs = 1;
        e = cudaLaunchKernelEx(&lc, gdn_tc_kernel<T>, q);
      }
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
}

}  // namespace

size_t gdn_workspace_bytes(int B, int H, int D, int64_t T) {
  const size_t per = D == 128 ? (size_t)kImgBytes : (size_t)kTpFloats * sizeof(float);
  return kWsHeader + (size_t)B * (size_t)H * (size_t)((T + kCt - 1) / kCt) * per;
}

size_t gdn_smem_bytes(int D, int dtype) {
  if (D == 64) return dtype == SA_BF16 ? GdnSmem<64, __nv_bfloat16>::bytes : GdnSmem<64, float>::bytes;
  return dtype == SA_BF16 ? GdnSmem<128, __nv_bfloat16>::bytes : GdnSmem<128, float>::bytes;
}

cudaError_t launch_gdn(const GdnParams& p, int D, int dtype, cudaStream_t st) {
  if (p.n_streams <= 0 || p.T <= 0) return cudaSuccess;
  if (D == 64)
    return dtype == SA_BF16 ? launch_gdn_t<64, __nv_bfloat16>(p, st) : launch_gdn_t<64, float>(p, st);
  return dtype == SA_BF16 ? launch_gdn_t<128, __nv_bfloat16>(p, st) : launch_gdn_t<128, float>(p, st);
}

}  // namespace sa
