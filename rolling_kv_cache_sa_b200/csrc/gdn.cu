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
//  * gdn_prep_kernel: one CTA per (stream, head, sub-chunk), all independent.
//    It computes what depends only on K, Q, g and beta -- T = (I + L)^-1 and
//    M = scale P T -- and writes both (64 x 64 fp32 each) to the workspace.
//    With U = T RHS, the intra-chunk part of the outputs is P U = M RHS, so the
//    sequential pass gets U and the outputs from one sweep over RHS.
//  * gdn_chunk_kernel: one CTA per (stream, head, 32 value rows of the state).
//    Rows of S evolve independently, so a CTA owns its 32 x D slice of the
//    state for the whole call (in registers, with a copy in shared memory for
//    the products that read it by rows) and walks the sub-chunks in order,
//    loading each one's T and P from the workspace one sub-chunk ahead.
// All arithmetic is fp32 on the CUDA cores.
#include <cuda_bf16.h>

#include "internal.h"

namespace sa {
namespace {

constexpr int kCt = 64;         // tokens per sub-chunk
constexpr int kDvs = 32;        // state rows (value dims) per CTA
constexpr int kGdnThreads = 256;
constexpr int kLp = kCt + 4;    // row pitch of the 64 x 64 matrices (16-byte rows)
constexpr int kVp = kDvs + 4;   // row pitch of the 64 x 32 matrices (16-byte rows)
constexpr int kTpFloats = 2 * kCt * kCt;   // T and P of one sub-chunk in the workspace
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

// One CTA per (stream, head, sub-chunk): T = (I + L)^-1 and M = scale P T of
// the sub-chunk into the workspace, both [64][64] row-major, zero above the
// diagonal.
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

  // ---- M = P T (lower triangular; L is no longer needed, M takes its place).
  // The outputs' intra-chunk part is P U = P T RHS = M RHS. Thread (ty, tx)
  // takes rows ty + 16a and columns tx + 16b, b <= a.
  {
    float* Mm = Lm;
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
    int i = 0;   // (the last reads of L were in the merges, before the barrier above)
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

  // ---- T and M to the workspace, zero above the diagonal
  float* dst = p.workspace + (((size_t)z * H + h) * (size_t)p.n_sub + (size_t)j) * kTpFloats;
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
  const float* wsp = p.workspace + ((size_t)blockIdx.z * H + h) * (size_t)p.n_sub * kTpFloats;
  auto prefetch_tp = [&](int64_t j) {
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

template <int D, typename T>
cudaError_t launch_gdn_t(const GdnParams& p, cudaStream_t st) {
  constexpr size_t smem = GdnSmem<D, T>::bytes;
  constexpr size_t psmem = GdnPrepSmem<D>::bytes;
  static unsigned configured = 0;   // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(gdn_chunk_kernel<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn_prep_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)psmem);
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  gdn_prep_kernel<D, T><<<dim3(p.n_sub, p.H, p.n_streams), kGdnThreads, psmem, st>>>(p);
  gdn_chunk_kernel<D, T><<<dim3(D / kDvs, p.H, p.n_streams), kGdnThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t gdn_workspace_bytes(int B, int H, int64_t T) {
  return (size_t)B * (size_t)H * (size_t)((T + kCt - 1) / kCt) * kTpFloats * sizeof(float);
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
