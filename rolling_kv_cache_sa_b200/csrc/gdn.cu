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
// The kernel runs the chunkwise form of that recurrence (the WY form of Yang
// et al., "Parallelizing Linear Transformers with the Delta Rule over
// Sequence Length", NeurIPS 2024) on sub-chunks of 64 tokens. With S0 the
// state before a sub-chunk and G_t = g_1 + ... + g_t inside it, the
// corrected values u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t) solve
//     (I + L) U = diag(beta) (V - diag(e^G) K S0^T),
//     L_ts = beta_t e^(G_t - G_s) k_t . k_s  (s < t),
// and then
//     o_t   = scale (e^(G_t) S0 q_t + sum_{s<=t} e^(G_t - G_s) (q_t . k_s) u_s)
//     S_end = e^(G_last) S0 + sum_s e^(G_last - G_s) u_s k_s^T.
// (I + L)^-1 is unit lower triangular: its 16 x 16 diagonal blocks come from
// forward substitution, and two merges use
//     [A 0; C B]^-1 = [A^-1 0; -B^-1 C A^-1  B^-1].
//
// Grid: one CTA per (active stream, head, 32 value rows of the state). Rows of
// S evolve independently, so a CTA owns its 32 x D slice of the state for the
// whole call (in registers, with a copy in shared memory for the products
// that read it by rows); the quantities that depend only on K, Q, g and beta
// (the Gram matrices and (I + L)^-1) are recomputed by each of the D/32 CTAs
// of a head. All arithmetic is fp32 on the CUDA cores.
#include <cuda_bf16.h>

#include "internal.h"

namespace sa {
namespace {

constexpr int kCt = 64;         // tokens per sub-chunk
constexpr int kDvs = 32;        // state rows (value dims) per CTA
constexpr int kGdnThreads = 256;
constexpr int kLp = kCt + 1;    // row pitch of the 64 x 64 matrices
constexpr int kVp = kDvs + 1;   // row pitch of the 64 x 32 matrices
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory layout in floats. Rows of K^, Q^ and S have pitch D + 4: a
// multiple of 4 (16-byte aligned rows) whose 16-byte groups step by an odd
// count, so float4 reads of consecutive rows fall in different bank groups.
template <int D>
struct GdnSmem {
  static constexpr int KP = D + 4;
  static constexpr int kh = 0;                    // [64][KP] normalised keys
  static constexpr int qh = kh + kCt * KP;        // [64][KP] normalised queries
  static constexpr int st = qh + kCt * KP;        // [32][KP] state slice S0
  static constexpr int lm = st + kDvs * KP;       // [64][65] L (strictly lower)
  static constexpr int pm = lm + kCt * kLp;       // [64][65] scale e^(G_t-G_s) q_t.k_s (s <= t)
  static constexpr int tm = pm + kCt * kLp;       // [64][65] (I + L)^-1 (lower)
  static constexpr int xm = tm + kCt * kLp;       // [32][33] merge scratch
  static constexpr int rv = xm + 32 * 33;         // [64][33] v slice, then the right-hand side
  static constexpr int uv = rv + kCt * kVp;       // [64][33] corrected values u
  static constexpr int gs = uv + kCt * kVp;       // [64] in-warp prefix sums of g log2(e)
  static constexpr int bs = gs + kCt;             // [64] beta
  static constexpr int ws = bs + kCt;             // [64] e^(G_last - G_t)
  static constexpr int total = ws + kCt;
  static constexpr size_t bytes = (size_t)total * sizeof(float);
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

__device__ __forceinline__ float ld_in(const float* p, size_t i) { return __ldg(p + i); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_out(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

template <int D, typename T>
__global__ void __launch_bounds__(kGdnThreads, 1) gdn_chunk_kernel(const __grid_constant__ GdnParams p) {
  using L = GdnSmem<D>;
  constexpr int KP = L::KP;
  constexpr int NE = D / 32;   // elements of a row per lane
  constexpr int NJ = D / 32;   // float4 groups of state per thread
  extern __shared__ __align__(16) float sm[];
  float* Kh = sm + L::kh;
  float* Qh = sm + L::qh;
  float* St = sm + L::st;
  float* Lm = sm + L::lm;
  float* Pm = sm + L::pm;
  float* Tm = sm + L::tm;
  float* Xm = sm + L::xm;
  float* Rv = sm + L::rv;
  float* Uv = sm + L::uv;
  float* Gs = sm + L::gs;
  float* Bs = sm + L::bs;
  float* Ws = sm + L::ws;

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

  // Cumulative log2 decay through token t of the sub-chunk (warp 1's prefix
  // sums lack warp 0's total, added here).
  auto gcum = [&](int t) -> float { return Gs[t] + (t >= 32 ? Gs[31] : 0.f); };

  // State rows this thread updates: row uc, columns uj + 32 m (+0..3).
  const int uc = warp * 4 + (lane >> 3);
  const int uj = 4 * (lane & 7);
  float4 sreg[NJ];
#pragma unroll
  for (int m = 0; m < NJ; ++m) {
    sreg[m] = *reinterpret_cast<const float4*>(Sg + (size_t)uc * D + uj + 32 * m);
    st4(St + uc * KP + uj + 32 * m, sreg[m]);
  }

  for (int64_t t0 = 0; t0 < Tn; t0 += kCt) {
    const int n = (int)(Tn - t0 < kCt ? Tn - t0 : kCt);

    // ---- normalised key and query rows, the value slice, the gates
    for (int r = warp; r < kCt; r += 8) {
      float kx[NE], qx[NE];
      float sk = 0.f, sq = 0.f;
      const size_t off = bh0 + (size_t)(t0 + r) * tok_stride;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        kx[e] = r < n ? ld_in(k, off + lane + 32 * e) : 0.f;
        qx[e] = r < n ? ld_in(q, off + lane + 32 * e) : 0.f;
        sk = fmaf(kx[e], kx[e], sk);
        sq = fmaf(qx[e], qx[e], sq);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float ik = sk > 0.f ? rsqrtf(sk) : 0.f;
      const float iq = sq > 0.f ? rsqrtf(sq) : 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        Kh[r * KP + lane + 32 * e] = kx[e] * ik;
        Qh[r * KP + lane + 32 * e] = qx[e] * iq;
      }
      Rv[r * kVp + lane] = r < n ? ld_in(v, off + vcol + lane) : 0.f;
    }
    if (tid < kCt) {   // warps 0 and 1
      const bool ok = tid < n;
      float gl = ok ? p.g[g0 + (size_t)(t0 + tid) * H] * kLog2e : 0.f;
      Bs[tid] = ok ? p.beta[g0 + (size_t)(t0 + tid) * H] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, gl, o);
        if (lane >= o) gl += y;
      }
      Gs[tid] = gl;
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
    // ---- K^ S0^T and Q^ S0^T for this CTA's rows: thread (warp, lane) takes
    // tokens warp + 8a and state row lane. The right-hand side
    // beta_t (v_t - e^(G_t) (S0 k_t)) replaces v in Rv; the inter-chunk part of
    // the output stays in registers.
    float oin[8];
    {
      float aks[8], aqs[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) aks[a] = aqs[a] = 0.f;
      const float* srow = St + lane * KP;
#pragma unroll 2
      for (int d = 0; d < D; d += 4) {
        const float4 s4 = ld4(srow + d);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          aks[a] = dot4(ld4(Kh + (warp + 8 * a) * KP + d), s4, aks[a]);
          aqs[a] = dot4(ld4(Qh + (warp + 8 * a) * KP + d), s4, aqs[a]);
        }
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int t = warp + 8 * a;
        const float gam = ex2f(gcum(t));
        Rv[t * kVp + lane] = Bs[t] * (Rv[t * kVp + lane] - gam * aks[a]);
        oin[a] = p.scale * gam * aqs[a];
      }
    }
    __syncthreads();

    // ---- diagonal 16 x 16 blocks of (I + L)^-1: thread (blk, j) solves for
    // column j of its block; the end-state weights e^(G_last - G_t)
    if (tid < 64) {
      const int r0 = (tid >> 4) * 16, j = tid & 15;
      float x[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < t; ++s) acc = fmaf(Lm[(r0 + t) * kLp + r0 + s], x[s], acc);
        x[t] = t < j ? 0.f : (t == j ? 1.f : -acc);
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) Tm[(r0 + t) * kLp + r0 + j] = x[t];
    } else if (tid < 64 + kCt) {
      const int t = tid - 64;
      Ws[t] = ex2f(gcum(kCt - 1) - gcum(t));
    }
    __syncthreads();

    // ---- merge to 32 x 32 blocks (rows r0+16.., columns r0.., r0 = 0, 32):
    // X = L21 T11, then T21 = -T22 X
    for (int e = tid; e < 512; e += kGdnThreads) {
      const int pp = e >> 8, i = (e >> 4) & 15, j = e & 15, r0 = pp * 32;
      float acc = 0.f;
      for (int s = j; s < 16; ++s)
        acc = fmaf(Lm[(r0 + 16 + i) * kLp + r0 + s], Tm[(r0 + s) * kLp + r0 + j], acc);
      Xm[pp * 272 + i * 17 + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 512; e += kGdnThreads) {
      const int pp = e >> 8, i = (e >> 4) & 15, j = e & 15, r0 = pp * 32;
      float acc = 0.f;
      for (int s = 0; s <= i; ++s)
        acc = fmaf(Tm[(r0 + 16 + i) * kLp + r0 + 16 + s], Xm[pp * 272 + s * 17 + j], acc);
      Tm[(r0 + 16 + i) * kLp + r0 + j] = -acc;
    }
    __syncthreads();
    // ---- merge to the full 64 x 64 inverse (rows 32.., columns 0..31)
    for (int e = tid; e < 1024; e += kGdnThreads) {
      const int i = e >> 5, j = e & 31;
      float acc = 0.f;
      for (int s = j; s < 32; ++s) acc = fmaf(Lm[(32 + i) * kLp + s], Tm[s * kLp + j], acc);
      Xm[i * 33 + j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += kGdnThreads) {
      const int i = e >> 5, j = e & 31;
      float acc = 0.f;
      for (int s = 0; s <= i; ++s) acc = fmaf(Tm[(32 + i) * kLp + 32 + s], Xm[s * 33 + j], acc);
      Tm[(32 + i) * kLp + j] = -acc;
    }
    __syncthreads();

    // ---- corrected values U = (I + L)^-1 RHS (tokens warp + 8a, row lane)
    {
      float acc[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) acc[a] = 0.f;
      for (int s = 0; s < n; ++s) {
        const float r = Rv[s * kVp + lane];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int t = warp + 8 * a;
          if (s <= t) acc[a] = fmaf(Tm[t * kLp + s], r, acc[a]);
        }
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) Uv[(warp + 8 * a) * kVp + lane] = acc[a];
    }
    __syncthreads();

    // ---- outputs: inter-chunk part + intra-chunk part P U
    {
      float acc[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) acc[a] = oin[a];
      for (int s = 0; s < n; ++s) {
        const float u = Uv[s * kVp + lane];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int t = warp + 8 * a;
          if (s <= t) acc[a] = fmaf(Pm[t * kLp + s], u, acc[a]);
        }
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int t = warp + 8 * a;
        if (t < n) st_out(out, bh0 + (size_t)(t0 + t) * tok_stride + vcol + lane, acc[a]);
      }
    }
    // ---- state: S = e^(G_last) S0 + sum_t e^(G_last - G_t) u_t k_t^T
    {
      const float dec = ex2f(gcum(kCt - 1));
#pragma unroll
      for (int m = 0; m < NJ; ++m) {
        sreg[m].x *= dec;
        sreg[m].y *= dec;
        sreg[m].z *= dec;
        sreg[m].w *= dec;
      }
      for (int t = 0; t < n; ++t) {
        const float uw = Uv[t * kVp + uc] * Ws[t];
#pragma unroll
        for (int m = 0; m < NJ; ++m) {
          const float4 k4 = ld4(Kh + t * KP + uj + 32 * m);
          sreg[m].x = fmaf(uw, k4.x, sreg[m].x);
          sreg[m].y = fmaf(uw, k4.y, sreg[m].y);
          sreg[m].z = fmaf(uw, k4.z, sreg[m].z);
          sreg[m].w = fmaf(uw, k4.w, sreg[m].w);
        }
      }
#pragma unroll
      for (int m = 0; m < NJ; ++m) st4(St + uc * KP + uj + 32 * m, sreg[m]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < NJ; ++m)
    *reinterpret_cast<float4*>(Sg + (size_t)uc * D + uj + 32 * m) = sreg[m];
}

template <int D, typename T>
cudaError_t launch_gdn_t(const GdnParams& p, cudaStream_t st) {
  constexpr size_t smem = GdnSmem<D>::bytes;
  static unsigned configured = 0;   // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(gdn_chunk_kernel<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  const dim3 grid(D / kDvs, p.H, p.n_streams);
  gdn_chunk_kernel<D, T><<<grid, kGdnThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t gdn_smem_bytes(int D) { return D == 64 ? GdnSmem<64>::bytes : GdnSmem<128>::bytes; }

cudaError_t launch_gdn(const GdnParams& p, int D, int dtype, cudaStream_t st) {
  if (p.n_streams <= 0 || p.T <= 0) return cudaSuccess;
  if (D == 64)
    return dtype == SA_BF16 ? launch_gdn_t<64, __nv_bfloat16>(p, st) : launch_gdn_t<64, float>(p, st);
  return dtype == SA_BF16 ? launch_gdn_t<128, __nv_bfloat16>(p, st) : launch_gdn_t<128, float>(p, st);
}

}  // namespace sa
