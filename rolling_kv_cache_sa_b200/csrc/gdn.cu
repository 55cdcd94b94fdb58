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
// Both run on the tensor core: gdn_prep_tc_kernel forms the Gram matrices
// with tcgen05 MMAs and writes bf16 hi/lo operand images of K^, Q^, T and M;
// gdn_tc_kernel keeps a 64-column state slice in TMEM (both described where
// they are defined). D = 64 uses the same kernels with the key dims of the
// images and of the state in TMEM padded to 128 with zeros, which the
// products carry through unchanged (measured 146 us per call at B = 1,
// H = 24, 2,048 tokens, against 336 us for an fp32 CUDA-core version).
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
constexpr int kGdnThreads = 256;
constexpr int kLp = kCt + 4;    // row pitch of the 64 x 64 matrices (16-byte rows)
// The workspace starts with a 1 KiB header holding the call's device status
// word (bounded waits); the per-sub-chunk blocks follow.
constexpr size_t kWsHeader = 1024;
// Per sub-chunk the prep kernel writes the operand images of the sequential
// kernel's MMAs, bf16, each value x as hi = bf16(x) and lo = bf16(x - hi),
// in the 128-byte-swizzled layout the
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

// Four consecutive input elements (16 bytes of fp32 or 8 of bf16) as floats.
__device__ __forceinline__ float4 ld_raw4(const float* p) { return ld4(p); }
__device__ __forceinline__ float4 ld_raw4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
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

// Prep (D = 64 or 128): one CTA per (stream, head,
// sub-chunk), computing T = (I + L)^-1 and M = scale P T, with the Gram
// matrices on the tensor core. The normalised
// key and query rows are split into bf16 hi and lo and written once, as the
// KQ operand image, to shared memory and to the workspace; one thread issues
// [K^;Q^] K^T (128 x 64, fp32 in TMEM) as the three-term split product over
// that image (the product the sequential pass uses for its own contractions,
// about 2^-16 relative per term); the threads read it back and form L and P
// (key rows and query rows of the product). Then T, M and the TM image.
template <int DI, typename T>
__device__ __forceinline__ void prep_tc_body(const GdnParams& p) {
  constexpr int D = 128;   // image width: head dims past DI are zero
  static_assert(DI == 64 || DI == 128, "head dim 64 or 128");
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
  const size_t tok_stride = (size_t)H * DI;
  const size_t row0 = ((size_t)b * (size_t)Tn + (size_t)t0) * tok_stride + (size_t)h * DI;
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
      if (r < n && 4 * lane < DI) {
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

template <int DI, typename T>
__global__ void __launch_bounds__(kGdnThreads, kPrepTcCtasPerSm)
    gdn_prep_tc_kernel(const __grid_constant__ GdnParams p) {
  prep_tc_body<DI, T>(p);
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

// ---------------------------------------------------------------- tensor-core sequential pass
// D = 64 or 128. One CTA per (stream, head, 64 value dims of the state): 16
// warps for the elementwise work (four threads per TMEM lane r, 16 value
// columns each) and 1 warp that issues the copies and the tcgen05 MMAs. The
// state slice lives in TMEM, transposed (lane = key dim k, column = value dim
// v: ST[k][v] = S[v][k]), for the whole launch; a launch walks the sub-chunk
// range [j_begin, j_end) of the call (a call may run in two pieces, see
// launch_gdn_t) and loads and stores the state in global memory at its ends.
// Per 64-token sub-chunk j, with its operand images from the prep kernel (KQ,
// TM) arriving by bulk copy one or two sub-chunks ahead:
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

template <int DI, typename T>
__global__ void __launch_bounds__(kTcThreads, 1) gdn_tc_kernel(const __grid_constant__ GdnParams p) {
  constexpr int D = 128;   // key dims of the images and of ST in TMEM (past DI: zero)
  static_assert(DI == 64 || DI == 128, "head dim 64 or 128");
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
  if (!SA_BOUNDS(b >= 0 && b < p.batch && z < p.n_streams && vcol + kTcSlice <= DI && j0 >= 0 &&
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
    const size_t tok_stride = (size_t)H * DI;
    const size_t bh0 = (size_t)b * (size_t)Tn * tok_stride + (size_t)h * DI + vcol + cb;
    const size_t g0 = (size_t)b * (size_t)Tn * H + h;
    float* Sg = p.state + ((size_t)b * H + h) * DI * DI;   // [v][k]
    const bool key_in = r < DI;   // ST lanes past DI stay zero
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
      // (from L2: the state was written by the previous pass piece or call,
      // whose completion this grid sees through the launch chain)
      for (int i = 0; i < kTcCols; ++i)
        x[i] = key_in ? __ldcg(Sg + (size_t)(vcol + cb + i) * DI + r) : 0.f;
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
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_RHS));
      } else {
        // query rows: MMA2 reads only the key rows' image, so they arrive first
        // and form their inter-chunk outputs (registers) while MMA2 runs
        // (0.1485 against 0.1496 ms per 512p call)
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_RHS));
        const float sc = p.scale * eg;
#pragma unroll
        for (int i = 0; i < kTcCols; ++i) vv[i] = sc * x[i];   // (query rows: the inter-chunk output)
      }
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
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_U));
      } else {
        // query rows: MMA3 reads only the key rows' image, so they arrive
        // before storing their outputs (the stores then overlap MMA3 instead
        // of delaying its start; measured 0.1497 against 0.1509 ms per 512p
        // call)
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_U));
        if (tok_in) {
#pragma unroll
          for (int i = 0; i < kTcCols; ++i) x[i] += vv[i];
          store_row<kTcCols>(out + bh0 + (size_t)(t0 + tr) * tok_stride, x);
        }
      }
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
        for (int i = 0; i < kTcCols; ++i)
          if (key_in) Sg[(size_t)(vcol + cb + i) * DI + r] = x[i];
      }
    }
    if (!ok) fail();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kTcElemWarps) ptx::tmem_dealloc(tmem, 256);
}

// The prep kernel writes the operand images and the tensor-core kernel runs
// the sequential pass (D = 64 through the same kernels, the key dims of the
// images and of the state in TMEM padded to 128 with zeros).
template <int D, typename T>
cudaError_t launch_gdn_t(const GdnParams& p, cudaStream_t st) {
  constexpr size_t smem = GdnTcSmem::bytes;
  constexpr size_t psmem = GdnPrepTcSmem::bytes;
  static unsigned configured = 0;   // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(gdn_tc_kernel<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn_prep_tc_kernel<D, T>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  {
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
        gdn_prep_tc_kernel<D, T><<<pg, kGdnThreads, psmem, st>>>(q);
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
        e = cudaLaunchKernelEx(&lc, gdn_prep_tc_kernel<D, T>, q);
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
        e = cudaLaunchKernelEx(&lc, gdn_tc_kernel<D, T>, q);
      }
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
}

}  // namespace

size_t gdn_workspace_bytes(int B, int H, int D, int64_t T) {
  (void)D;   // the images are 128 key dims wide for D = 64 too
  return kWsHeader + (size_t)B * (size_t)H * (size_t)((T + kCt - 1) / kCt) * (size_t)kImgBytes;
}

cudaError_t launch_gdn(const GdnParams& p, int D, int dtype, cudaStream_t st) {
  if (p.n_streams <= 0 || p.T <= 0) return cudaSuccess;
  if (D == 64)
    return dtype == SA_BF16 ? launch_gdn_t<64, __nv_bfloat16>(p, st) : launch_gdn_t<64, float>(p, st);
  return dtype == SA_BF16 ? launch_gdn_t<128, __nv_bfloat16>(p, st) : launch_gdn_t<128, float>(p, st);
}

}  // namespace sa
