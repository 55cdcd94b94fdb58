// attend_tc.cu -- bf16 flash attention over the visible key prefix of each
// (stream, head) of the rolling cache, on the sm_100a tensor cores.
//
// Work unit = one (stream, head) and a pair of 128-row query tiles. The key
// tiles of all units are laid end to end; a persistent grid of one CTA per SM
// takes equal contiguous ranges of that sequence (stream-K), so no SM idles
// in a last partial wave. A unit cut by range boundaries is finished inside
// the same launch: every piece stores its partial result (its output
// normalised by its own row sum, in fp16, and the running max and row sum in
// fp32) and counts itself in on a per-row counter; the
// thread that arrives last for a row merges all pieces of that row and
// writes it (no waiting on other CTAs). Without a partials buffer, ranges
// snap to whole units instead.
//
// CTA of 10 warps, per work unit:
//   warp 0     : TMA producer: Q tiles of the unit, then K and V tiles
//                (kStages each, separate barriers so QK^T starts before V lands)
//   warp 1     : TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..5 : softmax + epilogue of query tile 0 (one thread per row; a
//                warp reads TMEM lanes 32*(warp % 4) .. +31)
//   warps 6..9 : softmax + epilogue of query tile 1
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 after O0.
// P_i (bf16 pairs) overwrites the first 64 columns of S_i once S_i is in
// registers and feeds the PV MMA from TMEM (A operand), V being an MN-major
// shared-memory operand. Issue order per key tile j:
//   QK0(j), PV1(j-1), QK1(j), PV0(j)
// so each tile's softmax runs while the tensor core works on the other tile;
// tcgen05.mma ops issued by one thread execute in order, so QK_i(j+1) cannot
// overwrite P_i(j) before PV_i(j) has read it.
// Online softmax in the log2 domain; O is rescaled in TMEM only when the
// running max grows by more than 8; exact division by the row sum at the end.
// Every wait is bounded (about 1 s); on expiry the CTA records a device error,
// drains its outstanding copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

// debug build: the bounds word of this file (sites: 0 query tile coordinate,
// 1 key/value tile coordinate, 2 output row, 3 partial-result slot written,
// 4 arrival counter, 5 partial-result slot read by a merge, 31 self-test)
SA_DEFINE_BOUNDS_WORD(bounds_word_attend_tc)

namespace {

constexpr int BM = 128;                  // query rows per tile
constexpr int BN = 128;                  // keys per tile
constexpr uint32_t PANEL = 128u * 128u;  // one 128-row x 128-byte swizzled panel
constexpr uint64_t kTimeoutNs = 1000000000ull;
// A split unit's partial results are dead once merged: their L2 lines are
// dropped with discard.global.L2 instead of being written back to DRAM
// (measured on the 512p step: 3.5 MB less DRAM writing per launch, and the
// append kernel that follows runs 8 % faster with fewer dirty lines to
// evict; dropping the rotated-query rows as well was measured 1 % slower).
#ifndef SA_ATTN_DISCARD
#define SA_ATTN_DISCARD 1
#endif
constexpr bool kDiscardPartials = SA_ATTN_DISCARD != 0;
constexpr int kThreads = 320;
constexpr int kFirstSoftmaxWarp = 2;
constexpr int kMaxCtas = 256;


struct TcParams {
  int32_t H, Lc, n_q_tiles, n_pairs;
  int32_t n_streams, grid, split, units_per_stream;
  float scale_log2;
  int32_t batch;      // B (bounds checks)
  int64_t ntok;       // cache rows per (stream, head) (bounds checks)
  int64_t total;      // key tiles over all units
  void* out;          // [B][Lc][H][D] bf16
  uint4* part_o;      // [slots][2][D/8][128] the piece's O / l as fp16, 8 columns per
                      // 16 bytes, row-contiguous per group of 8 columns
  float2* part_ml;    // [slots][2][128] (m in log2 units, l)
  int* counters;      // [units][2][128] pieces counted in; back to 0 after the merge
  int* status;
  float inv_qk[kMaxF8Heads];  // e4m3: 1 / (q_scale * k_scale) per head
  float inv_v[kMaxF8Heads];   // e4m3: 1 / v_scale per head
  int32_t stream_of[kMaxAttnStreams];
  int32_t n_keys[kMaxAttnStreams];
  int32_t nkv[kMaxAttnStreams];
  int64_t prefix[kMaxAttnStreams + 1];  // key tiles before stream a's units
};

struct Seg {
  int a, b, h, qp, lo, hi, nkv;
  bool two, partial;
  int64_t t_end;
};

__host__ __device__ inline int64_t unit_tile_offset(const TcParams& p, int64_t u) {
  const int64_t U = (int64_t)p.n_streams * p.units_per_stream;
  if (u >= U) return p.total;
  const int a = (int)(u / p.units_per_stream);
  return p.prefix[a] + (u - (int64_t)a * p.units_per_stream) * p.nkv[a];
}

// The key tiles CTA c takes, [r0, r1): an equal share of all units' tiles in
// split mode (stream-K), else whole units.
__host__ __device__ inline void cta_range(const TcParams& p, int c, int64_t& r0, int64_t& r1) {
  if (p.split) {
    r0 = p.total * c / p.grid;
    r1 = p.total * (c + 1) / p.grid;
  } else {
    const int64_t U = (int64_t)p.n_streams * p.units_per_stream;
    r0 = unit_tile_offset(p, U * c / p.grid);
    r1 = unit_tile_offset(p, U * (c + 1) / p.grid);
  }
}

// Segment of the flattened key-tile sequence starting at t and ending at the
// end of t's unit or at r1, whichever comes first.
__host__ __device__ inline Seg make_seg(const TcParams& p, int64_t t, int64_t r1) {
  int a = 0;
  while (a + 1 < p.n_streams && p.prefix[a + 1] <= t) ++a;
  const int64_t rel = t - p.prefix[a];
  const int nk = p.nkv[a];
  const int64_t ul = rel / nk;
  Seg s;
  s.a = a;
  s.b = p.stream_of[a];
  s.h = (int)(ul / p.n_pairs);
  s.qp = (int)(ul - (int64_t)s.h * p.n_pairs);
  s.nkv = nk;
  s.lo = (int)(rel - ul * nk);
  const int64_t uend = p.prefix[a] + (ul + 1) * nk;
  s.t_end = uend < r1 ? uend : r1;
  s.hi = s.lo + (int)(s.t_end - t);
  s.two = 2 * s.qp + 1 < p.n_q_tiles;
  s.partial = s.lo > 0 || s.hi < nk;
  return s;
}

// The order in which a CTA takes the segments of its range [r0, r1): when r0
// falls inside a unit (its head piece, a unit the previous CTA began), that
// piece goes last, so both pieces of a unit split between CTAs c and c + 1
// end in the last part of the launch and the merge reads partials written
// more recently. Every role of the CTA walks the same cursor, so they agree
// on the order.
struct SegCursor {
  int64_t t, stop, r0, h_end;
  bool second;
  __device__ void init(const TcParams& p, int64_t r0_, int64_t r1) {
    r0 = r0_;
    h_end = r0_;
    if (r0_ < r1) {
      const Seg h = make_seg(p, r0_, r1);
      if (h.lo > 0 && h.t_end < r1) h_end = h.t_end;
    }
    t = h_end;
    stop = r1;
    second = false;
  }
  __device__ bool next(const TcParams& p, Seg& s) {
    if (t >= stop) {
      if (second || h_end <= r0) return false;
      t = r0;
      stop = h_end;
      second = true;
    }
    s = make_seg(p, t, stop);
    t = s.t_end;
    return true;
  }
};

// CTA whose range holds key tile t (split mode)
__device__ inline int cta_of(const TcParams& p, int64_t t) {
  int c = (int)(t * p.grid / p.total);
  while (c + 1 < p.grid && p.total * (c + 1) / p.grid <= t) ++c;
  while (c > 0 && p.total * c / p.grid > t) --c;
  return c;
}

// Partial slot of the piece that CTA c holds of the unit starting at tile us:
// slot 2c for the piece that starts c's range, 2c + 1 for the one that ends it.
__device__ inline int piece_slot(const TcParams& p, int c, int c_first, int64_t us) {
  return 2 * c + ((c == c_first && p.total * c / p.grid != us) ? 1 : 0);
}

// Eight fp16 of a 16-byte word as floats.
__device__ __forceinline__ void unpack_h8(uint4 u, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Eight floats as fp16 (round to nearest) in a 16-byte word.
__device__ __forceinline__ uint4 pack_h8(const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Merge of one query row of a split unit from the partial results of its
// pieces (CTAs c0..c1). Piece k stored its normalised output P_k = O_k / l_k
// in fp16 (|P_k| <= max |v|; relative step 2^-11, a quarter of the final bf16
// rounding) and (m_k, l_k) in fp32:
//   O = sum_k w_k P_k,  w_k = 2^(m_k - M) l_k / sum_j 2^(m_j - M) l_j,
// stored as bf16 to dst (nullptr: a padding row past Lc, nothing stored).
// All CTAs merge at about the same time, at the end of the launch, so the
// bytes read here bound the merge: fp16 halves them. The other piece's
// partials were written long before and are usually out of L2: the row's
// lines are prefetched into L2 first. Two pieces (the only case at the
// workload sizes, where a CTA's range is longer than a unit) are read
// together. Kept out of line so the softmax loop's register allocation does
// not see it.
template <int HD>
__device__ __noinline__ void merge_row(const TcParams& p, int ti, int row, int c0, int c1,
                                       int64_t us, __nv_bfloat16* dst) {
  constexpr int kG = HD / 8;  // 16-byte groups of a row
  if (c1 == c0 + 1) {
    const int s0 = piece_slot(p, c0, c0, us), s1 = piece_slot(p, c1, c0, us);
    if (!SA_BOUNDS(s0 >= 0 && s0 < 2 * p.grid && s1 >= 0 && s1 < 2 * p.grid, 5)) return;
    const uint4* a0 = p.part_o + ((int64_t)s0 * 2 + ti) * kG * BM + row;
    const uint4* a1 = p.part_o + ((int64_t)s1 * 2 + ti) * kG * BM + row;
    if (!dst) return;
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a0 + g * BM));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a1 + g * BM));
    }
    const float2 ml0 = __ldcg(p.part_ml + ((int64_t)s0 * 2 + ti) * BM + row);
    const float2 ml1 = __ldcg(p.part_ml + ((int64_t)s1 * 2 + ti) * BM + row);
    const float M = fmaxf(ml0.x, ml1.x);
    const float e0 = ptx::ex2(ml0.x - M) * ml0.y, e1 = ptx::ex2(ml1.x - M) * ml1.y;
    const float inv = 1.f / (e0 + e1);
    const float w0 = e0 * inv, w1 = e1 * inv;
    uint4 x0[kG], x1[kG];
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      x0[g] = __ldcg(a0 + g * BM);
      x1[g] = __ldcg(a1 + g * BM);
    }
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      float u[8], v[8];
      unpack_h8(x0[g], u);
      unpack_h8(x1[g], v);
      uint4 o;
      o.x = ptx::pack_bf16x2(fmaf(w0, u[0], w1 * v[0]), fmaf(w0, u[1], w1 * v[1]));
      o.y = ptx::pack_bf16x2(fmaf(w0, u[2], w1 * v[2]), fmaf(w0, u[3], w1 * v[3]));
      o.z = ptx::pack_bf16x2(fmaf(w0, u[4], w1 * v[4]), fmaf(w0, u[5], w1 * v[5]));
      o.w = ptx::pack_bf16x2(fmaf(w0, u[6], w1 * v[6]), fmaf(w0, u[7], w1 * v[7]));
      *reinterpret_cast<uint4*>(dst + g * 8) = o;
    }
    return;
  }
  float M = -INFINITY;
  for (int c = c0; c <= c1; ++c) {
    const int sl = piece_slot(p, c, c0, us);
    if (!SA_BOUNDS(sl >= 0 && sl < 2 * p.grid, 5)) return;
    M = fmaxf(M, __ldcg(p.part_ml + ((int64_t)sl * 2 + ti) * BM + row).x);
  }
  float Ls = 0.f;
  for (int c = c0; c <= c1; ++c) {
    const int sl = piece_slot(p, c, c0, us);
    const float2 ml = __ldcg(p.part_ml + ((int64_t)sl * 2 + ti) * BM + row);
    Ls += ptx::ex2(ml.x - M) * ml.y;
  }
  if (!dst) return;
  const float inv = 1.f / Ls;
#pragma unroll 1
  for (int g0 = 0; g0 < kG; g0 += 4) {  // 32 columns at a time
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int c = c0; c <= c1; ++c) {
      const int sl = piece_slot(p, c, c0, us);
      const float2 ml = __ldcg(p.part_ml + ((int64_t)sl * 2 + ti) * BM + row);
      const float w = ptx::ex2(ml.x - M) * ml.y * inv;
      const uint4* src = p.part_o + ((int64_t)sl * 2 + ti) * kG * BM + row;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float u[8];
        unpack_h8(__ldcg(src + (g0 + g) * BM), u);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[g * 8 + i] = fmaf(w, u[i], acc[g * 8 + i]);
      }
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint4 v;
      v.x = ptx::pack_bf16x2(acc[g * 8 + 0], acc[g * 8 + 1]);
      v.y = ptx::pack_bf16x2(acc[g * 8 + 2], acc[g * 8 + 3]);
      v.z = ptx::pack_bf16x2(acc[g * 8 + 4], acc[g * 8 + 5]);
      v.w = ptx::pack_bf16x2(acc[g * 8 + 6], acc[g * 8 + 7]);
      *reinterpret_cast<uint4*>(dst + (g0 + g) * 8) = v;
    }
  }
}

// F8: e4m3 operands, a 128-element row is one 128-byte panel
template <int HD, bool F8 = false>
struct Layout {
  static constexpr int kStages = F8 ? 4 : (HD == 128 ? 2 : 4);
  static constexpr uint32_t kPanels = F8 ? 1 : HD / 64;
  static constexpr uint32_t kTile = kPanels * PANEL;  // one Q, K or V tile
  static constexpr uint32_t q0 = 0;
  static constexpr uint32_t k0 = 2 * kTile;
  static constexpr uint32_t v0 = k0 + kStages * kTile;
  static constexpr uint32_t bars = v0 + kStages * kTile;
  static constexpr int B_QF = 0, B_QE = 1;
  static constexpr int B_KF = 2;
  static constexpr int B_KE = B_KF + kStages;
  static constexpr int B_VF = B_KE + kStages;
  static constexpr int B_VE = B_VF + kStages;
  static constexpr int B_SF = B_VE + kStages;  // [2] S_i written by QK_i
  static constexpr int B_PF = B_SF + 2;        // [2] P_i keys [0, 64) written by softmax i
  static constexpr int B_PB = B_PF + 2;        // [2] P_i keys [64, 128) written
  static constexpr int B_OD = B_PB + 2;        // [2] PV_i done
  static constexpr int B_OF = B_OD + 2;        // [2] O_i read by the epilogue
  static constexpr int B_DR = B_OF + 2;        // drain
  static constexpr int kNumBars = B_DR + 1;
  static constexpr uint32_t misc = bars + kNumBars * 8;
  static constexpr uint32_t bytes = misc + 16;
  static_assert(bytes <= 232448, "exceeds 227 KB of shared memory per CTA");
};

// P of 32 consecutive scores of a row as 16 words of bf16 pairs, and their
// sum added to ls (four packed partial sums). The exponentials run on the
// MUFU unit (4 per clock per SM sub-partition, in f32 or packed bf16x2 form
// alike); a polynomial on the FMA pipe costs more per element on this chip
// (FFMA2 issues at half rate), so none is used.
__device__ __forceinline__ void p_group(const uint32_t* sv, float2 sl2v, float2 nmv, float2* ls,
                                        uint32_t* w) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]),
                                            __uint_as_float(sv[2 * e + 1])), sl2v, nmv);
    const float2 pe = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
    ls[e & 3] = __fadd2_rn(ls[e & 3], pe);
    w[e] = ptx::pack_bf16x2(pe.x, pe.y);
  }
}

// O row *= alpha in TMEM (rare; out of line so that the softmax keeps its
// scores in registers without spilling around it)
template <int HD>
__device__ __noinline__ void rescale_o(uint32_t obuf, float alpha) {
#pragma unroll 1
  for (int c = 0; c < HD / 32; ++c) {
    float ov[32];
    ptx::tmem_ld32(obuf + c * 32, ov);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) ov[i] *= alpha;
    ptx::tmem_st32(obuf + c * 32, ov);
  }
}

// Softmax numerator of one query row for one key tile. The 128 scores are
// loaded from TMEM once (extra TMEM reads are expensive while the tensor core
// runs), so the max, the exponentials and the packing run from registers with
// no control flow between elements. Running max m in the log2 domain: it only
// moves when the tile's max exceeds it by more than 8 (alpha < 1 is then the
// factor for O), so P stays below 2^8. A rescale of O (rare) is done before
// any P is published (PV accumulates onto it); it only needs PV of the
// previous key tile complete (bar_od). P (bf16 pairs) overwrites S columns [0, 64) and is published in
// two halves, keys [0, 64) on bar_pa and [64, 128) on bar_pb, so the PV MMA
// of the first half runs while the second half is computed. The scale and
// subtract and the row sums use packed two-float FMA/add: the phase is bound
// by instruction count and latency rather than by the exponential unit's
// rate (moving a share of the exponentials to a polynomial on the FMA pipe
// made it slower). Adds the row sum
// of P to l (after scaling l by alpha). Returns false if a wait gave up.
template <int HD, bool F8>
__device__ __forceinline__ bool row_softmax(uint32_t sbuf, uint32_t obuf, int valid, bool first,
                                            float& m, float& l, float sl2, uint32_t bar_od,
                                            uint32_t od_parity, uint32_t bar_pa, uint32_t bar_pb,
                                            volatile int* abort_flag) {
  uint32_t sv[BN];
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) ptx::tmem_ld32u(sbuf + (uint32_t)c * 32u, sv + c * 32);
  ptx::tmem_wait_ld_dep(sv);
  ptx::tmem_wait_ld_dep(sv + 32);
  ptx::tmem_wait_ld_dep(sv + 64);
  ptx::tmem_wait_ld_dep(sv + 96);
  if (valid < BN) {
#pragma unroll
    for (int i = 0; i < BN; ++i)
      if (i >= valid) sv[i] = __float_as_uint(-INFINITY);
  }
  if (F8 && !first) {
    // e4m3 operands: optimistic pass with the running max, the tile max
    // tracked on the way; P stays in registers until the max is checked and
    // is then published whole. (With the shorter fp8 MMAs, taking the max off
    // the critical path gains more than starting the first half of PV early;
    // for bf16 it is the other way round.)
    constexpr int kW = BN / 4;
    uint32_t wo[kW];
    const float2 sl2o = make_float2(sl2, sl2), nmo = make_float2(-m, -m);
    float2 lo[4];
    float mo[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) lo[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) mo[i] = -INFINITY;
#pragma unroll
    for (int e = 0; e < BN / 2; ++e) {
      const float s0 = __uint_as_float(sv[2 * e]), s1 = __uint_as_float(sv[2 * e + 1]);
      mo[e & 7] = ptx::fmax3(mo[e & 7], s0, s1);
      const float2 x = __ffma2_rn(make_float2(s0, s1), sl2o, nmo);
      const float2 pe = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
      lo[e & 3] = __fadd2_rn(lo[e & 3], pe);
      const uint32_t pp = ptx::pack_e4m3x2(pe.x, pe.y);
      if (e & 1)
        wo[e >> 1] |= pp << 16;
      else
        wo[e >> 1] = pp;
    }
    const float tm = ptx::fmax3(ptx::fmax3(mo[0], mo[1], mo[2]), ptx::fmax3(mo[3], mo[4], mo[5]),
                                fmaxf(mo[6], mo[7])) * sl2;
    if (!__any_sync(0xffffffffu, tm > m + 8.0f)) {
#pragma unroll
      for (int q = 0; q < BN / 32; ++q) ptx::tmem_st8u(sbuf + (uint32_t)(q * 8), wo + q * 8);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar_pa);
      ptx::mbar_arrive(bar_pb);
      const float2 l2 = __fadd2_rn(__fadd2_rn(lo[0], lo[1]), __fadd2_rn(lo[2], lo[3]));
      l += l2.x + l2.y;
      return true;
    }
    // rare: nothing is stored yet, so S is intact in TMEM; take the exact path
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) ptx::tmem_ld32u(sbuf + (uint32_t)c * 32u, sv + c * 32);
    ptx::tmem_wait_ld_dep(sv);
    ptx::tmem_wait_ld_dep(sv + 32);
    ptx::tmem_wait_ld_dep(sv + 64);
    ptx::tmem_wait_ld_dep(sv + 96);
    if (valid < BN) {
#pragma unroll
      for (int i = 0; i < BN; ++i)
        if (i >= valid) sv[i] = __float_as_uint(-INFINITY);
    }
  }
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(__uint_as_float(sv[i]), __uint_as_float(sv[i + 8]));
#pragma unroll
  for (int i = 16; i < BN; i += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k)
      mx[k] = ptx::fmax3(mx[k], __uint_as_float(sv[i + k]), __uint_as_float(sv[i + 8 + k]));
  const float tmax =
      ptx::fmax3(ptx::fmax3(mx[0], mx[1], mx[2]), ptx::fmax3(mx[3], mx[4], mx[5]),
                 fmaxf(mx[6], mx[7])) * sl2;
  float alpha = 1.f;
  if (first) {
    m = tmax;
  } else if (tmax > m + 8.0f) {
    alpha = ptx::ex2(m - tmax);
    m = tmax;
  }
  const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(-m, -m);
  float2 ls[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
  if constexpr (!F8) {
    // bf16: groups of 32 keys; the third group is computed before waiting
    // for the first two groups' TMEM stores, so that wait overlaps work
    uint32_t wa[16], wb[16];
    p_group(sv, sl2v, nmv, ls, wa);
    ptx::tmem_st16u(sbuf, wa);
    p_group(sv + 32, sl2v, nmv, ls, wb);
    ptx::tmem_st16u(sbuf + 16u, wb);
    if (__any_sync(0xffffffffu, alpha < 1.f)) {
      // O holds PV of the previous key tile: MMAs complete in issue order and
      // QK of this tile (issued after that PV) has completed
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_od, od_parity, abort_flag, kTimeoutNs)))
        return false;
      ptx::tc_fence_after();
      rescale_o<HD>(obuf, alpha);
    }
    p_group(sv + 64, sl2v, nmv, ls, wa);
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar_pa);
    ptx::tmem_st16u(sbuf + 32u, wa);
    p_group(sv + 96, sl2v, nmv, ls, wb);
    ptx::tmem_st16u(sbuf + 48u, wb);
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(bar_pb);
    const float2 l2 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
    l = l * alpha + (l2.x + l2.y);
    return true;
  } else {
    // e4m3 exact path (first tile of a unit, or the running max jumped)
#pragma unroll
    for (int q = 0; q < BN / 32; ++q) {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[q * 32 + 2 * e]),
                                                __uint_as_float(sv[q * 32 + 2 * e + 1])),
                                    sl2v, nmv);
        const float2 pe = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
        ls[e & 3] = __fadd2_rn(ls[e & 3], pe);
        // four e4m3 per column: pairs e and e+1 share a word
        const uint32_t pp = ptx::pack_e4m3x2(pe.x, pe.y);
        if (e & 1)
          w[e >> 1] |= pp << 16;
        else
          w[e >> 1] = pp;
      }
      ptx::tmem_st8u(sbuf + (uint32_t)(q * 8), w);
      if (q == 1 && __any_sync(0xffffffffu, alpha < 1.f)) {
        // O holds PV of the previous key tile: MMAs complete in issue order
        // and QK of this tile (issued after that PV) has completed
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_od, od_parity, abort_flag, kTimeoutNs)))
          return false;
        ptx::tc_fence_after();
        rescale_o<HD>(obuf, alpha);
      }
      if (q == 1 || q == 3) {
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(q == 1 ? bar_pa : bar_pb);
      }
    }
    const float2 l2 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
    l = l * alpha + (l2.x + l2.y);
    return true;
  }
}

template <int HD, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ TcParams p) {
  using L = Layout<HD, F8>;
  constexpr int ST = L::kStages;
  // MMAs per QK^T tile, per half of a PV tile, and V bytes per PV MMA
  constexpr int kQkSteps = F8 ? HD / 32 : HD / 16;
  constexpr int kPvHalf = F8 ? BN / 64 : BN / 32;
  constexpr uint32_t kVStep = F8 ? 4096u : 2048u;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = ptx::smem_u32(smem);
  if (base & 1023u) {  // 128B-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.status, kDeviceErrTimeout);
    return;
  }
  const uint32_t bar0 = base + L::bars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + L::misc + 8);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(L::B_QF), 1);
    ptx::mbar_init(bar(L::B_QE), 1);
    for (int s = 0; s < ST; ++s) {
      ptx::mbar_init(bar(L::B_KF + s), 1);
      ptx::mbar_init(bar(L::B_KE + s), 1);
      ptx::mbar_init(bar(L::B_VF + s), 1);
      ptx::mbar_init(bar(L::B_VE + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(L::B_SF + i), 1);
      ptx::mbar_init(bar(L::B_PF + i), 128);
      ptx::mbar_init(bar(L::B_PB + i), 128);
      ptx::mbar_init(bar(L::B_OD + i), 1);
      ptx::mbar_init(bar(L::B_OF + i), 128);
    }
    ptx::mbar_init(bar(L::B_DR), 1);
    *abort_flag = 0;
    *no_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kDeviceErrTimeout);
  };
  int64_t r0, r1;
  cta_range(p, blockIdx.x, r0, r1);
  if (warp < kFirstSoftmaxWarp) {
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      int n = 0, g = 0;
      bool ok = true;
      SegCursor cur;
      cur.init(p, r0, r1);
      Seg sg;
      while (ok && cur.next(p, sg)) {
        if (n > 0 && !ptx::mbar_wait(bar(L::B_QE), (uint32_t)(n - 1) & 1, abort_flag, kTimeoutNs)) {
          ok = false;
          break;
        }
        int bh = sg.b * p.H + sg.h;
        // (a bad coordinate is clamped: the copy still completes the barrier)
        if (!SA_BOUNDS(bh >= 0 && bh < p.batch * p.H && sg.qp >= 0 &&
                           (2 * sg.qp + (sg.two ? 1 : 0)) < p.n_q_tiles, 0))
          bh = 0, sg.qp = 0;
        ptx::mbar_arrive_expect_tx(bar(L::B_QF), (sg.two ? 2u : 1u) * L::kTile);
        for (int i = 0; i < (sg.two ? 2 : 1); ++i)
          for (uint32_t pn = 0; pn < L::kPanels; ++pn)
            ptx::tma_load_3d(base + L::q0 + (uint32_t)i * L::kTile + pn * PANEL, &tm_q, bar(L::B_QF),
                             (int)pn * 64, (2 * sg.qp + i) * BM, bh);
        ++n;
        for (int kv = sg.lo; kv < sg.hi; ++kv, ++g) {
          const int s = g % ST;
          const uint32_t u = (uint32_t)(g / ST);
          if (u > 0 && !ptx::mbar_wait(bar(L::B_KE + s), (u - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          const int kr = SA_BOUNDS(kv >= 0 && kv < sg.nkv && (int64_t)kv * BN < p.ntok, 1) ? kv : 0;
          ptx::mbar_arrive_expect_tx(bar(L::B_KF + s), L::kTile);
          for (uint32_t pn = 0; pn < L::kPanels; ++pn)
            ptx::tma_load_3d(base + L::k0 + s * L::kTile + pn * PANEL, &tm_k, bar(L::B_KF + s),
                             (int)pn * 64, kr * BN, bh);
          if (u > 0 && !ptx::mbar_wait(bar(L::B_VE + s), (u - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            ++g;  // K of this tile is in flight: drain it below
            break;
          }
          ptx::mbar_arrive_expect_tx(bar(L::B_VF + s), L::kTile);
          for (uint32_t pn = 0; pn < L::kPanels; ++pn)
            ptx::tma_load_3d(base + L::v0 + s * L::kTile + pn * PANEL, &tm_v, bar(L::B_VF + s),
                             (int)pn * 64, kr * BN, bh);
        }
      }
      if (!ok) fail();
      // drain: the copies this thread issued have landed before the CTA exits
      if (n > 0) ptx::mbar_wait(bar(L::B_QF), (uint32_t)(n - 1) & 1, no_abort, kTimeoutNs);
      for (int x = g - 1; x >= 0 && x >= g - ST; --x) {
        ptx::mbar_wait(bar(L::B_KF + x % ST), (uint32_t)(x / ST) & 1, no_abort, kTimeoutNs);
        ptx::mbar_wait(bar(L::B_VF + x % ST), (uint32_t)(x / ST) & 1, no_abort, kTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk =
          F8 ? ptx::idesc_e4m3_f32(BM, BN, false) : ptx::idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_pv =
          F8 ? ptx::idesc_e4m3_f32(BM, HD, true) : ptx::idesc_bf16_f32(BM, HD, true);
      // K offset of QK^T step kk inside a K-major tile (32 bytes per step)
      auto qk_off = [](int kk) -> uint32_t {
        return F8 ? (uint32_t)kk * 32u : (uint32_t)(kk >> 2) * PANEL + (uint32_t)(kk & 3) * 32u;
      };
      auto mma_ss = [](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (F8) ptx::umma_ss_f8(d, a, b, id, acc); else ptx::umma_ss(d, a, b, id, acc);
      };
      auto mma_ts = [](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (F8) ptx::umma_ts_f8(d, a, b, id, acc); else ptx::umma_ts(d, a, b, id, acc);
      };
      const uint32_t o0 = tmem + 256u, o1 = tmem + 256u + HD;
      const uint64_t dq = ptx::sdesc_sw128(base + L::q0, 16, 1024);
      int n = 0, g = 0, g1 = 0, nseg1 = 0;
      bool ok = true;
      // PV1 of the previous key tile, issued after the next QK0
      bool pend = false, pend_first = false;
      int pend_g = 0, pend_g1 = 0, pend_nseg1 = 0;
      auto issue_pv1 = [&]() -> bool {
        if (pend_first && pend_nseg1 > 0 &&
            !ptx::mbar_wait(bar(L::B_OF + 1), (uint32_t)(pend_nseg1 - 1) & 1, abort_flag, kTimeoutNs))
          return false;
        const int s = pend_g % ST;
        const uint64_t dv = ptx::sdesc_sw128(base + L::v0 + s * L::kTile, PANEL, 1024);
        for (int h2 = 0; h2 < 2; ++h2) {
          if (!ptx::mbar_wait(bar((h2 == 0 ? L::B_PF : L::B_PB) + 1), (uint32_t)pend_g1 & 1,
                              abort_flag, kTimeoutNs))
            return false;
          ptx::tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < kPvHalf; ++k2) {
            const int kk = h2 * kPvHalf + k2;
            mma_ts(o1, tmem + 128u + (uint32_t)kk * 8u, ptx::sdesc_add(dv, (uint32_t)kk * kVStep),
                   idesc_pv, (!pend_first || kk > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(bar(L::B_OD + 1));
        ptx::umma_commit(bar(L::B_VE + s));
        pend = false;
        return true;
      };
      SegCursor cur;
      cur.init(p, r0, r1);
      Seg sg;
      while (ok && cur.next(p, sg)) {
        if (pend && !issue_pv1()) { ok = false; break; }
        if (!ptx::mbar_wait(bar(L::B_QF), (uint32_t)n & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
        for (int kv = sg.lo; kv < sg.hi; ++kv, ++g) {
          const int s = g % ST;
          const uint32_t u = (uint32_t)(g / ST);
          if (!ptx::mbar_wait(bar(L::B_KF + s), u & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t dk = ptx::sdesc_sw128(base + L::k0 + s * L::kTile, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kQkSteps; ++kk) {
            const uint32_t off = qk_off(kk);
            mma_ss(tmem, ptx::sdesc_add(dq, off), ptx::sdesc_add(dk, off), idesc_qk,
                   kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar(L::B_SF + 0));
          if (pend && !issue_pv1()) { ok = false; break; }
          if (sg.two) {
#pragma unroll
            for (int kk = 0; kk < kQkSteps; ++kk) {
              const uint32_t off = qk_off(kk);
              mma_ss(tmem + 128u, ptx::sdesc_add(dq, L::kTile + off), ptx::sdesc_add(dk, off),
                     idesc_qk, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar(L::B_SF + 1));
          }
          ptx::umma_commit(bar(L::B_KE + s));
          if (kv == sg.hi - 1) ptx::umma_commit(bar(L::B_QE));
          if (!ptx::mbar_wait(bar(L::B_VF + s), u & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          if (kv == sg.lo && n > 0 &&
              !ptx::mbar_wait(bar(L::B_OF + 0), (uint32_t)(n - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          const uint64_t dv = ptx::sdesc_sw128(base + L::v0 + s * L::kTile, PANEL, 1024);
          for (int h2 = 0; h2 < 2 && ok; ++h2) {
            if (!ptx::mbar_wait(bar((h2 == 0 ? L::B_PF : L::B_PB) + 0), (uint32_t)g & 1, abort_flag,
                                kTimeoutNs)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll
            for (int k2 = 0; k2 < kPvHalf; ++k2) {
              const int kk = h2 * kPvHalf + k2;
              mma_ts(o0, tmem + (uint32_t)kk * 8u, ptx::sdesc_add(dv, (uint32_t)kk * kVStep),
                     idesc_pv, (kv > sg.lo || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          ptx::umma_commit(bar(L::B_OD + 0));
          if (sg.two) {
            pend = true;
            pend_g = g;
            pend_g1 = g1;
            pend_first = kv == sg.lo;
            pend_nseg1 = nseg1;
            ++g1;
          } else {
            ptx::umma_commit(bar(L::B_VE + s));
          }
        }
        ++n;
        if (sg.two) ++nseg1;
      }
      if (ok && pend && !issue_pv1()) ok = false;
      if (!ok) fail();
      // drain: all MMAs issued by this thread have completed
      ptx::umma_commit(bar(L::B_DR));
      ptx::mbar_wait(bar(L::B_DR), 0, no_abort, kTimeoutNs);
    }
  }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int ti = (warp - kFirstSoftmaxWarp) >> 2;  // query tile of this warp's warpgroup
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t sbuf = t_lane + (uint32_t)ti * 128u;
    const uint32_t obuf = t_lane + 256u + (uint32_t)(ti * HD);
    int gi = 0;
    bool ok = true;
    SegCursor cur;
    cur.init(p, r0, r1);
    Seg sg;
    while (ok && cur.next(p, sg)) {
      if (ti == 1 && !sg.two) continue;
      // e4m3: scores carry the head's q and k scales, O its v scale
      const float sl2 = F8 ? p.scale_log2 * p.inv_qk[sg.h] : p.scale_log2;
      const float o_scale = F8 ? p.inv_v[sg.h] : 1.f;
      const int n_keys = p.n_keys[sg.a];
      float m_used = 0.f, l = 0.f;
      for (int kv = sg.lo; kv < sg.hi; ++kv, ++gi) {
        // waits are made warp-uniform: the TMEM accesses below are .sync.aligned
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_SF + ti), (uint32_t)gi & 1,
                                                    abort_flag, kTimeoutNs))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const int valid = n_keys - kv * BN;
        if (!row_softmax<HD, F8>(sbuf, obuf, valid, kv == sg.lo, m_used, l, sl2, bar(L::B_OD + ti),
                             (uint32_t)(gi - 1) & 1, bar(L::B_PF + ti), bar(L::B_PB + ti),
                             abort_flag)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_OD + ti), (uint32_t)(gi - 1) & 1,
                                                  abort_flag, kTimeoutNs))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // ---- epilogue of this unit piece
      const int tok = (2 * sg.qp + ti) * BM + row;
      if (!sg.partial) {
        const bool st_ok = SA_BOUNDS(sg.b >= 0 && sg.b < p.batch && sg.h < p.H, 2);
        const float inv = o_scale / l;
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                             (((int64_t)sg.b * p.Lc + tok) * p.H + sg.h) * HD;
        // the whole O row in one TMEM round trip
        float ov[HD];
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) ptx::tmem_ld32(obuf + c * 32, ov + c * 32);
        ptx::tmem_wait_ld();
        if (tok < p.Lc && st_ok) {
#pragma unroll
          for (int g8 = 0; g8 < HD / 8; ++g8) {
            uint4 v;
            v.x = ptx::pack_bf16x2(ov[g8 * 8 + 0] * inv, ov[g8 * 8 + 1] * inv);
            v.y = ptx::pack_bf16x2(ov[g8 * 8 + 2] * inv, ov[g8 * 8 + 3] * inv);
            v.z = ptx::pack_bf16x2(ov[g8 * 8 + 4] * inv, ov[g8 * 8 + 5] * inv);
            v.w = ptx::pack_bf16x2(ov[g8 * 8 + 6] * inv, ov[g8 * 8 + 7] * inv);
            *reinterpret_cast<uint4*>(dst + g8 * 8) = v;
          }
        }
      } else {
        // slot 2c holds the piece that starts the CTA's range, 2c + 1 the
        // other (a CTA has at most two partial pieces: its first and last)
        const int slot = 2 * (int)blockIdx.x + (sg.t_end - (sg.hi - sg.lo) == r0 ? 0 : 1);
        const bool sl_ok = SA_BOUNDS(slot >= 0 && slot < 2 * p.grid, 3);
        uint4* po = p.part_o + ((int64_t)slot * 2 + ti) * (HD / 8) * BM + row;
        float ov[HD];
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) ptx::tmem_ld32(obuf + c * 32, ov + c * 32);
        ptx::tmem_wait_ld();
        if (sl_ok) {
          // normalised, in output units (v scale removed), fp16
          const float nrm = o_scale / l;
#pragma unroll
          for (int i = 0; i < HD; ++i) ov[i] *= nrm;
#pragma unroll
          for (int g = 0; g < HD / 8; ++g) po[g * BM] = pack_h8(ov + g * 8);
        }
        if (sl_ok) p.part_ml[((int64_t)slot * 2 + ti) * BM + row] = make_float2(m_used, l);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_OF + ti));  // O_i is free for the next unit

      if (sg.partial) {
        // count this piece in for the row; the last one merges all pieces
        const int64_t us = sg.t_end - (sg.hi - sg.lo) - sg.lo;
        const int c0 = cta_of(p, us), c1 = cta_of(p, us + sg.nkv - 1);
        const int64_t u = (int64_t)sg.a * p.units_per_stream + (int64_t)sg.h * p.n_pairs + sg.qp;
        int* ctr = p.counters + (u * 2 + ti) * BM + row;
        __threadfence();
        bool merged = false;
        if (SA_BOUNDS(u >= 0 && u < (int64_t)p.n_streams * p.units_per_stream && c0 >= 0 &&
                          c1 < p.grid && c0 <= c1, 4) &&
            atomicAdd(ctr, 1) == c1 - c0) {
          atomicExch(ctr, 0);
          __threadfence();
          merge_row<HD>(p, ti, row, c0, c1, us,
                        tok < p.Lc ? static_cast<__nv_bfloat16*>(p.out) +
                                         (((int64_t)sg.b * p.Lc + tok) * p.H + sg.h) * HD
                                   : nullptr);
          merged = true;
        }
        if (kDiscardPartials && __all_sync(0xffffffffu, merged)) {
          // every row of this warp is merged: the pieces' partial results of
          // these 32 rows are dead; drop their L2 lines without a write-back
          // (a 128-byte line holds 8 rows of one 8-column group)
          for (int c = c0; c <= c1; ++c) {
            const int sl = piece_slot(p, c, c0, us);
            const char* pb = reinterpret_cast<const char*>(
                p.part_o + ((int64_t)sl * 2 + ti) * (HD / 8) * BM + quad * 32);
#pragma unroll 1
            for (int i = lane; i < (HD / 8) * 4; i += 32)
              asm volatile("discard.global.L2 [%0], 128;" ::"l"(pb + (i >> 2) * (BM * 16) +
                                                                 (i & 3) * 128)
                           : "memory");
            if (lane < 2)
              asm volatile("discard.global.L2 [%0], 128;" ::"l"(
                               reinterpret_cast<const char*>(p.part_ml + ((int64_t)sl * 2 + ti) * BM +
                                                             quad * 32) + lane * 128)
                           : "memory");
          }
        }
      }
    }
    if (!ok) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

template <int HD, bool F8>
cudaError_t launch_tc(const AttnParams& ap, const CUtensorMap* tq, const CUtensorMap* tk,
                      const CUtensorMap* tv, void* partials, size_t partials_bytes, int num_sms,
                      cudaStream_t st, int* n_kernels) {
  using L = Layout<HD, F8>;
  static unsigned configured = 0;  // one bit per device ordinal < 32
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<HD, F8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.H = ap.H;
  p.Lc = ap.Lc;
  p.n_q_tiles = ap.n_q_tiles;
  p.n_pairs = (ap.n_q_tiles + 1) / 2;
  p.n_streams = ap.n_streams;
  p.units_per_stream = p.H * p.n_pairs;
  p.scale_log2 = ap.scale_log2;
  p.batch = ap.batch;
  p.ntok = ap.ntok;
  p.out = ap.out;
  p.status = ap.status;
  if (F8)
    for (int hh = 0; hh < ap.H && hh < kMaxF8Heads; ++hh) {
      p.inv_qk[hh] = ap.inv_qk[hh];
      p.inv_v[hh] = ap.inv_v[hh];
    }
  int64_t total = 0;
  for (int a = 0; a < ap.n_streams; ++a) {
    p.stream_of[a] = ap.stream_of[a];
    p.n_keys[a] = ap.n_keys[a];
    p.nkv[a] = (ap.n_keys[a] + BN - 1) / BN;
    p.prefix[a] = total;
    total += (int64_t)p.units_per_stream * p.nkv[a];
  }
  p.prefix[ap.n_streams] = total;
  p.total = total;
  const int64_t units = (int64_t)ap.n_streams * p.units_per_stream;
  int G = std::min(num_sms, kMaxCtas);
  const size_t need = attend_partials_bytes(HD, G, units);
  p.split = partials != nullptr && partials_bytes >= need && total >= G;
  if (!p.split) G = (int)std::min<int64_t>(G, units);
  p.grid = G;
  if (p.split) {
    char* w = static_cast<char*>(partials);
    p.part_o = reinterpret_cast<uint4*>(w);
    w += (size_t)2 * G * 2 * BM * HD * sizeof(float);
    p.part_ml = reinterpret_cast<float2*>(w);
    w += (size_t)2 * G * 2 * BM * sizeof(float2);
    p.counters = reinterpret_cast<int*>(w);
  }
  attend_tc_kernel<HD, F8><<<G, kThreads, L::bytes, st>>>(*tq, *tk, *tv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int launched = 1;
  if (n_kernels) *n_kernels = launched;
  return cudaSuccess;
}

#ifdef SA_DEBUG_BOUNDS
__global__ void bounds_selftest_kernel() { (void)SA_BOUNDS(threadIdx.x != 0, 31); }
#endif

}  // namespace

#ifdef SA_DEBUG_BOUNDS
cudaError_t bounds_selftest(cudaStream_t st) {
  bounds_selftest_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}
#endif

size_t attend_partials_bytes(int D, int num_sms, int64_t max_units) {
  const size_t G = (size_t)std::min(num_sms, kMaxCtas);
  return 2 * G * 2 * BM * ((size_t)D * 4 + 8) + (size_t)max_units * 2 * BM * sizeof(int);
}

cudaError_t launch_attend_tc_bf16(const AttnParams& p, int D, const CUtensorMap* tm_q,
                                  const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                  void* partials, size_t partials_bytes, int num_sms,
                                  cudaStream_t st, int* n_kernels) {
  if (p.fp8)
    return D == 128 ? launch_tc<128, true>(p, tm_q, tm_k, tm_v, partials, partials_bytes, num_sms,
                                           st, n_kernels)
                    : cudaErrorInvalidValue;
  if (D == 128)
    return launch_tc<128, false>(p, tm_q, tm_k, tm_v, partials, partials_bytes, num_sms, st,
                                 n_kernels);
  if (D == 64)
    return launch_tc<64, false>(p, tm_q, tm_k, tm_v, partials, partials_bytes, num_sms, st,
                                n_kernels);
  return cudaErrorInvalidValue;
}

}  // namespace sa
