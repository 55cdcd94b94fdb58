// attend_tc.cu -- bf16 flash attention over the visible key prefix of each
// (stream, head) of the rolling cache, on the sm_100a tensor cores.
//
// Work unit = one (stream, head) and a pair of 128-row query tiles. The key
// tiles of all units are laid end to end; a persistent grid of one CTA per SM
// takes equal contiguous ranges of that sequence (stream-K), so no SM idles
// in a last partial wave. A unit cut by a range boundary is finished by the
// combine kernel from fp32 partial results (unnormalised O, running max,
// row sum) of its pieces. Without a partials buffer, ranges snap to whole
// units instead.
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
#include <string.h>

#include <algorithm>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace sa {
namespace {

constexpr int BM = 128;                  // query rows per tile
constexpr int BN = 128;                  // keys per tile
constexpr uint32_t PANEL = 128u * 128u;  // one 128-row x 128-byte swizzled panel
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kThreads = 320;
constexpr int kMaxCtas = 256;

struct TcParams {
  int32_t H, Lc, n_q_tiles, n_pairs;
  int32_t n_streams, grid, split, units_per_stream;
  float scale_log2;
  int32_t pad_;
  int64_t total;      // key tiles over all units
  void* out;          // [B][Lc][H][D] bf16
  float* part_o;      // [slots][2][128][D] fp32
  float* part_ml;     // [slots][2][128][2] fp32 (m in log2 units, l)
  int* status;
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

template <int HD>
struct Layout {
  static constexpr int kStages = HD == 128 ? 2 : 4;
  static constexpr uint32_t kPanels = HD / 64;
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
  static constexpr int B_PF = B_SF + 2;        // [2] P_i written by softmax i
  static constexpr int B_OD = B_PF + 2;        // [2] PV_i done
  static constexpr int B_OF = B_OD + 2;        // [2] O_i read by the epilogue
  static constexpr int B_DR = B_OF + 2;        // drain
  static constexpr int kNumBars = B_DR + 1;
  static constexpr uint32_t misc = bars + kNumBars * 8;
  static constexpr uint32_t bytes = misc + 16;
  static_assert(bytes <= 232448, "exceeds 227 KB of shared memory per CTA");
};

// Softmax numerator of one query row for one key tile. The 128 scores are
// loaded from TMEM once (extra TMEM reads are expensive while the tensor core
// runs), so the max, the exponentials and the packing run from registers with
// no control flow between elements. Running max m in the log2 domain: it only
// moves when the tile's max exceeds it by more than 8 (alpha < 1 is then the
// factor for O), so P stays below 2^8. P (bf16 pairs) overwrites S columns
// [0, 64). Returns the fp32 row sum of P.
__device__ __forceinline__ float row_softmax(uint32_t sbuf, int valid, bool first, float& m,
                                            float sl2, float& alpha) {
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
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(sv[i]);
#pragma unroll
  for (int i = 8; i < BN; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[i]));
#pragma unroll
  for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
    for (int i = 0; i < w2; ++i) mx[i] = fmaxf(mx[i], mx[i + w2]);
  const float tmax = mx[0] * sl2;
  alpha = 1.f;
  if (first) {
    m = tmax;
  } else if (tmax > m + 8.0f) {
    alpha = ptx::ex2(m - tmax);
    m = tmax;
  }
  float ls[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ls[i] = 0.f;
#pragma unroll
  for (int q = 0; q < BN / 32; ++q) {
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = ptx::ex2(fmaf(__uint_as_float(sv[q * 32 + 2 * e]), sl2, -m));
      const float p1 = ptx::ex2(fmaf(__uint_as_float(sv[q * 32 + 2 * e + 1]), sl2, -m));
      ls[(e & 3) * 2] += p0;
      ls[(e & 3) * 2 + 1] += p1;
      w[e] = ptx::pack_bf16x2(p0, p1);
    }
    ptx::tmem_st16u(sbuf + (uint32_t)(q * 16), w);
  }
  return ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ TcParams p) {
  using L = Layout<HD>;
  constexpr int ST = L::kStages;
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      int n = 0, g = 0;
      bool ok = true;
      for (int64_t t = r0; ok && t < r1;) {
        const Seg sg = make_seg(p, t, r1);
        t = sg.t_end;
        if (n > 0 && !ptx::mbar_wait(bar(L::B_QE), (uint32_t)(n - 1) & 1, abort_flag, kTimeoutNs)) {
          ok = false;
          break;
        }
        const int bh = sg.b * p.H + sg.h;
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
          ptx::mbar_arrive_expect_tx(bar(L::B_KF + s), L::kTile);
          for (uint32_t pn = 0; pn < L::kPanels; ++pn)
            ptx::tma_load_3d(base + L::k0 + s * L::kTile + pn * PANEL, &tm_k, bar(L::B_KF + s),
                             (int)pn * 64, kv * BN, bh);
          if (u > 0 && !ptx::mbar_wait(bar(L::B_VE + s), (u - 1) & 1, abort_flag, kTimeoutNs)) {
            ok = false;
            ++g;  // K of this tile is in flight: drain it below
            break;
          }
          ptx::mbar_arrive_expect_tx(bar(L::B_VF + s), L::kTile);
          for (uint32_t pn = 0; pn < L::kPanels; ++pn)
            ptx::tma_load_3d(base + L::v0 + s * L::kTile + pn * PANEL, &tm_v, bar(L::B_VF + s),
                             (int)pn * 64, kv * BN, bh);
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
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(BM, HD, true);
      const uint32_t o0 = tmem + 256u, o1 = tmem + 256u + HD;
      int n = 0, g = 0, g1 = 0, nseg1 = 0;
      bool ok = true;
      // PV1 of the previous key tile, issued after the next QK0
      bool pend = false, pend_first = false;
      int pend_g = 0, pend_g1 = 0, pend_nseg1 = 0;
      auto issue_pv1 = [&]() -> bool {
        if (pend_first && pend_nseg1 > 0 &&
            !ptx::mbar_wait(bar(L::B_OF + 1), (uint32_t)(pend_nseg1 - 1) & 1, abort_flag, kTimeoutNs))
          return false;
        if (!ptx::mbar_wait(bar(L::B_PF + 1), (uint32_t)pend_g1 & 1, abort_flag, kTimeoutNs))
          return false;
        ptx::tc_fence_after();
        const int s = pend_g % ST;
        const uint32_t vb = base + L::v0 + s * L::kTile;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          ptx::umma_ts(o1, tmem + 128u + (uint32_t)kk * 8u,
                       ptx::sdesc_sw128(vb + (uint32_t)kk * 2048u, PANEL, 1024), idesc_pv,
                       (!pend_first || kk > 0) ? 1u : 0u);
        ptx::umma_commit(bar(L::B_OD + 1));
        ptx::umma_commit(bar(L::B_VE + s));
        pend = false;
        return true;
      };
      for (int64_t t = r0; ok && t < r1;) {
        const Seg sg = make_seg(p, t, r1);
        t = sg.t_end;
        if (pend && !issue_pv1()) { ok = false; break; }
        if (!ptx::mbar_wait(bar(L::B_QF), (uint32_t)n & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
        for (int kv = sg.lo; kv < sg.hi; ++kv, ++g) {
          const int s = g % ST;
          const uint32_t u = (uint32_t)(g / ST);
          if (!ptx::mbar_wait(bar(L::B_KF + s), u & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t kb = base + L::k0 + s * L::kTile;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * PANEL + (uint32_t)(kk & 3) * 32u;
            ptx::umma_ss(tmem, ptx::sdesc_sw128(base + L::q0 + off, 16, 1024),
                         ptx::sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar(L::B_SF + 0));
          if (pend && !issue_pv1()) { ok = false; break; }
          if (sg.two) {
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
              const uint32_t off = (uint32_t)(kk >> 2) * PANEL + (uint32_t)(kk & 3) * 32u;
              ptx::umma_ss(tmem + 128u, ptx::sdesc_sw128(base + L::q0 + L::kTile + off, 16, 1024),
                           ptx::sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
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
          if (!ptx::mbar_wait(bar(L::B_PF + 0), (uint32_t)g & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t vb = base + L::v0 + s * L::kTile;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            ptx::umma_ts(o0, tmem + (uint32_t)kk * 8u,
                         ptx::sdesc_sw128(vb + (uint32_t)kk * 2048u, PANEL, 1024), idesc_pv,
                         (kv > sg.lo || kk > 0) ? 1u : 0u);
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
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int ti = (warp - 2) >> 2;  // query tile: warps 2..5 -> 0, warps 6..9 -> 1
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t sbuf = t_lane + (uint32_t)ti * 128u;
    const uint32_t obuf = t_lane + 256u + (uint32_t)(ti * HD);
    const float sl2 = p.scale_log2;
    int gi = 0;
    bool ok = true, first = true;
    for (int64_t t = r0; ok && t < r1;) {
      const Seg sg = make_seg(p, t, r1);
      t = sg.t_end;
      const bool seg_first = first;
      first = false;
      if (ti == 1 && !sg.two) continue;
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
        // the first tile of a piece sets the running max exactly; later tiles
        // use it as is and only take the slow path (exact max, rescale,
        // recompute) when the row sum shows a value above 2^16 (or not finite)
        float alpha;
        const float lsum = row_softmax(sbuf, valid, kv == sg.lo, m_used, sl2, alpha);
        const bool rescale = alpha < 1.f;
        l = l * alpha + lsum;
        if (__any_sync(0xffffffffu, rescale)) {
          // O_i holds PV_i of the previous key tile: MMAs complete in issue
          // order and QK_i of this tile (issued after that PV) has completed
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_OD + ti), (uint32_t)(gi - 1) & 1,
                                                      abort_flag, kTimeoutNs))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float ov[32];
            ptx::tmem_ld32(obuf + c * 32, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            ptx::tmem_st32(obuf + c * 32, ov);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(L::B_PF + ti));
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
        const float inv = 1.f / l;
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                             (((int64_t)sg.b * p.Lc + tok) * p.H + sg.h) * HD;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          float ov[32];
          ptx::tmem_ld32(obuf + c * 32, ov);
          ptx::tmem_wait_ld();
          if (tok < p.Lc) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              uint4 v;
              v.x = ptx::pack_bf16x2(ov[g8 * 8 + 0] * inv, ov[g8 * 8 + 1] * inv);
              v.y = ptx::pack_bf16x2(ov[g8 * 8 + 2] * inv, ov[g8 * 8 + 3] * inv);
              v.z = ptx::pack_bf16x2(ov[g8 * 8 + 4] * inv, ov[g8 * 8 + 5] * inv);
              v.w = ptx::pack_bf16x2(ov[g8 * 8 + 6] * inv, ov[g8 * 8 + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c * 32 + g8 * 8) = v;
            }
          }
        }
      } else {
        const int slot = 2 * (int)blockIdx.x + (seg_first ? 0 : 1);
        float* po = p.part_o + (((int64_t)slot * 2 + ti) * BM + row) * HD;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          float ov[32];
          ptx::tmem_ld32(obuf + c * 32, ov);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int g4 = 0; g4 < 8; ++g4)
            *reinterpret_cast<float4*>(po + c * 32 + g4 * 4) =
                make_float4(ov[g4 * 4], ov[g4 * 4 + 1], ov[g4 * 4 + 2], ov[g4 * 4 + 3]);
        }
        *reinterpret_cast<float2*>(p.part_ml + (((int64_t)slot * 2 + ti) * BM + row) * 2) =
            make_float2(m_used, l);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_OF + ti));
    }
    if (!ok) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- combine
constexpr int kMaxCombine = kMaxCtas;

struct CombineParams {
  int32_t H, Lc, n_q_tiles, n_units;
  const float* part_o;
  const float* part_ml;
  void* out;
  int32_t unit_b[kMaxCombine];
  int32_t unit_h[kMaxCombine];
  int32_t unit_qp[kMaxCombine];
  int32_t slot_begin[kMaxCombine + 1];
  int32_t slots[2 * kMaxCtas];
};

// One warp per output row: O = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k.
template <int HD>
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ CombineParams p) {
  constexpr int PER = HD / 32;
  const int u = blockIdx.x, ti = blockIdx.y;
  const int row = blockIdx.z * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int qt = 2 * p.unit_qp[u] + ti;
  if (qt >= p.n_q_tiles) return;
  const int tok = qt * BM + row;
  if (tok >= p.Lc) return;
  const int k0 = p.slot_begin[u], k1 = p.slot_begin[u + 1];
  float M = -INFINITY;
  for (int k = k0; k < k1; ++k)
    M = fmaxf(M, p.part_ml[(((int64_t)p.slots[k] * 2 + ti) * BM + row) * 2]);
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float Lsum = 0.f;
  for (int k = k0; k < k1; ++k) {
    const int64_t r = ((int64_t)p.slots[k] * 2 + ti) * BM + row;
    const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + r * 2);
    const float w = exp2f(ml.x - M);
    Lsum += w * ml.y;
    const float* src = p.part_o + r * HD + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += w * src[e];
  }
  const float inv = 1.f / Lsum;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                       (((int64_t)p.unit_b[u] * p.Lc + tok) * p.H + p.unit_h[u]) * HD + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t*>(dst + e) = ptx::pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

template <int HD>
cudaError_t launch_tc(const AttnParams& ap, const CUtensorMap* tq, const CUtensorMap* tk,
                      const CUtensorMap* tv, void* partials, size_t partials_bytes, int num_sms,
                      cudaStream_t st, int* n_kernels) {
  using L = Layout<HD>;
  static unsigned configured = 0;  // one bit per device ordinal < 32
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<HD>,
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
  p.out = ap.out;
  p.status = ap.status;
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
  const size_t need = attend_partials_bytes(HD, G);
  p.split = partials != nullptr && partials_bytes >= need && total >= G;
  if (!p.split) G = (int)std::min<int64_t>(G, units);
  p.grid = G;
  p.part_o = static_cast<float*>(partials);
  p.part_ml = p.part_o ? p.part_o + (size_t)2 * G * 2 * BM * HD : nullptr;
  attend_tc_kernel<HD><<<G, kThreads, L::bytes, st>>>(*tq, *tk, *tv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int launched = 1;
  if (p.split) {
    // the units cut by CTA range boundaries, with the partial slot of each piece in key order
    CombineParams cp;
    memset(&cp, 0, sizeof(cp));
    cp.H = p.H;
    cp.Lc = p.Lc;
    cp.n_q_tiles = p.n_q_tiles;
    cp.part_o = p.part_o;
    cp.part_ml = p.part_ml;
    cp.out = p.out;
    struct Piece { int64_t unit_start; int lo; int slot; int b, h, qp; };
    std::vector<Piece> pieces;
    for (int c = 0; c < G; ++c) {
      int64_t r0, r1;
      cta_range(p, c, r0, r1);
      bool first = true;
      for (int64_t t = r0; t < r1;) {
        const Seg sg = make_seg(p, t, r1);
        if (sg.partial)
          pieces.push_back({t - sg.lo, sg.lo, 2 * c + (first ? 0 : 1), sg.b, sg.h, sg.qp});
        first = false;
        t = sg.t_end;
      }
    }
    std::stable_sort(pieces.begin(), pieces.end(), [](const Piece& x, const Piece& y) {
      return x.unit_start != y.unit_start ? x.unit_start < y.unit_start : x.lo < y.lo;
    });
    int nu = 0, ns = 0;
    for (size_t i = 0; i < pieces.size(); ++i) {
      if (i == 0 || pieces[i].unit_start != pieces[i - 1].unit_start) {
        if (nu >= kMaxCombine) return cudaErrorInvalidValue;
        cp.unit_b[nu] = pieces[i].b;
        cp.unit_h[nu] = pieces[i].h;
        cp.unit_qp[nu] = pieces[i].qp;
        cp.slot_begin[nu] = ns;
        ++nu;
      }
      if (ns >= 2 * kMaxCtas) return cudaErrorInvalidValue;
      cp.slots[ns++] = pieces[i].slot;
    }
    cp.slot_begin[nu] = ns;
    cp.n_units = nu;
    if (nu > 0) {
      combine_kernel<HD><<<dim3(nu, 2, BM / 8), 256, 0, st>>>(cp);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      ++launched;
    }
  }
  if (n_kernels) *n_kernels = launched;
  return cudaSuccess;
}

}  // namespace

size_t attend_partials_bytes(int D, int num_sms) {
  const size_t G = (size_t)std::min(num_sms, kMaxCtas);
  return 2 * G * 2 * BM * ((size_t)D * 4 + 8);
}

cudaError_t launch_attend_tc_bf16(const AttnParams& p, int D, const CUtensorMap* tm_q,
                                  const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                  void* partials, size_t partials_bytes, int num_sms,
                                  cudaStream_t st, int* n_kernels) {
  if (D == 128)
    return launch_tc<128>(p, tm_q, tm_k, tm_v, partials, partials_bytes, num_sms, st, n_kernels);
  if (D == 64)
    return launch_tc<64>(p, tm_q, tm_k, tm_v, partials, partials_bytes, num_sms, st, n_kernels);
  return cudaErrorInvalidValue;
}

}  // namespace sa
