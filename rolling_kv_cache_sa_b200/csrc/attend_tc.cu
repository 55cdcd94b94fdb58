// attend_tc.cu -- bf16 flash attention over the visible key prefix of each
// (stream, head) of the rolling cache, on the sm_100a tensor cores.
//
// One CTA = one 128-row query tile of one (stream, head); 8 warps:
//   warp 0     : TMA producer (Q tile once, then K and V tiles, kStages each)
//   warp 1     : TMEM allocator + single-thread tcgen05.mma issuer
//   warps 4..7 : softmax, one thread per query row (TMEM lane = row), then
//                the epilogue
// TMEM (512 columns): S double buffer at columns [0,128) and [128,256), the
// O accumulator at [256, 256 + D). P_j (bf16) overwrites the first 64
// columns of its own S buffer once S_j is in registers.
// Per key tile j:  S[j%2] = Q' K'_j^T (SS MMA, K = D) -> softmax reads S,
// writes P_j into TMEM -> O += P_j V_j (TS MMA: A = P from TMEM, B = V as an
// MN-major shared-memory operand). MMAs issued by one thread execute in
// order, so QK_{j+2}, issued after PV_j, cannot overwrite P_j before PV_j has
// read it. The online softmax keeps a per-row running max in the log2 domain
// and only rescales O (in TMEM) when the max grows by more than 8 (a factor
// 256), which keeps P in bf16 range and makes the rescale rare; the final
// division by the row sum is exact.
// Every wait is bounded (about 1 s); on expiry the CTA records a device error,
// drains its outstanding copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {
namespace {

constexpr int BM = 128;                  // query rows per tile
constexpr int BN = 128;                  // keys per tile
constexpr uint32_t PANEL = 128u * 128u;  // one 128-row x 128-byte swizzled panel
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HD>
struct Layout {
  static constexpr int kStages = HD == 128 ? 3 : 4;
  static constexpr uint32_t kPanels = HD / 64;
  static constexpr uint32_t kTile = kPanels * PANEL;  // Q, K or V tile bytes
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k0 = q + kTile;
  static constexpr uint32_t v0 = k0 + kStages * kTile;
  static constexpr uint32_t bars = v0 + kStages * kTile;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr uint32_t kNumBars = 1 + 4 * kStages + 6;
  static constexpr uint32_t misc = bars + kNumBars * 8;
  static constexpr uint32_t bytes = misc + 16;
  static constexpr uint32_t alloc = bytes + 1024;  // slack to align the base to 1024
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;
  static constexpr int B_KE = B_KF + kStages;
  static constexpr int B_VF = B_KE + kStages;
  static constexpr int B_VE = B_VF + kStages;
  static constexpr int B_SF = B_VE + kStages;  // 2: S buffer written by QK
  static constexpr int B_PF = B_SF + 2;        // 2: P written into the S buffer
  static constexpr int B_OD = B_PF + 2;        // PV done
  static constexpr int B_DR = B_OD + 1;        // drain
};

template <int HD>
__global__ void __launch_bounds__(256, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ AttnParams p) {
  using L = Layout<HD>;
  constexpr int ST = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const uint32_t sQ = base + L::q;
  const uint32_t bar0 = base + L::bars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = blockIdx.z;
  const int b = p.stream_of[a];
  const int h = blockIdx.y;
  const int qt = blockIdx.x;
  const int n_keys = p.n_keys[a];
  const int nkv = (n_keys + BN - 1) / BN;
  const int bh = b * p.H + h;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(L::B_Q), 1);
    for (int s = 0; s < ST; ++s) {
      ptx::mbar_init(bar(L::B_KF + s), 1);
      ptx::mbar_init(bar(L::B_KE + s), 1);
      ptx::mbar_init(bar(L::B_VF + s), 1);
      ptx::mbar_init(bar(L::B_VE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(L::B_SF + s), 1);
      ptx::mbar_init(bar(L::B_PF + s), 128);
    }
    ptx::mbar_init(bar(L::B_OD), 1);
    ptx::mbar_init(bar(L::B_DR), 1);
    *abort_flag = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_q);
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      ptx::mbar_arrive_expect_tx(bar(L::B_Q), L::kTile);
      for (uint32_t pn = 0; pn < L::kPanels; ++pn)
        ptx::tma_load_3d(sQ + pn * PANEL, &tm_q, bar(L::B_Q), (int)pn * 64, qt * BM, bh);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % ST;
        const uint32_t u = (uint32_t)(j / ST);
        if (u > 0 && !ptx::mbar_wait(bar(L::B_KE + s), (u - 1) & 1, abort_flag, kTimeoutNs)) {
          fail();
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(L::B_KF + s), L::kTile);
        for (uint32_t pn = 0; pn < L::kPanels; ++pn)
          ptx::tma_load_3d(base + L::k0 + s * L::kTile + pn * PANEL, &tm_k, bar(L::B_KF + s),
                           (int)pn * 64, j * BN, bh);
        if (u > 0 && !ptx::mbar_wait(bar(L::B_VE + s), (u - 1) & 1, abort_flag, kTimeoutNs)) {
          fail();
          issued = 2 * j + 1;
          break;
        }
        ptx::mbar_arrive_expect_tx(bar(L::B_VF + s), L::kTile);
        for (uint32_t pn = 0; pn < L::kPanels; ++pn)
          ptx::tma_load_3d(base + L::v0 + s * L::kTile + pn * PANEL, &tm_v, bar(L::B_VF + s),
                           (int)pn * 64, j * BN, bh);
        issued = 2 * j + 2;
      }
      // drain: every issued copy has landed before the CTA may exit
      ptx::mbar_wait(bar(L::B_Q), 0, abort_flag, kTimeoutNs);
      for (int t = issued - 1; t >= 0 && t >= issued - 2 * ST; --t) {
        const int j = t >> 1;
        const int which = (t & 1) ? L::B_VF : L::B_KF;
        ptx::mbar_wait(bar(which + j % ST), (uint32_t)(j / ST) & 1, abort_flag, kTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(BM, HD, true);
      bool ok = ptx::mbar_wait(bar(L::B_Q), 0, abort_flag, kTimeoutNs);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j % ST;
          const uint32_t u = (uint32_t)(j / ST);
          if (!ptx::mbar_wait(bar(L::B_KF + s), u & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem + (uint32_t)(j & 1) * 128u;
          const uint32_t kb = base + L::k0 + s * L::kTile;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * PANEL + (uint32_t)(kk & 3) * 32u;
            ptx::umma_ss(d_tmem, ptx::sdesc_sw128(sQ + off, 16, 1024),
                         ptx::sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar(L::B_SF + (j & 1)));
          ptx::umma_commit(bar(L::B_KE + s));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % ST;
          const uint32_t u = (uint32_t)(jj / ST);
          if (!ptx::mbar_wait(bar(L::B_VF + s), u & 1, abort_flag, kTimeoutNs)) { ok = false; break; }
          if (!ptx::mbar_wait(bar(L::B_PF + (jj & 1)), (uint32_t)(jj >> 1) & 1, abort_flag,
                              kTimeoutNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t pt = tmem + (uint32_t)(jj & 1) * 128u;
          const uint32_t vb = base + L::v0 + s * L::kTile;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            ptx::umma_ts(tmem + 256u, pt + (uint32_t)kk * 8u,
                         ptx::sdesc_sw128(vb + (uint32_t)kk * 2048u, PANEL, 1024), idesc_pv,
                         (jj > 0 || kk > 0) ? 1u : 0u);
          ptx::umma_commit(bar(L::B_OD));
          ptx::umma_commit(bar(L::B_VE + s));
        }
      }
      if (!ok) fail();
      // drain: all MMAs issued by this thread have completed
      ptx::umma_commit(bar(L::B_DR));
      ptx::mbar_wait(bar(L::B_DR), 0, abort_flag, kTimeoutNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_used = 0.f, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const uint32_t sbuf = t_lane + (uint32_t)s * 128u;
      // waits are made warp-uniform: the TMEM accesses below are .sync.aligned
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_SF + s), (uint32_t)(j >> 1) & 1,
                                                  abort_flag, kTimeoutNs))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) ptx::tmem_ld32(sbuf + c * 32, sv + c * 32);
      ptx::tmem_wait_ld();

      const int valid = n_keys - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i >= valid) sv[i] = -INFINITY;
      }
      // row max: eight independent chains, then a tree
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = sv[i];
#pragma unroll
      for (int i = 8; i < BN; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
#pragma unroll
      for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int i = 0; i < w2; ++i) mx8[i] = fmaxf(mx8[i], mx8[i + w2]);
      const float m_tile = mx8[0] * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_used = m_tile;
      } else if (m_tile > m_used + kRescaleThreshold) {
        alpha = ptx::ex2(m_used - m_tile);
        m_used = m_tile;
        rescale = true;
      }
      // P_j = exp2(S * scale * log2e - m) as bf16 pairs into the S buffer's
      // first 64 columns (this thread's lane = its row)
      float ls8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls8[i] = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ptx::ex2(fmaf(sv[c * 32 + 2 * e], sl2, -m_used));
          const float p1 = ptx::ex2(fmaf(sv[c * 32 + 2 * e + 1], sl2, -m_used));
          ls8[e & 7] += p0 + p1;
          w[e] = ptx::pack_bf16x2(p0, p1);
        }
        ptx::tmem_st16u(sbuf + (uint32_t)c * 16u, w);
      }
#pragma unroll
      for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int i = 0; i < w2; ++i) ls8[i] += ls8[i + w2];
      l = l * alpha + ls8[0];
      if (j >= 1) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled or accumulated into
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar(L::B_OD), (uint32_t)(j - 1) & 1,
                                                    abort_flag, kTimeoutNs))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float ov[32];
            ptx::tmem_ld32(t_lane + 256u + c * 32, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            ptx::tmem_st32(t_lane + 256u + c * 32, ov);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(L::B_PF + s));
    }
    if (ok && nkv > 0 &&
        !__all_sync(0xffffffffu,
                    ptx::mbar_wait(bar(L::B_OD), (uint32_t)(nkv - 1) & 1, abort_flag, kTimeoutNs)))
      ok = false;
    if (!ok) {
      fail();
    } else {
      ptx::tc_fence_after();
      const int tok = qt * BM + row;
      const float inv = 1.f / l;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                           (((int64_t)b * p.Lc + tok) * p.H + h) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float ov[32];
        ptx::tmem_ld32(t_lane + 256u + c * 32, ov);
        ptx::tmem_wait_ld();
        if (tok < p.Lc) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 v;
            v.x = ptx::pack_bf16x2(ov[g * 8 + 0] * inv, ov[g * 8 + 1] * inv);
            v.y = ptx::pack_bf16x2(ov[g * 8 + 2] * inv, ov[g * 8 + 3] * inv);
            v.z = ptx::pack_bf16x2(ov[g * 8 + 4] * inv, ov[g * 8 + 5] * inv);
            v.w = ptx::pack_bf16x2(ov[g * 8 + 6] * inv, ov[g * 8 + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c * 32 + g * 8) = v;
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

template <int HD>
cudaError_t launch_tc(const AttnParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                      const CUtensorMap* tv, cudaStream_t st) {
  using L = Layout<HD>;
  static unsigned configured = 0;  // one bit per device ordinal < 32
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 32 || !(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::alloc);
    if (e != cudaSuccess) return e;
    if (dev < 32) configured |= 1u << dev;
  }
  dim3 grid((unsigned)p.n_q_tiles, (unsigned)p.H, (unsigned)p.n_streams);
  attend_tc_kernel<HD><<<grid, 256, L::alloc, st>>>(*tq, *tk, *tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc_bf16(const AttnParams& p, int D, const CUtensorMap* tm_q,
                                  const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                  cudaStream_t st) {
  if (D == 128) return launch_tc<128>(p, tm_q, tm_k, tm_v, st);
  if (D == 64) return launch_tc<64>(p, tm_q, tm_k, tm_v, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
