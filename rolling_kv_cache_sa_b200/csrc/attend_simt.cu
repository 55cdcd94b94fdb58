// attend_simt.cu -- fp32 attention over each (stream, head)'s visible key
// prefix, for the fp32 configuration (tensor-core tf32 cannot hold 1e-4).
//
// Block = 8 warps, 16 query rows of one (stream, head); each warp owns 2
// rows. Keys and values stream through shared memory 32 at a time. For one
// tile, lane j computes the full score of key j against the warp's row, the
// row max and the row sum are warp-shuffle reductions, and the P.V update
// broadcasts p_j by shuffle while each lane accumulates D/32 output dims.
// Online softmax in fp32 with base-2 exponentials.
#include "internal.h"

namespace sa {

// debug build: the bounds word of this file (sites: 0 stream / key prefix of
// a (stream, head), 1 output row)
SA_DEFINE_BOUNDS_WORD(bounds_word_attend_simt)

namespace {

constexpr int kRows = 16;  // query rows per block
constexpr int kKeys = 32;  // keys per tile

template <int D>
__global__ void __launch_bounds__(256) attend_simt_kernel(const __grid_constant__ AttnParams p) {
  constexpr int DP = D + 1;  // padded key row: lane j reads row j conflict-free
  constexpr int PER_LANE = D / 32;
  __shared__ float sq[kRows][D];
  __shared__ float sk[kKeys][DP];
  __shared__ float sv[kKeys][D];

  const int a = blockIdx.z;
  const int b = p.stream_of[a];
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * kRows;
  const int n_keys = p.n_keys[a];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // (block-uniform: the whole block leaves before any barrier)
  if (!SA_BOUNDS(b >= 0 && b < p.batch && n_keys >= 0 && n_keys <= p.ntok, 0)) return;
  const int64_t bh = (int64_t)b * p.H + h;
  const float* q = static_cast<const float*>(p.q_ws) + bh * p.Lc * D;
  const float* kc = static_cast<const float*>(p.k_cache) + bh * p.ntok * D;
  const float* vc = static_cast<const float*>(p.v_cache) + bh * p.ntok * D;

  for (int i = threadIdx.x; i < kRows * D; i += blockDim.x) {
    const int r = i / D, d = i % D;
    sq[r][d] = row0 + r < p.Lc ? q[(int64_t)(row0 + r) * D + d] : 0.f;
  }

  float m[2], l[2], o[2][PER_LANE];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) o[rr][c] = 0.f;
  }

  for (int k0 = 0; k0 < n_keys; k0 += kKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeys * D; i += blockDim.x) {
      const int r = i / D, d = i % D;
      const bool ok = k0 + r < n_keys;
      sk[r][d] = ok ? kc[(int64_t)(k0 + r) * D + d] : 0.f;
      sv[r][d] = ok ? vc[(int64_t)(k0 + r) * D + d] : 0.f;
    }
    __syncthreads();
    const bool key_ok = k0 + lane < n_keys;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp * 2 + rr;
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) s = fmaf(sq[r][d], sk[lane][d], s);
      s = key_ok ? s * p.scale_log2 : -INFINITY;
      float mx = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[rr], mx);
      const float alpha = exp2f(m[rr] - m_new);  // 0 on the first tile (m = -inf)
      const float pj = exp2f(s - m_new);
      float sum = pj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[rr] = l[rr] * alpha + sum;
      m[rr] = m_new;
#pragma unroll
      for (int c = 0; c < PER_LANE; ++c) o[rr][c] *= alpha;
#pragma unroll 4
      for (int jj = 0; jj < kKeys; ++jj) {
        const float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
        for (int c = 0; c < PER_LANE; ++c) o[rr][c] = fmaf(pb, sv[jj][lane + 32 * c], o[rr][c]);
      }
    }
  }

  float* out = static_cast<float*>(p.out);
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int tok = row0 + warp * 2 + rr;
    if (tok >= p.Lc) continue;
    if (!SA_BOUNDS(h < p.H, 1)) continue;
    const float inv = 1.f / l[rr];
    float* dst = out + (((int64_t)b * p.Lc + tok) * p.H + h) * D;
#pragma unroll
    for (int c = 0; c < PER_LANE; ++c) dst[lane + 32 * c] = o[rr][c] * inv;
  }
}

}  // namespace

cudaError_t launch_attend_simt_f32(const AttnParams& p, int D, cudaStream_t st) {
  dim3 grid((unsigned)((p.Lc + kRows - 1) / kRows), (unsigned)p.H, (unsigned)p.n_streams);
  if (D == 64)
    attend_simt_kernel<64><<<grid, 256, 0, st>>>(p);
  else if (D == 128)
    attend_simt_kernel<128><<<grid, 256, 0, st>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace sa
