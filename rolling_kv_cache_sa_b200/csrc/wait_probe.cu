// wait_probe.cu -- exercises, on the GPU, the bounded mbarrier wait that every
// kernel of the library uses, without any fault: two warps wait on a barrier
// that nothing ever completes. Warp 0 gives up after the short limit, sets
// the CTA's abort flag and the device error word; warp 1 has a limit 20 times
// longer and must leave early because it watches the abort flag. Each warp
// records how long it waited (%globaltimer).
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {
namespace {

struct ProbeOut {
  int status;
  int pad_;
  unsigned long long waited_ns[2];
};

__device__ ProbeOut g_probe;

__global__ void __launch_bounds__(64, 1) wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  __shared__ volatile int no_abort;
  const uint32_t b = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    abort_flag = 0;
    no_abort = 0;
    g_probe.status = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const uint64_t t0 = ptx::globaltimer();
  if (warp == 0) {
    if (!ptx::mbar_wait(b, 0, &no_abort, limit_ns)) {
      abort_flag = 1;
      if (threadIdx.x == 0) atomicOr(&g_probe.status, kDeviceErrTimeout);
    }
  } else {
    ptx::mbar_wait(b, 0, &abort_flag, 20 * limit_ns);
  }
  const uint64_t t1 = ptx::globaltimer();
  if ((threadIdx.x & 31) == 0) g_probe.waited_ns[warp] = t1 - t0;
}

}  // namespace

cudaError_t run_wait_probe(uint64_t limit_ns, cudaStream_t st, int* status,
                           unsigned long long waited_ns[2]) {
  wait_probe_kernel<<<1, 64, 0, st>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ProbeOut h;
  e = cudaMemcpyFromSymbolAsync(&h, g_probe, sizeof(h), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  *status = h.status;
  waited_ns[0] = h.waited_ns[0];
  waited_ns[1] = h.waited_ns[1];
  return cudaSuccess;
}

}  // namespace sa
