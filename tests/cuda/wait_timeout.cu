// Test-only kernels for the library's bounded mbarrier wait (puro::mbar_wait): a wait on
// a barrier whose phase never completes must give up after its limit and return false;
// a wait on a completed phase must return true at once. No fault, trap or endless loop.
#include <cuda_runtime.h>
#include <cstdint>

#include "../../fp8_blockwise_scaled_e4m3_b200/csrc/ptx.cuh"

namespace {

// out[0] = wait result on a barrier nothing arrives on; out[1] = elapsed ns;
// out[2] = wait result after the only expected arrival; out[3] = elapsed ns.
__global__ void k_wait(unsigned long long timeout_ns, unsigned long long *out) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    puro::mbar_init(puro::smem_u32(&bar[0]), 1);
    puro::mbar_init(puro::smem_u32(&bar[1]), 1);
    abort_flag = 0;
    puro::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  uint64_t t0 = puro::globaltimer_ns();
  const bool never = puro::mbar_wait(puro::smem_u32(&bar[0]), 0, timeout_ns, &abort_flag);
  uint64_t t1 = puro::globaltimer_ns();
  out[0] = never;
  out[1] = t1 - t0;
  puro::mbar_arrive(puro::smem_u32(&bar[1]));
  t0 = puro::globaltimer_ns();
  const bool done = puro::mbar_wait(puro::smem_u32(&bar[1]), 0, timeout_ns, &abort_flag);
  t1 = puro::globaltimer_ns();
  out[2] = done;
  out[3] = t1 - t0;
}

}  // namespace

extern "C" int run_wait_check(unsigned long long timeout_ns, unsigned long long *host_out) {
  unsigned long long *d = nullptr;
  if (cudaMalloc(&d, 4 * sizeof(unsigned long long)) != cudaSuccess) return 1;
  k_wait<<<1, 32>>>(timeout_ns, d);
  if (cudaGetLastError() != cudaSuccess) return 2;
  if (cudaMemcpy(host_out, d, 4 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return 3;
  cudaFree(d);
  return 0;
}
