// Failure path of the tensor-core kernels' bounded waits, exercised without a
// fault: one CTA allocates tensor memory the way the kernels do, waits on an
// mbarrier that nothing ever arrives on (hadq::tc::mbar_wait, the kernels'
// own wait), and must come back after the wait limit, record where it gave
// up, free the tensor memory and exit, leaving the context usable.
#include <cstdint>

#include "hadq_tc.cuh"

namespace {

__global__ void wait_timeout_kernel(unsigned int* result, unsigned long long* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    hadq::tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(hadq::tc::smem_u32(&tmem_slot)), "r"(32));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  hadq::tc::tc_fence_before();
  __syncthreads();
  hadq::tc::tc_fence_after();
  if (threadIdx.x == 0) {
    const uint64_t t0 = hadq::tc::globaltimer_ns();
    const bool completed = hadq::tc::mbar_wait(&bar, 0);   // phase 0 never completes
    waited_ns[0] = hadq::tc::globaltimer_ns() - t0;
    if (!completed) atomicOr(&hadq::tc::hadq_tc_fault, hadq::tc::kFaultEpilogue);
    result[0] = completed ? 1u : 2u;
  }
  hadq::tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    hadq::tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_slot), "r"(32));
  }
}

}  // namespace

// result[0]: 2 = the wait gave up (expected), 1 = it completed; waited_ns[0]:
// how long it waited; fault: the kernel's fault word after the launch.
extern "C" __attribute__((visibility("default"))) int run_wait_timeout(unsigned int* result_host,
                                                                      unsigned long long* waited_host,
                                                                      unsigned int* fault_host) {
  unsigned int* r = nullptr;
  unsigned long long* w = nullptr;
  if (cudaMalloc(&r, sizeof(unsigned int)) != cudaSuccess) return 1;
  if (cudaMalloc(&w, sizeof(unsigned long long)) != cudaSuccess) return 2;
  const unsigned int zero = 0;
  cudaMemcpyToSymbol(hadq::tc::hadq_tc_fault, &zero, sizeof(zero));
  cudaMemset(r, 0, sizeof(unsigned int));
  wait_timeout_kernel<<<1, 128>>>(r, w);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return 10 + static_cast<int>(e);
  cudaMemcpy(result_host, r, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaMemcpy(waited_host, w, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaMemcpyFromSymbol(fault_host, hadq::tc::hadq_tc_fault, sizeof(unsigned int));
  cudaFree(r);
  cudaFree(w);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
