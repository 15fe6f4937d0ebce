// Test-only probe of the bounded mbarrier wait used by every product kernel
// (newton_schulz_matrix_b200/csrc/tc_common.cuh).  One thread waits on an
// mbarrier that, unless `arrive` is set, nothing ever completes; the wait must
// give up after `timeout_ns`, raise the CTA-wide abort flag and return false,
// leaving the context usable.  No copies or MMAs are in flight.
#include <cuda_runtime.h>

#include "../../newton_schulz_matrix_b200/csrc/tc_common.cuh"

using namespace muon::tc;

__global__ void wait_probe_kernel(long long timeout_ns, int arrive, long long* out) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(smem_u32(&bar));
    const uint64_t t0 = global_timer();
    const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, timeout_ns);
    out[0] = ok ? 1 : 0;
    out[1] = abort_flag;
    out[2] = (long long)(global_timer() - t0);
  }
}

extern "C" int run_wait_probe(long long timeout_ns, int arrive, long long* host_out) {
  long long* d = nullptr;
  if (cudaMalloc(&d, 3 * sizeof(long long)) != cudaSuccess) return 1;
  wait_probe_kernel<<<1, 32>>>(timeout_ns, arrive, d);
  cudaError_t e = cudaMemcpy(host_out, d, 3 * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e == cudaSuccess ? 0 : 2;
}
