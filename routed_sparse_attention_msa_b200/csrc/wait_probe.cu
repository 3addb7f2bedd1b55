// A kernel whose bounded wait nothing ends, for testing the failure path of
// the tensor-core kernels without faulting the GPU: one thread waits on an
// mbarrier no one arrives on; the wait runs out (2 s), records the error in
// this file's flag and returns, and msa_sync_check reports MSA_ERR_TIMEOUT.
#include "msa_internal.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

using namespace tc;

__global__ void wait_probe_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0, &abort_flag);
}

}  // namespace

msa_status launch_wait_probe(cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>();
  return launch_check("wait probe");
}

int probe_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa
