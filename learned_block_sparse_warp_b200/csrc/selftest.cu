// Diagnostics: the bounded wait's timeout path, on demand.
//
// Every mbarrier wait in the tcgen05 kernels goes through sm100::mbar_wait,
// which gives up after about one second of clock cycles, raises
// SAS_ERR_TIMEOUT in the device error word and returns. This kernel runs that
// same wait on an mbarrier that nothing ever completes, so a caller can check
// that the timeout is reported and that the context stays usable afterwards.
// Nothing faults, traps or spins without a bound.
#include "sm100.cuh"

namespace sas {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(int* err) {
  using namespace sm100;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x != 0) return;
  abort_s = 0;
  mbar_init(smem_u32(&bar), 1);  // one arrival expected, none ever made
  fence_barrier_init();
  mbar_wait(smem_u32(&bar), 0, &abort_s, err);  // returns false after the bound, with SAS_ERR_TIMEOUT raised
}

cudaError_t launch_wait_timeout(int* err, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

}  // namespace sas
