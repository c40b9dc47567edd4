// dfp_selftest_wait_timeout: the bounded-wait machinery of the kernels, exercised on purpose.
//
// Every mbarrier wait in libdfp's kernels gives up after a fixed number of SM clocks,
// records an error code in a device word and lets the kernel wind down, so a lost arrival
// becomes an error status on the host instead of a hung GPU.  This entry point runs one
// thread that waits, through the same mbar_wait, on an mbarrier that nothing will ever
// arrive on, and returns the code the wait recorded (and the wait's duration), with the
// CUDA context still usable afterwards.
#include <chrono>

#include "../../include/dfp.h"
#include "dfp_common.cuh"

namespace {

__global__ void wait_for_nothing_kernel(int* err, long long* cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  dfp::mbar_init(dfp::smem_u32(&bar), 1);
  dfp::fence_mbar_init();
  const long long t0 = clock64();
  const bool ok = dfp::mbar_wait(dfp::smem_u32(&bar), 0, err, dfp::kErrWaitTmaFull);   // nobody arrives
  *cycles = clock64() - t0;
  if (ok) atomicExch(err, -1);   // would mean the wait returned without its phase completing
}

}  // namespace

extern "C" DFP_API dfp_status dfp_selftest_wait_timeout(int* code_out, long long* cycles_out) {
  if (!code_out) return DFP_E_ARG;
  int* d_err = nullptr;
  long long* d_cyc = nullptr;
  cudaError_t e = cudaMalloc(&d_err, sizeof(int));
  if (e == cudaSuccess) e = cudaMalloc(&d_cyc, sizeof(long long));
  if (e == cudaSuccess) e = cudaMemset(d_err, 0, sizeof(int));
  if (e == cudaSuccess) {
    wait_for_nothing_kernel<<<1, 32>>>(d_err, d_cyc);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int code = 0;
  long long cyc = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&code, d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&cyc, d_cyc, sizeof(long long), cudaMemcpyDeviceToHost);
  if (d_err) cudaFree(d_err);
  if (d_cyc) cudaFree(d_cyc);
  if (e != cudaSuccess) return DFP_E_CUDA;
  *code_out = code;
  if (cycles_out) *cycles_out = cyc;
  return DFP_OK;
}
