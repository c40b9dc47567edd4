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
#include "exp2_poly.cuh"

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

// 2^x of consecutive pairs through the attention softmax's polynomial (exp2_poly.cuh),
// as fp32 and as the truncated bf16 pairs the softmax stores.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, uint32_t* __restrict__ y_bf16,
                                 int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const uint64_t x2 = dfp::f2(x[i], two ? x[i + 1] : 0.f);
  uint32_t r0, r1;
  dfp::ex2_poly_pair_f32(x2, r0, r1);
  y[i] = __uint_as_float(r0);
  if (two) y[i + 1] = __uint_as_float(r1);
  if (y_bf16) {
    const uint32_t b = dfp::ex2_poly_pair_bf16(x2);
    if (two) y_bf16[i / 2] = b;
    else reinterpret_cast<uint16_t*>(y_bf16)[i] = (uint16_t)(b & 0xFFFFu);
  }
}

}  // namespace

extern "C" DFP_API dfp_status dfp_selftest_exp2_poly(const float* x, float* y, void* y_bf16, int n, void* stream) {
  if (n < 0 || n > (1 << 30)) return DFP_E_ARG;
  if (n == 0) return DFP_OK;
  if (!x || !y) return DFP_E_ARG;
  if (y_bf16 && (reinterpret_cast<uintptr_t>(y_bf16) & 3)) return DFP_E_ARG;
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y, static_cast<uint32_t*>(y_bf16), n);
  return cudaGetLastError() == cudaSuccess ? DFP_OK : DFP_E_CUDA;
}

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
