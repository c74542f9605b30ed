// diag.cu -- diagnostic entry point: evaluates the kernels' device exp2
// helpers on caller data so tests can check them against the hardware exp2.
#include "../../include/gqe.h"
#include "sm100.cuh"

namespace gqe {
namespace {

__global__ void exp2_diag_kernel(const float* __restrict__ x, float* y_poly, float* y_pair, float* y_hw, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = x[i];
  y_poly[i] = exp2_poly(v);
  float a, b;
  exp2_poly2(f2_pack(v, v), a, b);
  y_pair[i] = (a == b) ? a : __int_as_float(0x7fc00000);   // both lanes must agree
  y_hw[i] = ex2(v);
}

// One thread waits, through the kernels' own bounded wait, on an mbarrier that
// nothing ever arrives at: after the wait limit it records kErrTimeoutDebug in
// the error word and the kernel returns normally.
__global__ void debug_wait_kernel(unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    volatile int* abort = &abort_flag;
    mbar_wait(&bar, 0, abort, err, kErrTimeoutDebug);
  }
}

}  // namespace

cudaError_t launch_debug_wait(unsigned* err, cudaStream_t stream) {
  debug_wait_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace gqe

extern "C" gqe_status gqe_debug_exp2(const float* x, float* y_poly, float* y_pair, float* y_hw, int n,
                                     gqe_stream stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_pair || !y_hw))) return GQE_ERR_INVALID_ARG;
  if (n == 0) return GQE_OK;
  gqe::exp2_diag_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y_poly, y_pair,
                                                                                             y_hw, n);
  return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}
