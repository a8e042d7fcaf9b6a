// Diagnostic entry point: the prefill kernel's FMA-pipe exponential
// (exp2_poly.cuh) and the MUFU ex2.approx instruction, evaluated on the
// caller's inputs, so that tests can check the polynomial on the device
// against exact 2^x and against the hardware instruction.
#include <cuda_runtime.h>

#include "exp2_poly.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

// Thread i evaluates inputs 2i and 2i + 1 as one pair, the way the prefill
// kernel feeds exp2_poly2; an odd last input is paired with itself.
__global__ void __launch_bounds__(256) exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                                            float* __restrict__ y_mufu, int n) {
  const long long i = 2LL * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool pair = i + 1 < n;
  const float x0 = x[i], x1 = pair ? x[i + 1] : x0;
  const float2 p = exp2_poly2(make_float2(x0, x1));
  y_poly[i] = p.x;
  if (y_mufu) y_mufu[i] = ex2_approx(x0);
  if (pair) {
    y_poly[i + 1] = p.y;
    if (y_mufu) y_mufu[i + 1] = ex2_approx(x1);
  }
}

}  // namespace
}  // namespace attn

extern "C" attn_status_t attn_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int n, attn_stream_t stream) {
  if (n < 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  if (!x || !y_poly) return ATTN_ERR_INVALID_ARG;
  attn_status_t st = attn::check_device();
  if (st != ATTN_OK) return st;
  const long long pairs = (n + 1LL) / 2;
  const long long blocks = (pairs + 255) / 256;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  attn::exp2_selftest_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu,
                                                                                                    n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
