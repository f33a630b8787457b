// Diagnostic entry point: evaluates the attention kernel's polynomial 2^x on
// a caller buffer, so tests can check it against its error bound.
#include "exp2_poly.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

__global__ void exp2_poly_kernel(const float *x, float *y, int64_t n) {
  for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.0f;
    float r0, r1;
    unf2(ex2_poly2(f2(a, b)), r0, r1);
    y[i] = r0;
    if (i + 1 < n) y[i + 1] = r1;
  }
}

}  // namespace
}  // namespace wf

extern "C" wf_status wf_debug_exp2_poly(const float *x, float *y, int64_t n, wf_stream_t stream) {
  if (!x || !y || n < 0) return WF_ERR_INVALID_ARG;
  if (n == 0) return WF_OK;
  const int64_t pairs = (n + 1) / 2;
  const int blocks = static_cast<int>(pairs / 256 + 1 < 4096 ? pairs / 256 + 1 : 4096);
  wf::exp2_poly_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}
