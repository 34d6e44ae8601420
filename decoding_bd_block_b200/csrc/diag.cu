// Diagnostic entry point: evaluates the library's own exponential
// approximations on caller-given arguments, so that tests can hold them to
// their stated error bounds on the device they run on.
#include "bd_common.cuh"

namespace bd {
namespace {

// grid-stride over n arguments: y_poly = poly_exp2(x), y_pair = poly_exp2x2
// on the pair (x[2i], x[2i+1]) (the last odd element alone), y_mufu =
// ex2.approx (fast_exp2).
__global__ void eval_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                 float* __restrict__ y_pair, float* __restrict__ y_mufu, int n) {
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    y_poly[i] = poly_exp2(x[i]);
    y_mufu[i] = fast_exp2(x[i]);
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; 2 * i < n; i += stride) {
    const float a = x[2 * i], b = 2 * i + 1 < n ? x[2 * i + 1] : 0.f;
    const float2 r = poly_exp2x2(make_float2(a, b));
    y_pair[2 * i] = r.x;
    if (2 * i + 1 < n) y_pair[2 * i + 1] = r.y;
  }
}

}  // namespace
}  // namespace bd

extern "C" int bd_eval_exp2(const float* x, float* y_poly, float* y_pair, float* y_mufu,
                            int32_t n, void* stream) {
  if (!x || !y_poly || !y_pair || !y_mufu || n < 0) return BD_ERR_INVALID_ARG;
  if (n == 0) return BD_OK;
  bd::eval_exp2_kernel<<<148, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_pair,
                                                                            y_mufu, n);
  bd::count_launches(1);
  return bd::report_cuda_error(cudaGetLastError());
}
