// Diagnostic evaluation of the FMA-pipe exponential (exp2_fma, common.cuh)
// that the one-tile query x summary kernel uses for a share of its softmax
// exponentials: y[i] = 2^x[i] for float x, two elements per call as in the
// kernel.  It lets the tests check the approximation against a reference
// over the whole input range the kernel feeds it.
#include "common.cuh"
#include "internal.h"

namespace pack3d {
namespace {

__global__ void __launch_bounds__(256) exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y,
                                                       long long n) {
  for (long long i = 2 * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n;
       i += 2LL * gridDim.x * blockDim.x) {
    const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
    const float2 r = exp2_fma(v);
    y[i] = r.x;
    if (i + 1 < n) y[i + 1] = r.y;
  }
}

}  // namespace

cudaError_t launch_exp2_fma_eval(const float* x, float* y, long long n, cudaStream_t st) {
  const long long want = (n / 2 + 255) / 256 + 1;
  const int grid = (int)(want < 148LL * 8 ? want : 148LL * 8);
  exp2_fma_kernel<<<grid, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace pack3d
