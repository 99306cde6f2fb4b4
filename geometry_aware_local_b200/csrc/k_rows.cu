// Row gather for the z-slab split of one volume over several ranks
// ("Geometry Matters in Packed 3D Attention", Key design 3: a query's local
// window reaches r_z planes into the neighbouring slab, so each rank sends the
// local keys and values of its boundary planes).  The rows of those planes,
// found through the slab's grid-to-packed map, are packed into one contiguous
// buffer in raster order: dst row i = src row idx[i] (a negative index gives a
// zero row).  Rows are whole multiples of 16 bytes; each thread moves one
// 16-byte chunk, so the copy is coalesced on the destination side.
#include "common.cuh"
#include "internal.h"

namespace pack3d {
namespace {

__global__ void __launch_bounds__(256) gather_rows_kernel(const int32_t* __restrict__ idx, long long n,
                                                          const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          int chunks) {
  const long long total = n * chunks;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total;
       c += (long long)gridDim.x * blockDim.x) {
    const long long r = c / chunks;
    const int k = (int)(c - r * chunks);
    const int s = __ldg(idx + r);
    dst[c] = s >= 0 ? __ldg(src + (long long)s * chunks + k) : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

cudaError_t launch_gather_rows(const int32_t* idx, long long n, const void* src, void* dst, long long row_bytes,
                               cudaStream_t st) {
  const int chunks = (int)(row_bytes / 16);
  const long long total = n * chunks;
  const long long want = (total + 255) / 256;
  const int grid = (int)(want < 148LL * 8 ? (want > 0 ? want : 1) : 148LL * 8);
  gather_rows_kernel<<<grid, 256, 0, st>>>(idx, n, (const uint4*)src, (uint4*)dst, chunks);
  return cudaGetLastError();
}

}  // namespace pack3d
