// Memory-bound stages of the PACK3D forward pass on sm_100a:
//   - the grid-to-packed index map and block membership,
//   - axial grid RoPE on Q and K ("Geometry Matters in Packed 3D Attention",
//     Key design 1, equation R(c)),
//   - rotate-before-compress block summaries (Key design 2, equations k~_j^R
//     and v~_j).
// All three stream 16-byte chunks with several loads in flight per thread; the
// RoPE and summary kernels first build the per-axis cos/sin tables in shared
// memory so that no transcendental is evaluated per element.
#include "common.cuh"
#include "internal.h"

namespace pack3d {

// ---- index map ---------------------------------------------------------

__global__ void fill_i32_kernel(int32_t* __restrict__ p, int n, int32_t v) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

// One thread per token: scatter its packed index to its lattice site and to
// its slot in its block.  A repeated site is caught by the exchange returning
// a previous owner.
__global__ void index_kernel(Shape s, const int32_t* __restrict__ coords, int32_t* __restrict__ g2p,
                             int32_t* __restrict__ members, int32_t* err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= s.N) return;
  const int z = coords[3 * i], y = coords[3 * i + 1], x = coords[3 * i + 2];
  if (z < 0 || z >= s.Z || y < 0 || y >= s.H || x < 0 || x >= s.W) {
    set_err(err, PACK3D_DEVERR_COORD_RANGE);
    return;
  }
  const int site = (z * s.H + y) * s.W + x;
  if (atomicExch(&g2p[site], i) != -1) set_err(err, PACK3D_DEVERR_DUPLICATE);
  const int j = ((z / s.bz) * s.nby + y / s.by) * s.nbx + x / s.bx;
  const int t = ((z % s.bz) * s.by + y % s.by) * s.bx + x % s.bx;
  members[j * s.v + t] = i;
}

cudaError_t launch_build_index(const Shape& s, const int32_t* coords, int32_t* g2p,
                               int32_t* members, int32_t* err, cudaStream_t st) {
  // Both maps start at -1 so that a slot no valid token claims (bad input)
  // is recognisable downstream and never dereferenced.
  fill_i32_kernel<<<min((s.N + 255) / 256, 148 * 8), 256, 0, st>>>(g2p, s.N, -1);
  fill_i32_kernel<<<min((s.M * s.v + 255) / 256, 148 * 8), 256, 0, st>>>(members, s.M * s.v, -1);
  index_kernel<<<(s.N + 255) / 256, 256, 0, st>>>(s, coords, g2p, members, err);
  return cudaGetLastError();
}

// ---- axial RoPE ----------------------------------------------------------

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;

// Rotates up to two tensors (e.g. Q and K_loc) in one launch; y may alias x.
template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(Shape s, const int32_t* __restrict__ coords,
                                                            const T* x0, T* y0, int h0,
                                                            const T* x1, T* y1, int h1) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int CPR = kDh / NE;  // chunks per head row
  const unsigned stride = gridDim.x * blockDim.x;
  for (int t = 0; t < 2; ++t) {
    const T* x = t ? x1 : x0;
    T* y = t ? y1 : y0;
    const int heads = t ? h1 : h0;
    if (x == nullptr) continue;
    const unsigned per_tok = (unsigned)heads * CPR;
    const unsigned total = (unsigned)s.N * per_tok;
    for (unsigned base = blockIdx.x * blockDim.x + threadIdx.x; base < total;
         base += kRopeUnroll * stride) {
      uint4 u[kRopeUnroll];
#pragma unroll
      for (int k = 0; k < kRopeUnroll; ++k) {
        const unsigned c = base + k * stride;
        if (c < total) u[k] = *reinterpret_cast<const uint4*>(x + (size_t)c * NE);
      }
#pragma unroll
      for (int k = 0; k < kRopeUnroll; ++k) {
        const unsigned c = base + k * stride;
        if (c >= total) continue;
        const unsigned tok = c / per_tok;
        const int part = c % CPR;
        // Clamped so that a bad coordinate (reported by the index map) cannot
        // index outside the tables.
        const int cz = min(max(__ldg(coords + 3 * tok), 0), s.Z - 1);
        const int cy = min(max(__ldg(coords + 3 * tok + 1), 0), s.H - 1);
        const int cx = min(max(__ldg(coords + 3 * tok + 2), 0), s.W - 1);
        float f[NE];
        chunk_to_float(u[k], f, T());
        rotate_chunk<NE>(f, part * NE, tab, s, cz, cy, cx);
        stg16(y + (size_t)c * NE, float_to_chunk(f, T()));
      }
    }
  }
}

static int rope_grid(const Shape& s, int heads, int chunk_elems) {
  long chunks = (long)s.N * heads * (kDh / chunk_elems);
  long want = (chunks + kRopeThreads * kRopeUnroll - 1) / (kRopeThreads * kRopeUnroll);
  return (int)max(1L, min(want, 148L * 6));
}

template <typename T>
static cudaError_t rope_t(const Shape& s, const int32_t* coords, const void* x0, void* y0, int h0,
                          const void* x1, void* y1, int h1, cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = cudaFuncSetAttribute(rope_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int grid = rope_grid(s, h0 + (x1 ? h1 : 0), Elem<T>::kPerChunk);
  rope_kernel<T><<<grid, kRopeThreads, smem, st>>>(
      s, coords, (const T*)x0, (T*)y0, h0, (const T*)x1, (T*)y1, h1);
  return cudaGetLastError();
}

cudaError_t launch_rope(const Shape& s, int dtype, const int32_t* coords, const void* x0, void* y0,
                        int h0, const void* x1, void* y1, int h1, cudaStream_t st) {
  if (dtype == PACK3D_BF16) return rope_t<__nv_bfloat16>(s, coords, x0, y0, h0, x1, y1, h1, st);
  return rope_t<float>(s, coords, x0, y0, h0, x1, y1, h1, st);
}

// ---- rotate-before-compress summaries ----------------------------------

constexpr int kSumThreads = 256;

// A unit is (block j, kv head g, K or V); kDh/NE lanes share a unit, each lane
// owning one 16-byte chunk of the 64 dims.  Member t of block j sits at the
// t-th raster site of the block, so its coordinates follow from (j, t).
template <typename T>
__global__ void __launch_bounds__(kSumThreads) summaries_kernel(
    Shape s, const int32_t* __restrict__ members, const T* __restrict__ kc,
    const T* __restrict__ vc, const float* __restrict__ scores, T* __restrict__ ks,
    T* __restrict__ vs) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int LPU = kDh / NE;
  const int units_per_cta = kSumThreads / LPU;
  const long units = (long)s.M * s.Hkv * 2;
  const int part = threadIdx.x % LPU;
  for (long ub = (long)blockIdx.x * units_per_cta; ub < units; ub += (long)gridDim.x * units_per_cta) {
    const long u = ub + threadIdx.x / LPU;
    if (u >= units) continue;
    const int is_v = (int)(u & 1);
    const long jg = u >> 1;
    const int g = (int)(jg % s.Hkv);
    const int j = (int)(jg / s.Hkv);
    const int32_t* mem = members + (size_t)j * s.v;
    const int jx = j % s.nbx, jy = (j / s.nbx) % s.nby, jz = j / (s.nbx * s.nby);
    // a_{j,u}: softmax of the block's scores for kv head g.
    // Members left at -1 (only possible for coordinates that are not a
    // bijection, which the index map reports) are skipped.
    float smax = -INFINITY;
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m >= 0) smax = fmaxf(smax, __ldg(scores + (size_t)m * s.Hkv + g));
    }
    float den = 0.f;
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m >= 0) den += expf(__ldg(scores + (size_t)m * s.Hkv + g) - smax);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const T* src = is_v ? vc : kc;
    float acc[NE];
#pragma unroll
    for (int k = 0; k < NE; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m < 0) continue;
      const float a = expf(__ldg(scores + (size_t)m * s.Hkv + g) - smax) * inv;
      const uint4 c = ldg16(src + ((size_t)m * s.Hkv + g) * kDh + part * NE);
      float f[NE];
      chunk_to_float(c, f, T());
      if (!is_v) {
        const int tz = t / (s.by * s.bx), ty = (t / s.bx) % s.by, tx = t % s.bx;
        rotate_chunk<NE>(f, part * NE, tab, s, jz * s.bz + tz, jy * s.by + ty, jx * s.bx + tx);
      }
#pragma unroll
      for (int k = 0; k < NE; ++k) acc[k] = fmaf(a, f[k], acc[k]);
    }
    T* dst = is_v ? vs : ks;
    stg16(dst + ((size_t)j * s.Hkv + g) * kDh + part * NE, float_to_chunk(acc, T()));
  }
}

template <typename T>
static cudaError_t summaries_t(const Shape& s, const int32_t* members, const void* kc, const void* vc,
                               const float* scores, void* ks, void* vs, cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = cudaFuncSetAttribute(summaries_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int lpu = kDh / Elem<T>::kPerChunk;
  const long units = (long)s.M * s.Hkv * 2;
  const long per_cta = kSumThreads / lpu;
  const int grid = (int)max(1L, min((units + per_cta - 1) / per_cta, 148L * 8));
  summaries_kernel<T><<<grid, kSumThreads, smem, st>>>(s, members, (const T*)kc, (const T*)vc, scores,
                                                        (T*)ks, (T*)vs);
  return cudaGetLastError();
}

cudaError_t launch_summaries(const Shape& s, int dtype, const int32_t* members, const void* kc,
                             const void* vc, const float* scores, void* ks, void* vs,
                             cudaStream_t st) {
  if (dtype == PACK3D_BF16)
    return summaries_t<__nv_bfloat16>(s, members, kc, vc, scores, ks, vs, st);
  return summaries_t<float>(s, members, kc, vc, scores, ks, vs, st);
}

}  // namespace pack3d
