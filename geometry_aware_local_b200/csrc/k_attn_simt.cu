// CUDA-core attention kernels of the PACK3D forward pass on sm_100a.
//
// local_attn_kernel: exact local attention ("Geometry Matters in Packed 3D
// Attention", Key design 3).  CTAs walk the lattice in 1 x 8 x 8 bricks of
// query sites, not the packed order, so the clipped 3D windows of a brick
// overlap in L1 whatever the packing is.  Every neighbour is reached through
// the grid-to-packed map; no gathered neighbour tensor exists.  One thread
// owns one (query, head) row: the G heads of a site are adjacent lanes and read
// the same key/value rows.  Float accumulation, online softmax in base 2.
//
// summary_attn_simt_kernel: every query against all M summaries (Key design 3)
// with the tokenwise gate (overall framework) in the epilogue.  This is the
// float path (the bf16 path runs on tcgen05 tensor cores); summary tiles are
// staged in shared memory as float and read by broadcast.
#include "common.cuh"
#include "internal.h"

namespace pack3d {

constexpr int kBrickY = 8, kBrickX = 8, kBrickSites = kBrickY * kBrickX;

template <typename T>
__device__ __forceinline__ void load_row_f32(const T* p, float* f) {
  constexpr int NE = Elem<T>::kPerChunk;
#pragma unroll
  for (int c = 0; c < kDh / NE; ++c) chunk_to_float(ldg16(p + c * NE), f + c * NE, T());
}

template <typename T, int G>
__global__ void __launch_bounds__(kBrickSites * G) local_attn_kernel(
    Shape s, const int32_t* __restrict__ g2p, const T* __restrict__ qr, const T* __restrict__ kr,
    const T* __restrict__ vl, float* __restrict__ oloc, float* __restrict__ stats) {
  constexpr int NE = Elem<T>::kPerChunk;
  const int bricks_x = (s.W + kBrickX - 1) / kBrickX;
  const int bricks_y = (s.H + kBrickY - 1) / kBrickY;
  const int b = blockIdx.x;
  const int z = b / (bricks_x * bricks_y);
  const int y = ((b / bricks_x) % bricks_y) * kBrickY + (threadIdx.x / G) / kBrickX;
  const int x = (b % bricks_x) * kBrickX + (threadIdx.x / G) % kBrickX;
  if (y >= s.H || x >= s.W) return;
  const int g = blockIdx.y;
  const int h = g * G + threadIdx.x % G;
  const int i = __ldg(g2p + (z * s.H + y) * s.W + x);
  if (i < 0) return;  // site no token claimed: invalid coordinates, already reported

  float q[kDh];
  load_row_f32(qr + ((size_t)i * s.Hq + h) * kDh, q);
#pragma unroll
  for (int e = 0; e < kDh; ++e) q[e] *= s.scale_log2;

  float m = -INFINITY, l = 0.f, acc[kDh];
#pragma unroll
  for (int e = 0; e < kDh; ++e) acc[e] = 0.f;

  const int z0 = max(0, z - s.rz), z1 = min(s.Z - 1, z + s.rz);
  const int y0 = max(0, y - s.ry), y1 = min(s.H - 1, y + s.ry);
  const int x0 = max(0, x - s.rx), x1 = min(s.W - 1, x + s.rx);
  for (int zz = z0; zz <= z1; ++zz)
    for (int yy = y0; yy <= y1; ++yy) {
      const int32_t* grow = g2p + (zz * s.H + yy) * s.W;
      for (int xx = x0; xx <= x1; ++xx) {
        const int jj = __ldg(grow + xx);
        if (jj < 0) continue;
        const size_t j = (size_t)jj;
        const T* krow = kr + (j * s.Hkv + g) * kDh;
        float sd = 0.f;
#pragma unroll
        for (int c = 0; c < kDh / NE; ++c) {
          float f[NE];
          chunk_to_float(ldg16(krow + c * NE), f, T());
#pragma unroll
          for (int k = 0; k < NE; ++k) sd = fmaf(q[c * NE + k], f[k], sd);
        }
        if (sd > m) {
          const float corr = exp2f(m - sd);
          l *= corr;
#pragma unroll
          for (int e = 0; e < kDh; ++e) acc[e] *= corr;
          m = sd;
        }
        const float p = exp2f(sd - m);
        l += p;
        const T* vrow = vl + (j * s.Hkv + g) * kDh;
#pragma unroll
        for (int c = 0; c < kDh / NE; ++c) {
          float f[NE];
          chunk_to_float(ldg16(vrow + c * NE), f, T());
#pragma unroll
          for (int k = 0; k < NE; ++k) acc[c * NE + k] = fmaf(p, f[k], acc[c * NE + k]);
        }
      }
    }
  const float inv = 1.f / l;
  if (stats) stats[4 * ((size_t)i * s.Hq + h)] = m + log2f(l);
  float* o = oloc + ((size_t)i * s.Hq + h) * kDh;
#pragma unroll
  for (int c = 0; c < kDh / 4; ++c)
    *reinterpret_cast<float4*>(o + 4 * c) =
        make_float4(acc[4 * c] * inv, acc[4 * c + 1] * inv, acc[4 * c + 2] * inv, acc[4 * c + 3] * inv);
}

template <typename T, int G>
static cudaError_t local_t(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                           const void* vl, float* oloc, cudaStream_t st, float* stats) {
  const int bricks = s.Z * ((s.H + kBrickY - 1) / kBrickY) * ((s.W + kBrickX - 1) / kBrickX);
  dim3 grid(bricks, s.Hkv);
  local_attn_kernel<T, G><<<grid, kBrickSites * G, 0, st>>>(s, g2p, (const T*)qr, (const T*)kr,
                                                            (const T*)vl, oloc, stats);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t local_g(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                           const void* vl, float* oloc, cudaStream_t st, float* stats) {
  switch (s.G) {
    case 1: return local_t<T, 1>(s, g2p, qr, kr, vl, oloc, st, stats);
    case 2: return local_t<T, 2>(s, g2p, qr, kr, vl, oloc, st, stats);
    case 4: return local_t<T, 4>(s, g2p, qr, kr, vl, oloc, st, stats);
    case 8: return local_t<T, 8>(s, g2p, qr, kr, vl, oloc, st, stats);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_local_attn(const Shape& s, int dtype, const int32_t* g2p, const void* qr,
                              const void* kr, const void* vl, float* oloc, cudaStream_t st, float* stats) {
  if (dtype == PACK3D_BF16) return local_g<__nv_bfloat16>(s, g2p, qr, kr, vl, oloc, st, stats);
  return local_g<float>(s, g2p, qr, kr, vl, oloc, st, stats);
}

// ---- query x summary, CUDA cores ----------------------------------------

constexpr int kSaRows = 128, kSaTile = 32;

template <typename T>
__device__ __forceinline__ void store_row(T* dst, const float* f) {
  constexpr int NE = Elem<T>::kPerChunk;
#pragma unroll
  for (int c = 0; c < kDh / NE; ++c) stg16(dst + c * NE, float_to_chunk(f + c * NE, T()));
}

// Gate epilogue shared by both query x summary kernels' float results:
// out = softmax(gate)[0] * o_loc + softmax(gate)[1] * o_cmp, or o_cmp alone.
__device__ __forceinline__ void gate_mix_row(float* o, const float* __restrict__ gate,
                                             const float* __restrict__ oloc, size_t row) {
  if (gate == nullptr) return;
  const float g0 = __ldg(gate + 2 * row), g1 = __ldg(gate + 2 * row + 1);
  const float gm = fmaxf(g0, g1);
  const float e0 = expf(g0 - gm), e1 = expf(g1 - gm);
  const float w0 = e0 / (e0 + e1), w1 = e1 / (e0 + e1);
  const float* lo = oloc + row * kDh;
#pragma unroll
  for (int c = 0; c < kDh / 4; ++c) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(lo) + c);
    o[4 * c] = w0 * a.x + w1 * o[4 * c];
    o[4 * c + 1] = w0 * a.y + w1 * o[4 * c + 1];
    o[4 * c + 2] = w0 * a.z + w1 * o[4 * c + 2];
    o[4 * c + 3] = w0 * a.w + w1 * o[4 * c + 3];
  }
}

template <typename T>
__global__ void __launch_bounds__(kSaRows) summary_attn_simt_kernel(
    Shape s, const T* __restrict__ qr, const T* __restrict__ ks, const T* __restrict__ vs,
    const float* __restrict__ oloc, const float* __restrict__ gate, T* __restrict__ out,
    float* __restrict__ stats, const T* __restrict__ dout, float* __restrict__ dgate) {
  __shared__ float Ksh[kSaTile][kDh], Vsh[kSaTile][kDh];
  const int g = blockIdx.y;
  const long rows = (long)s.N * s.G;
  const long r = (long)blockIdx.x * kSaRows + threadIdx.x;
  const bool valid = r < rows;
  const long tok = valid ? r / s.G : 0;
  const int h = g * s.G + (int)(r % s.G);
  const size_t orow = (size_t)tok * s.Hq + h;

  float q[kDh];
  load_row_f32(qr + orow * kDh, q);
#pragma unroll
  for (int e = 0; e < kDh; ++e) q[e] *= s.scale_log2;
  float m = -INFINITY, l = 0.f, acc[kDh];
#pragma unroll
  for (int e = 0; e < kDh; ++e) acc[e] = 0.f;

  for (int j0 = 0; j0 < s.M; j0 += kSaTile) {
    const int nj = min(kSaTile, s.M - j0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nj * kDh; idx += kSaRows) {
      const int jj = idx / kDh, e = idx % kDh;
      const size_t off = ((size_t)(j0 + jj) * s.Hkv + g) * kDh + e;
      Ksh[jj][e] = (float)ks[off];
      Vsh[jj][e] = (float)vs[off];
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      float sd = 0.f;
#pragma unroll
      for (int e = 0; e < kDh; ++e) sd = fmaf(q[e], Ksh[jj][e], sd);
      if (sd > m) {
        const float corr = exp2f(m - sd);
        l *= corr;
#pragma unroll
        for (int e = 0; e < kDh; ++e) acc[e] *= corr;
        m = sd;
      }
      const float p = exp2f(sd - m);
      l += p;
#pragma unroll
      for (int e = 0; e < kDh; ++e) acc[e] = fmaf(p, Vsh[jj][e], acc[e]);
    }
  }
  if (!valid) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < kDh; ++e) acc[e] *= inv;
  if (stats) train_epilogue_row(acc, gate, oloc, dout, orow, m + log2f(l), stats, dgate);
  gate_mix_row(acc, gate, oloc, orow);
  store_row(out + orow * kDh, acc);
}

cudaError_t launch_summary_attn_simt(const Shape& s, int dtype, const void* qr, const void* ks,
                                     const void* vs, const float* oloc, const float* gate,
                                     void* out, cudaStream_t st, const Train* tr) {
  const long rows = (long)s.N * s.G;
  dim3 grid((unsigned)((rows + kSaRows - 1) / kSaRows), s.Hkv);
  float* stats = tr ? tr->stats : nullptr;
  float* dgate = tr ? tr->dgate : nullptr;
  const void* dout = tr ? tr->dout : nullptr;
  if (dtype == PACK3D_BF16)
    summary_attn_simt_kernel<__nv_bfloat16><<<grid, kSaRows, 0, st>>>(
        s, (const __nv_bfloat16*)qr, (const __nv_bfloat16*)ks, (const __nv_bfloat16*)vs, oloc, gate,
        (__nv_bfloat16*)out, stats, (const __nv_bfloat16*)dout, dgate);
  else
    summary_attn_simt_kernel<float><<<grid, kSaRows, 0, st>>>(s, (const float*)qr, (const float*)ks,
                                                              (const float*)vs, oloc, gate,
                                                              (float*)out, stats, (const float*)dout, dgate);
  return cudaGetLastError();
}

}  // namespace pack3d
