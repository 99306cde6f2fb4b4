// Shared device helpers of the PACK3D sm_100a kernels: the resolved shape
// passed to every kernel, bf16/float row access and the per-CTA shared-memory
// cos/sin tables of the axial grid RoPE ("Geometry Matters in Packed 3D
// Attention", Key design 1, equation R(c)).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pack3d.h"

namespace pack3d {

constexpr int kDh = 64;           // head dim supported by every kernel
constexpr int kMaxPairs = kDh / 2;
constexpr int kMaxTableBytes = 96 * 1024;

// Everything a kernel needs about one operator instance, resolved on the host.
struct Shape {
  int Z, H, W, N, M;
  int Hq, Hkv, G;                 // G = Hq / Hkv query heads per kv head
  int bz, by, bx, v;              // block dims and volume
  int nbz, nby, nbx;              // block grid
  int rz, ry, rx;                 // window radii
  int mz, my, mx;                 // rotary planes per axis
  int tab_entries;                // Z*mz + H*my + W*mx
  int npairs;                     // mz + my + mx rotated planes
  float scale;                    // softmax scale
  float scale_log2;               // scale * log2(e)
  double omega[kMaxPairs];        // per rotary plane p: base^(-r/m_axis), 0 if unused
  int pair_axis[kMaxPairs];       // 0 = z, 1 = y, 2 = x, 3 = untouched
  int pair_off[kMaxPairs];        // first table entry of plane p
  int center;                     // summaries: rotate the pooled key at the block centre
};

Shape make_shape(const pack3d_config& c);

// ---- element access ------------------------------------------------------

template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerChunk = 4;  // elements per 16-byte chunk
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
};

// 16-byte chunk <-> float values.
__device__ __forceinline__ void chunk_to_float(const uint4& u, float* f, float) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ void chunk_to_float(const uint4& u, float* f, __nv_bfloat16) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}
__device__ __forceinline__ uint4 float_to_chunk(const float* f, float) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 float_to_chunk(const float* f, __nv_bfloat16) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void stg16(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}

// ---- axial RoPE tables -----------------------------------------------------
// Table layout (float2 = cos, sin): plane p owns the contiguous entries
// [pair_off[p], pair_off[p] + extent of its axis), one per coordinate value.
// The angle omega * c is formed in double and reduced modulo 2*pi in double
// (a two-part 2*pi, Cody-Waite style), so the float sincos sees an argument in
// [-pi, pi].

__device__ __forceinline__ float2 rope_cos_sin(double angle) {
  const double kTwoPiHi = 6.283185307179586;       // nearest double to 2*pi
  const double kTwoPiLo = 2.4492935982947064e-16;  // 2*pi - kTwoPiHi
  const double k = rint(angle * 0.15915494309189535);
  double r = fma(-k, kTwoPiHi, angle);
  r = fma(-k, kTwoPiLo, r);
  float s, c;
  sincosf((float)r, &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ int axis_extent(const Shape& s, int axis) {
  return axis == 0 ? s.Z : (axis == 1 ? s.H : s.W);
}

// All threads fill the table together: entry e belongs to the last plane whose
// first entry is <= e (a binary search over the increasing pair_off).
__device__ __forceinline__ void build_rope_table(float2* tab, const Shape& s) {
  for (int e = threadIdx.x; e < s.tab_entries; e += blockDim.x) {
    int p = 0;
#pragma unroll
    for (int step = kMaxPairs / 2; step > 0; step >>= 1)
      if (p + step < s.npairs && s.pair_off[p + step] <= e) p += step;
    tab[e] = rope_cos_sin(s.omega[p] * (double)(e - s.pair_off[p]));
  }
}

// Per-thread lookup constants for the NP planes starting at plane p0 (the
// planes one 16-byte chunk covers): axis and first table entry.
template <int NP>
struct PlaneLut {
  int axis[NP];
  int off[NP];
  __device__ __forceinline__ void init(const Shape& s, int p0) {
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const int p = p0 + k;
      axis[k] = p < s.npairs ? s.pair_axis[p] : 3;
      off[k] = p < s.npairs ? s.pair_off[p] : 0;
    }
  }
  // Rotates the 2*NP values f (planes p0 .. p0+NP-1) at coordinate (z, y, x).
  __device__ __forceinline__ void rotate(float* f, const float2* tab, int z, int y, int x) const {
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      if (axis[k] == 3) continue;
      const int cval = axis[k] == 0 ? z : (axis[k] == 1 ? y : x);
      const float2 cs = tab[off[k] + cval];
      const float x0 = f[2 * k], x1 = f[2 * k + 1];
      f[2 * k] = x0 * cs.x - x1 * cs.y;
      f[2 * k + 1] = x0 * cs.y + x1 * cs.x;
    }
  }
};

// Rotates the 2*NP values f (planes p0 .. p0+NP-1) by R at the coordinate
// (z, y, x), which may be fractional (a block centre): the angles are formed
// directly, without the integer-coordinate tables.
template <int NP>
__device__ __forceinline__ void rotate_at(float* f, const Shape& s, int p0, double z, double y, double x) {
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    const int p = p0 + k;
    if (p >= s.npairs || s.pair_axis[p] == 3) continue;
    const int a = s.pair_axis[p];
    const float2 cs = rope_cos_sin(s.omega[p] * (a == 0 ? z : (a == 1 ? y : x)));
    const float x0 = f[2 * k], x1 = f[2 * k + 1];
    f[2 * k] = x0 * cs.x - x1 * cs.y;
    f[2 * k + 1] = x0 * cs.y + x1 * cs.x;
  }
}

__device__ __forceinline__ void set_err(int32_t* err, int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace pack3d
