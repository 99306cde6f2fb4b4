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
  unsigned long long wait_ns;     // limit of every bounded pipeline wait
  int stall;                      // diagnostic: withhold one pipeline step (PACK3D_FLAG_DIAG_STALL)
  int sa_build;                   // query x summary build: 0 by size, 1 one-tile, 2 two-tile
  int origin[3];                  // lattice origin: rotation angles use origin[a] + c_a
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

// ---- 2^x on the FMA pipe ----------------------------------------------------
// For a pair: x = n + f with n = rint(x) (added to the float's exponent field)
// and f in [-1/2, 1/2], 2^f from a cubic whose coefficients are the minimax
// fit of the relative error by the Remez exchange (fit_exp2.py next to this
// library reproduces them); the largest relative error of the float Horner
// evaluation is 7.5e-5, far below bf16's 3.9e-3.  Inputs are clamped at -125
// so the result stays a normal float (about 2.4e-38 in place of 0).
__device__ __forceinline__ float2 exp2_fma(float2 x) {
  constexpr float kC0 = 0.99992806f, kC1 = 0.69326097f, kC2 = 0.24261113f, kC3 = 0.055171669f;
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23: adding it rounds to an integer
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(f, make_float2(kC3, kC3), make_float2(kC2, kC2));
  p = __ffma2_rn(p, f, make_float2(kC1, kC1));
  p = __ffma2_rn(p, f, make_float2(kC0, kC0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// ---- axial RoPE tables -----------------------------------------------------
// Table layout (float2 = cos, sin): plane p owns the contiguous entries
// [pair_off[p], pair_off[p] + extent of its axis), one per local coordinate
// value c; the entry holds the angle of the coordinate origin[axis] + c.
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
    tab[e] = rope_cos_sin(s.omega[p] * (double)(e - s.pair_off[p] + s.origin[s.pair_axis[p]]));
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
// directly, without the integer-coordinate tables.  The coordinate is the
// rotation frame's (callers add the lattice origin).
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

// Rotates the 2*np values f (planes p0 .. p0+np-1) of one row at the lattice
// site (z, y, x) by R(c) (transpose = false) or by R(c)^T (transpose = true),
// reading the per-CTA table.  R(c)^T is the RoPE backward: each active pair
// (y0, y1) becomes (y0 cos t + y1 sin t, -y0 sin t + y1 cos t).
__device__ __forceinline__ void rope_planes(float* f, const Shape& s, const float2* tab, int p0, int np, int z,
                                            int y, int x, bool transpose) {
  const float sg = transpose ? -1.f : 1.f;
#pragma unroll
  for (int k = 0; k < np; ++k) {
    const int p = p0 + k;
    if (p >= s.npairs) break;
    const int ax = s.pair_axis[p];
    const int cval = ax == 0 ? z : (ax == 1 ? y : x);
    const float2 cs = tab[s.pair_off[p] + cval];
    const float sn = sg * cs.y;
    const float x0 = f[2 * k], x1 = f[2 * k + 1];
    f[2 * k] = x0 * cs.x - x1 * sn;
    f[2 * k + 1] = x0 * sn + x1 * cs.x;
  }
}

// Training epilogue of a query x summary row (the gate's backward): with
// gamma = softmax(gate row), A = <dout, o_loc> and B = <dout, o_cmp>,
//   dgate = (gamma0 (A - m), gamma1 (B - m)),  m = gamma0 A + gamma1 B,
// and the row statistics the branches' backward reads: stats[4 row + 1] =
// lse2 of the compressed softmax, [4 row + 2] = gamma0 A = <gamma0 dout, o_loc>
// and [4 row + 3] = gamma1 B (the softmax-backward deltas of the two branches;
// [4 row] holds the local branch's lse2, written by the local kernel).
template <typename T>
__device__ __forceinline__ void train_epilogue_row(const float* o_cmp, const float* __restrict__ gate,
                                                   const float* __restrict__ oloc, const T* __restrict__ dout,
                                                   size_t row, float lse2, float* __restrict__ stats,
                                                   float* __restrict__ dgate) {
  constexpr int NE = Elem<T>::kPerChunk;
  const float g0 = __ldg(gate + 2 * row), g1 = __ldg(gate + 2 * row + 1);
  const float gm = fmaxf(g0, g1);
  const float e0 = expf(g0 - gm), e1 = expf(g1 - gm);
  const float w0 = e0 / (e0 + e1), w1 = e1 / (e0 + e1);
  const float* lo = oloc + row * kDh;
  float A = 0.f, B = 0.f;
#pragma unroll
  for (int c = 0; c < kDh / NE; ++c) {
    float f[NE];
    chunk_to_float(ldg16(dout + row * kDh + c * NE), f, T());
#pragma unroll
    for (int k = 0; k < NE; ++k) {
      A = fmaf(f[k], __ldg(lo + c * NE + k), A);
      B = fmaf(f[k], o_cmp[c * NE + k], B);
    }
  }
  const float m = w0 * A + w1 * B;
  *reinterpret_cast<float2*>(dgate + 2 * row) = make_float2(w0 * (A - m), w1 * (B - m));
  stats[4 * row + 1] = lse2;
  stats[4 * row + 2] = w0 * A;
  stats[4 * row + 3] = w1 * B;
}

// Gate weights (gamma0, gamma1) = softmax(gate row).
__device__ __forceinline__ float2 gate_weights(const float* __restrict__ gate, size_t row) {
  const float g0 = __ldg(gate + 2 * row), g1 = __ldg(gate + 2 * row + 1);
  const float gm = fmaxf(g0, g1);
  const float e0 = expf(g0 - gm), e1 = expf(g1 - gm);
  return make_float2(e0 / (e0 + e1), e1 / (e0 + e1));
}

__device__ __forceinline__ void set_err(int32_t* err, int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace pack3d
