// Backward pass of the PACK3D training block on sm_100a: CUDA-core kernels.
//
// "Geometry Matters in Packed 3D Attention" describes the operator as a fused
// forward/backward training block; these kernels give the gradients of
// L = <dout, out> by the chain rule through the forward stages in reverse:
// the tokenwise gate (its backward runs in the forward's query x summary
// epilogue, which also leaves per-row statistics), both softmax attention
// branches (Key design 3), the rotate-before-compress summaries (Key design
// 2) and the axial RoPE (Key design 1, applied transposed).
//
// For a softmax row over logits l_j = scale <q, k_j> with output
// o = sum_j P_j v_j and output gradient do, dl_j = P_j (<do, v_j> - delta)
// with delta = <do, o>; then dq = scale sum_j dl_j k_j, dk_j += scale dl_j q
// and dv_j += P_j do.  P_j is recomputed from the saved log-sum-exp (base 2,
// in units of the scaled logits: P_j = 2^(l_j log2(e) - lse2)); the local
// branch's do is gamma0 dout and the compressed branch's gamma1 dout, with
// gamma = softmax(gate row).
//
// Kernels:
//   summary_bwd_dq   one thread per query row, summary tiles staged in shared
//                    memory; writes the compressed part of dQ_rot (float).
//   summary_bwd_dkv  two threads per summary (one per half of d_h), query
//                    rows staged in shared memory 32 at a time, the rows of a
//                    kv head split over grid.z; float atomics into dk~, dv~.
//   local_bwd_dq     two threads per (query site, head) over its clipped box,
//                    adds the compressed part and applies R(c)^T: dQ.
//   local_bwd_dkv    two threads per key site (halves of d_h) over the queries
//                    whose box holds it (the box around the key: the window
//                    relation is symmetric), all q heads of the kv head;
//                    applies R(c)^T: dK_loc, and dV_loc.
//   summaries_bwd    one warp per (block, kv head), lane = rotary plane: dK_cmp = R(c_u)^T
//                    (a_u dk~), dV_cmp = a_u dv~, dscores = a_u (da_u - sum a da)
//                    with da_u = <dk~, R(c_u) k_u> + <dv~, v_u>; for the
//                    summary-centre variant R(c_u) is replaced by one R(cbar)
//                    on the pooled key: dK_cmp = a_u R(cbar)^T dk~ and
//                    da_u = <R(cbar)^T dk~, k_u> + <dv~, v_u>.
#include "common.cuh"
#include "internal.h"

namespace pack3d {
namespace {

// n (a multiple of the chunk width) values of a row as float.
template <typename T>
__device__ __forceinline__ void load_f32(const T* p, float* f, int n) {
  constexpr int NE = Elem<T>::kPerChunk;
#pragma unroll
  for (int c = 0; c < n / NE; ++c) chunk_to_float(ldg16(p + c * NE), f + c * NE, T());
}

template <typename T>
__device__ __forceinline__ void store_f32(T* p, const float* f, int n) {
  constexpr int NE = Elem<T>::kPerChunk;
#pragma unroll
  for (int c = 0; c < n / NE; ++c) stg16(p + c * NE, float_to_chunk(f + c * NE, T()));
}

cudaError_t set_table_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// ---- compressed branch, query side ----------------------------------------

constexpr int kDqRows = 128, kDqTile = 32;

template <typename T>
__global__ void __launch_bounds__(kDqRows) summary_bwd_dq_kernel(
    Shape s, const T* __restrict__ qr, const T* __restrict__ ks, const T* __restrict__ vs,
    const T* __restrict__ dout, const float* __restrict__ gate, const float* __restrict__ stats,
    float* __restrict__ dqr) {
  __shared__ float Ksh[kDqTile][kDh], Vsh[kDqTile][kDh];
  const int g = blockIdx.y;
  const long rows = (long)s.N * s.G;
  const long r = (long)blockIdx.x * kDqRows + threadIdx.x;
  const bool valid = r < rows;
  const long tok = valid ? r / s.G : 0;
  const int h = g * s.G + (int)(valid ? r % s.G : 0);
  const size_t orow = (size_t)tok * s.Hq + h;

  float q[kDh], dO[kDh], dq[kDh];
  load_f32(qr + orow * kDh, q, kDh);
  load_f32(dout + orow * kDh, dO, kDh);
  const float w1 = gate_weights(gate, orow).y;
#pragma unroll
  for (int e = 0; e < kDh; ++e) {
    q[e] *= s.scale_log2;
    dO[e] *= w1;
    dq[e] = 0.f;
  }
  const float lse2 = stats[4 * orow + 1], delta = stats[4 * orow + 3];

  for (int j0 = 0; j0 < s.M; j0 += kDqTile) {
    const int nj = min(kDqTile, s.M - j0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nj * kDh; idx += kDqRows) {
      const int jj = idx / kDh, e = idx % kDh;
      const size_t off = ((size_t)(j0 + jj) * s.Hkv + g) * kDh + e;
      Ksh[jj][e] = (float)ks[off];
      Vsh[jj][e] = (float)vs[off];
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      float sd = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < kDh; ++e) {
        sd = fmaf(q[e], Ksh[jj][e], sd);
        dp = fmaf(dO[e], Vsh[jj][e], dp);
      }
      const float ds = exp2f(sd - lse2) * (dp - delta);
#pragma unroll
      for (int e = 0; e < kDh; ++e) dq[e] = fmaf(ds, Ksh[jj][e], dq[e]);
    }
  }
  if (!valid) return;
  float4* o = reinterpret_cast<float4*>(dqr + orow * kDh);
#pragma unroll
  for (int c = 0; c < kDh / 4; ++c)
    o[c] = make_float4(s.scale * dq[4 * c], s.scale * dq[4 * c + 1], s.scale * dq[4 * c + 2], s.scale * dq[4 * c + 3]);
}

// ---- compressed branch, summary side --------------------------------------

constexpr int kDkvSums = 64, kDkvThreads = 2 * kDkvSums, kDkvStage = 32;
constexpr int kHalf = kDh / 2, kHalfPad = kHalf + 4;   // padded so the two halves sit in different banks

template <typename T>
__global__ void __launch_bounds__(kDkvThreads) summary_bwd_dkv_kernel(
    Shape s, const T* __restrict__ qr, const T* __restrict__ ks, const T* __restrict__ vs,
    const T* __restrict__ dout, const float* __restrict__ gate, const float* __restrict__ stats,
    long rows_per_split, float* __restrict__ dks, float* __restrict__ dvs) {
  __shared__ __align__(16) float Qs[kDkvStage][2][kHalfPad];
  __shared__ __align__(16) float Os[kDkvStage][2][kHalfPad];
  __shared__ float Ls[kDkvStage], Dl[kDkvStage];
  const int g = blockIdx.y;
  const int j = blockIdx.x * kDkvSums + (threadIdx.x >> 1);
  const int half = threadIdx.x & 1;
  const bool jvalid = j < s.M;
  float k[kHalf], v[kHalf], dk[kHalf], dv[kHalf];
  if (jvalid) {
    load_f32(ks + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, k, kHalf);
    load_f32(vs + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, v, kHalf);
  }
#pragma unroll
  for (int e = 0; e < kHalf; ++e) {
    if (!jvalid) k[e] = v[e] = 0.f;
    dk[e] = dv[e] = 0.f;
  }
  const long rows = (long)s.N * s.G;
  const long r0 = (long)blockIdx.z * rows_per_split;
  const long r1 = min(rows, r0 + rows_per_split);
  for (long rb = r0; rb < r1; rb += kDkvStage) {
    __syncthreads();
    {
      // Staging: thread = (row, quarter of d_h); q raw, do = gamma1 dout.
      const int rr = threadIdx.x >> 2, qd = threadIdx.x & 3;
      const long r = rb + rr;
      float fq[16], fo[16];
      if (r < r1) {
        const size_t orow = (size_t)(r / s.G) * s.Hq + g * s.G + (int)(r % s.G);
        load_f32(qr + orow * kDh + qd * 16, fq, 16);
        load_f32(dout + orow * kDh + qd * 16, fo, 16);
        const float w1 = gate_weights(gate, orow).y;
#pragma unroll
        for (int e = 0; e < 16; ++e) fo[e] *= w1;
        if (qd == 0) {
          Ls[rr] = stats[4 * orow + 1];
          Dl[rr] = stats[4 * orow + 3];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) fq[e] = fo[e] = 0.f;
        if (qd == 0) {
          Ls[rr] = INFINITY;   // P = 0 for rows past the split
          Dl[rr] = 0.f;
        }
      }
      float* dq = &Qs[rr][qd >> 1][(qd & 1) * 16];
      float* doo = &Os[rr][qd >> 1][(qd & 1) * 16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        dq[e] = fq[e];
        doo[e] = fo[e];
      }
    }
    __syncthreads();
    const int nr = (int)min((long)kDkvStage, r1 - rb);
    for (int rr = 0; rr < nr; ++rr) {
      const float4* q4 = reinterpret_cast<const float4*>(&Qs[rr][half][0]);
      const float4* o4 = reinterpret_cast<const float4*>(&Os[rr][half][0]);
      float sh = 0.f, ph = 0.f;
#pragma unroll
      for (int c = 0; c < kHalf / 4; ++c) {
        const float4 a = q4[c], b = o4[c];
        sh = fmaf(a.x, k[4 * c], fmaf(a.y, k[4 * c + 1], fmaf(a.z, k[4 * c + 2], fmaf(a.w, k[4 * c + 3], sh))));
        ph = fmaf(b.x, v[4 * c], fmaf(b.y, v[4 * c + 1], fmaf(b.z, v[4 * c + 2], fmaf(b.w, v[4 * c + 3], ph))));
      }
      sh += __shfl_xor_sync(0xffffffffu, sh, 1);
      ph += __shfl_xor_sync(0xffffffffu, ph, 1);
      const float p = exp2f(sh * s.scale_log2 - Ls[rr]);
      const float ds = p * (ph - Dl[rr]);
#pragma unroll
      for (int c = 0; c < kHalf / 4; ++c) {
        const float4 a = q4[c], b = o4[c];
        dk[4 * c] = fmaf(ds, a.x, dk[4 * c]);
        dk[4 * c + 1] = fmaf(ds, a.y, dk[4 * c + 1]);
        dk[4 * c + 2] = fmaf(ds, a.z, dk[4 * c + 2]);
        dk[4 * c + 3] = fmaf(ds, a.w, dk[4 * c + 3]);
        dv[4 * c] = fmaf(p, b.x, dv[4 * c]);
        dv[4 * c + 1] = fmaf(p, b.y, dv[4 * c + 1]);
        dv[4 * c + 2] = fmaf(p, b.z, dv[4 * c + 2]);
        dv[4 * c + 3] = fmaf(p, b.w, dv[4 * c + 3]);
      }
    }
  }
  if (!jvalid) return;
  float* pk = dks + ((size_t)j * s.Hkv + g) * kDh + half * kHalf;
  float* pv = dvs + ((size_t)j * s.Hkv + g) * kDh + half * kHalf;
#pragma unroll
  for (int e = 0; e < kHalf; ++e) {
    atomicAdd(pk + e, s.scale * dk[e]);
    atomicAdd(pv + e, dv[e]);
  }
}

// ---- local branch, query side ---------------------------------------------

constexpr int kBY = 8, kBX = 8, kBSites = kBY * kBX;

// Two threads per (query site of an 8 x 8 brick of one z layer, head), one
// per half of d_h; GT <= 2 heads per CTA, grid.z covers the rest of the kv group.
template <typename T, int GT>
__global__ void __launch_bounds__(2 * kBSites * GT) local_bwd_dq_kernel(
    Shape s, const int32_t* __restrict__ g2p, const T* __restrict__ qr, const T* __restrict__ kr,
    const T* __restrict__ vl, const T* __restrict__ dout, const float* __restrict__ gate,
    const float* __restrict__ stats, const float* __restrict__ dqr, T* __restrict__ dq_out) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  const int bx = (s.W + kBX - 1) / kBX, by = (s.H + kBY - 1) / kBY;
  const int b = blockIdx.x;
  const int half = threadIdx.x & 1, rowt = threadIdx.x >> 1;
  const int site = rowt / GT;
  const int z = b / (bx * by);
  const int y = ((b / bx) % by) * kBY + site / kBX;
  const int x = (b % bx) * kBX + site % kBX;
  if (y >= s.H || x >= s.W) return;   // both lanes of the pair leave together
  const int g = blockIdx.y;
  const int h = g * s.G + blockIdx.z * GT + rowt % GT;
  const int i = __ldg(g2p + (z * s.H + y) * s.W + x);
  if (i < 0) return;
  const unsigned pair = 3u << ((threadIdx.x & 31) & ~1);
  const size_t orow = (size_t)i * s.Hq + h;
  const int d0 = half * kHalf;

  float q[kHalf], dO[kHalf], dq[kHalf];
  load_f32(qr + orow * kDh + d0, q, kHalf);
  load_f32(dout + orow * kDh + d0, dO, kHalf);
  const float w0 = gate_weights(gate, orow).x;
#pragma unroll
  for (int e = 0; e < kHalf; ++e) {
    q[e] *= s.scale_log2;
    dO[e] *= w0;
    dq[e] = 0.f;
  }
  const float lse2 = stats[4 * orow], delta = stats[4 * orow + 2];
  const int z0 = max(0, z - s.rz), z1 = min(s.Z - 1, z + s.rz);
  const int y0 = max(0, y - s.ry), y1 = min(s.H - 1, y + s.ry);
  const int x0 = max(0, x - s.rx), x1 = min(s.W - 1, x + s.rx);
  for (int zz = z0; zz <= z1; ++zz)
    for (int yy = y0; yy <= y1; ++yy)
      for (int xx = x0; xx <= x1; ++xx) {
        const int jj = __ldg(g2p + (zz * s.H + yy) * s.W + xx);
        if (jj < 0) continue;
        const size_t kv = ((size_t)jj * s.Hkv + g) * kDh + d0;
        float kf[kHalf], vf[kHalf];
        load_f32(kr + kv, kf, kHalf);
        load_f32(vl + kv, vf, kHalf);
        float sd = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < kHalf; ++e) {
          sd = fmaf(q[e], kf[e], sd);
          dp = fmaf(dO[e], vf[e], dp);
        }
        sd += __shfl_xor_sync(pair, sd, 1);
        dp += __shfl_xor_sync(pair, dp, 1);
        const float ds = exp2f(sd - lse2) * (dp - delta);
#pragma unroll
        for (int e = 0; e < kHalf; ++e) dq[e] = fmaf(ds, kf[e], dq[e]);
      }
  const float4* c4 = reinterpret_cast<const float4*>(dqr + orow * kDh + d0);
#pragma unroll
  for (int c = 0; c < kHalf / 4; ++c) {
    const float4 a = __ldg(c4 + c);
    dq[4 * c] = fmaf(s.scale, dq[4 * c], a.x);
    dq[4 * c + 1] = fmaf(s.scale, dq[4 * c + 1], a.y);
    dq[4 * c + 2] = fmaf(s.scale, dq[4 * c + 2], a.z);
    dq[4 * c + 3] = fmaf(s.scale, dq[4 * c + 3], a.w);
  }
  rope_planes(dq, s, tab, half * (kHalf / 2), kHalf / 2, z, y, x, true);
  store_f32(dq_out + orow * kDh + d0, dq, kHalf);
}

// ---- local branch, key side -----------------------------------------------

template <typename T>
__global__ void __launch_bounds__(2 * kBSites) local_bwd_dkv_kernel(
    Shape s, const int32_t* __restrict__ g2p, const T* __restrict__ qr, const T* __restrict__ kr,
    const T* __restrict__ vl, const T* __restrict__ dout, const float* __restrict__ gate,
    const float* __restrict__ stats, T* __restrict__ dk_out, T* __restrict__ dv_out) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  const int bx = (s.W + kBX - 1) / kBX, by = (s.H + kBY - 1) / kBY;
  const int b = blockIdx.x;
  const int site = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int z = b / (bx * by);
  const int y = ((b / bx) % by) * kBY + site / kBX;
  const int x = (b % bx) * kBX + site % kBX;
  const int g = blockIdx.y;
  const int j = (y < s.H && x < s.W) ? __ldg(g2p + (z * s.H + y) * s.W + x) : -1;
  if (j < 0) return;   // both lanes of the pair leave together
  const unsigned pair = 3u << ((threadIdx.x & 31) & ~1);

  float k[kHalf], v[kHalf], dk[kHalf], dv[kHalf];
  load_f32(kr + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, k, kHalf);
  load_f32(vl + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, v, kHalf);
#pragma unroll
  for (int e = 0; e < kHalf; ++e) dk[e] = dv[e] = 0.f;
  const int z0 = max(0, z - s.rz), z1 = min(s.Z - 1, z + s.rz);
  const int y0 = max(0, y - s.ry), y1 = min(s.H - 1, y + s.ry);
  const int x0 = max(0, x - s.rx), x1 = min(s.W - 1, x + s.rx);
  for (int zz = z0; zz <= z1; ++zz)
    for (int yy = y0; yy <= y1; ++yy)
      for (int xx = x0; xx <= x1; ++xx) {
        const int i = __ldg(g2p + (zz * s.H + yy) * s.W + xx);
        if (i < 0) continue;
        for (int hh = 0; hh < s.G; ++hh) {
          const size_t orow = (size_t)i * s.Hq + g * s.G + hh;
          float qh[kHalf], oh[kHalf];
          load_f32(qr + orow * kDh + half * kHalf, qh, kHalf);
          load_f32(dout + orow * kDh + half * kHalf, oh, kHalf);
          const float w0 = gate_weights(gate, orow).x;
          float sh = 0.f, ph = 0.f;
#pragma unroll
          for (int e = 0; e < kHalf; ++e) {
            oh[e] *= w0;
            sh = fmaf(qh[e], k[e], sh);
            ph = fmaf(oh[e], v[e], ph);
          }
          sh += __shfl_xor_sync(pair, sh, 1);
          ph += __shfl_xor_sync(pair, ph, 1);
          const float p = exp2f(sh * s.scale_log2 - stats[4 * orow]);
          const float ds = p * (ph - stats[4 * orow + 2]);
#pragma unroll
          for (int e = 0; e < kHalf; ++e) {
            dk[e] = fmaf(ds, qh[e], dk[e]);
            dv[e] = fmaf(p, oh[e], dv[e]);
          }
        }
      }
#pragma unroll
  for (int e = 0; e < kHalf; ++e) dk[e] *= s.scale;
  rope_planes(dk, s, tab, half * (kHalf / 2), kHalf / 2, z, y, x, true);
  store_f32(dk_out + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, dk, kHalf);
  store_f32(dv_out + ((size_t)j * s.Hkv + g) * kDh + half * kHalf, dv, kHalf);
}

// ---- summaries ------------------------------------------------------------

constexpr int kSbThreads = 256, kMaxBlockVolume = 64;

// One warp per (block, kv head); lane p owns rotary plane p, i.e. dims 2p and
// 2p+1 of every row, so R(c) and R(c)^T act lane-locally and every load and
// store of a 64-dim row is one coalesced warp access.
template <typename T>
__device__ __forceinline__ float2 load_pair(const T* p);
template <>
__device__ __forceinline__ float2 load_pair<float>(const float* p) {
  return __ldg(reinterpret_cast<const float2*>(p));
}
template <>
__device__ __forceinline__ float2 load_pair<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p));
  return make_float2(bf16_lo(w), bf16_hi(w));
}
__device__ __forceinline__ void store_pair(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void store_pair(__nv_bfloat16* p, float2 v) {
  *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v.x, v.y);
}

// (x0, x1) of plane p at coordinate value cval: R (sg = +1) or R^T (sg = -1).
__device__ __forceinline__ float2 rot_pair(float2 f, const float2* tab, int off, int cval, float sg) {
  const float2 cs = tab[off + cval];
  const float sn = sg * cs.y;
  return make_float2(f.x * cs.x - f.y * sn, f.x * sn + f.y * cs.x);
}

template <typename T>
__global__ void __launch_bounds__(kSbThreads) summaries_bwd_kernel(
    Shape s, const int32_t* __restrict__ coords, const int32_t* __restrict__ members,
    const T* __restrict__ kc, const T* __restrict__ vc, const float* __restrict__ scores,
    const float* __restrict__ dks, const float* __restrict__ dvs, T* __restrict__ dkc, T* __restrict__ dvc,
    float* __restrict__ dsc) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long w = (long)blockIdx.x * (kSbThreads / 32) + (threadIdx.x >> 5);
  if (w >= (long)s.M * s.Hkv) return;
  const int j = (int)(w / s.Hkv), g = (int)(w % s.Hkv);
  // This lane's rotary plane: axis and first table entry (untouched planes: identity).
  const int ax = lane < s.npairs ? s.pair_axis[lane] : 3;
  const int toff = lane < s.npairs ? s.pair_off[lane] : 0;
  const size_t srow = ((size_t)j * s.Hkv + g) * kDh + 2 * lane;
  float2 dk = __ldg(reinterpret_cast<const float2*>(dks + srow));
  const float2 dv = __ldg(reinterpret_cast<const float2*>(dvs + srow));
  if (s.center) {
    // Summary-centre variant: k~ = R(cbar) sum_u a_u k_u, so the pooled key's
    // gradient is R(cbar)^T dk~ = R(-cbar) dk~ and the members are unrotated.
    float f[2] = {dk.x, dk.y};
    const int jx = j % s.nbx, jy = (j / s.nbx) % s.nby, jz = j / (s.nbx * s.nby);
    if (lane < s.npairs)
      rotate_at<1>(f, s, lane, -(s.origin[0] + jz * s.bz + 0.5 * (s.bz - 1)),
                   -(s.origin[1] + jy * s.by + 0.5 * (s.by - 1)), -(s.origin[2] + jx * s.bx + 0.5 * (s.bx - 1)));
    dk = make_float2(f[0], f[1]);
  }
  const int32_t* mem = members + (size_t)j * s.v;
  // Block weights: the scores of the block's members (lanes hold two members each).
  float smax = -INFINITY;
  for (int m = lane; m < s.v; m += 32) smax = fmaxf(smax, __ldg(scores + (size_t)__ldg(mem + m) * s.Hkv + g));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
  float den = 0.f;
  for (int m = lane; m < s.v; m += 32) den += expf(__ldg(scores + (size_t)__ldg(mem + m) * s.Hkv + g) - smax);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  const float inv = 1.f / den;
  // da_u for every member, then the mean sum_u a_u da_u.
  float a[kMaxBlockVolume], da[kMaxBlockVolume];
  float mean = 0.f;
  for (int m = 0; m < s.v; ++m) {
    const size_t u = (size_t)__ldg(mem + m);
    a[m] = expf(__ldg(scores + u * s.Hkv + g) - smax) * inv;
    const size_t row = (u * s.Hkv + g) * kDh + 2 * lane;
    float2 kr = load_pair(kc + row);
    if (!s.center && ax < 3) {
      const int cval = __ldg(coords + 3 * u + ax);
      kr = rot_pair(kr, tab, toff, cval, 1.f);
    }
    const float2 vv = load_pair(vc + row);
    float acc = dk.x * kr.x + dk.y * kr.y + dv.x * vv.x + dv.y * vv.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    da[m] = acc;
    mean = fmaf(a[m], acc, mean);
  }
  for (int m = 0; m < s.v; ++m) {
    const size_t u = (size_t)__ldg(mem + m);
    if (lane == 0) dsc[u * s.Hkv + g] = a[m] * (da[m] - mean);
    const size_t row = (u * s.Hkv + g) * kDh + 2 * lane;
    float2 k2 = make_float2(a[m] * dk.x, a[m] * dk.y);
    if (!s.center && ax < 3) {
      const int cval = __ldg(coords + 3 * u + ax);
      k2 = rot_pair(k2, tab, toff, cval, -1.f);
    }
    store_pair(dkc + row, k2);
    store_pair(dvc + row, make_float2(a[m] * dv.x, a[m] * dv.y));
  }
}

// ---- finalize of the tensor-core local backward ----------------------------

// dq = R(c)^T dqr, dk_loc = R(c)^T dk_acc, dv_loc = dv_acc (float accumulators
// to the operator's dtype); blockIdx.y picks the tensor, thread = 16 dims of a row.
template <typename T>
__global__ void __launch_bounds__(256) local_bwd_finalize_kernel(
    Shape s, const int32_t* __restrict__ coords, const float* __restrict__ dqr, const float* __restrict__ dka,
    const float* __restrict__ dva, T* __restrict__ dq, T* __restrict__ dk, T* __restrict__ dv) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  const int which = blockIdx.y;
  const int heads = which == 0 ? s.Hq : s.Hkv;
  const float* src = which == 0 ? dqr : (which == 1 ? dka : dva);
  T* dst = which == 0 ? dq : (which == 1 ? dk : dv);
  const long n = (long)s.N * heads * 4;
  for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (long)gridDim.x * blockDim.x) {
    const long row = t >> 2;
    const int qd = (int)(t & 3);
    float f[16];
    const float4* s4 = reinterpret_cast<const float4*>(src + row * kDh + qd * 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 v = __ldg(s4 + c);
      f[4 * c] = v.x; f[4 * c + 1] = v.y; f[4 * c + 2] = v.z; f[4 * c + 3] = v.w;
    }
    if (which < 2) {
      const long tok = row / heads;
      rope_planes(f, s, tab, qd * 8, 8, __ldg(coords + 3 * tok), __ldg(coords + 3 * tok + 1),
                  __ldg(coords + 3 * tok + 2), true);
    }
    store_f32(dst + row * kDh + qd * 16, f, 16);
  }
}

// ---- launchers --------------------------------------------------------------

template <typename T>
cudaError_t bwd_dq_t(const Shape& s, const void* qr, const void* ks, const void* vs, const void* dout,
                     const float* gate, const float* stats, float* dqr, cudaStream_t st) {
  const long rows = (long)s.N * s.G;
  dim3 grid((unsigned)((rows + kDqRows - 1) / kDqRows), s.Hkv);
  summary_bwd_dq_kernel<T><<<grid, kDqRows, 0, st>>>(s, (const T*)qr, (const T*)ks, (const T*)vs, (const T*)dout,
                                                     gate, stats, dqr);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_dkv_t(const Shape& s, const void* qr, const void* ks, const void* vs, const void* dout,
                      const float* gate, const float* stats, float* dks, float* dvs, cudaStream_t st) {
  const long rows = (long)s.N * s.G;
  const int tiles = (s.M + kDkvSums - 1) / kDkvSums;
  // About four CTAs per SM over the whole grid, each at least 256 rows.
  long splits = (4L * 148 + (long)tiles * s.Hkv - 1) / ((long)tiles * s.Hkv);
  splits = max(1L, min(splits, (rows + 255) / 256));
  long per = (rows + splits - 1) / splits;
  per = (per + kDkvStage - 1) / kDkvStage * kDkvStage;
  splits = (rows + per - 1) / per;
  dim3 grid((unsigned)tiles, s.Hkv, (unsigned)splits);
  summary_bwd_dkv_kernel<T><<<grid, kDkvThreads, 0, st>>>(s, (const T*)qr, (const T*)ks, (const T*)vs,
                                                          (const T*)dout, gate, stats, per, dks, dvs);
  return cudaGetLastError();
}

template <typename T, int GT>
cudaError_t local_dq_t(const Shape& s, const int32_t* g2p, const void* qr, const void* kr, const void* vl,
                       const void* dout, const float* gate, const float* stats, const float* dqr, void* dq,
                       cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = set_table_smem((const void*)local_bwd_dq_kernel<T, GT>, smem);
  if (e != cudaSuccess) return e;
  const int bricks = s.Z * ((s.H + kBY - 1) / kBY) * ((s.W + kBX - 1) / kBX);
  dim3 grid(bricks, s.Hkv, s.G / GT);
  local_bwd_dq_kernel<T, GT><<<grid, 2 * kBSites * GT, smem, st>>>(s, g2p, (const T*)qr, (const T*)kr, (const T*)vl,
                                                               (const T*)dout, gate, stats, dqr, (T*)dq);
  return cudaGetLastError();
}

template <typename T>
cudaError_t local_dq_g(const Shape& s, const int32_t* g2p, const void* qr, const void* kr, const void* vl,
                       const void* dout, const float* gate, const float* stats, const float* dqr, void* dq,
                       cudaStream_t st) {
  if (s.G == 1) return local_dq_t<T, 1>(s, g2p, qr, kr, vl, dout, gate, stats, dqr, dq, st);
  return local_dq_t<T, 2>(s, g2p, qr, kr, vl, dout, gate, stats, dqr, dq, st);   // G = 2, 4, 8
}

template <typename T>
cudaError_t local_dkv_t(const Shape& s, const int32_t* g2p, const void* qr, const void* kr, const void* vl,
                        const void* dout, const float* gate, const float* stats, void* dk, void* dv,
                        cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = set_table_smem((const void*)local_bwd_dkv_kernel<T>, smem);
  if (e != cudaSuccess) return e;
  const int bricks = s.Z * ((s.H + kBY - 1) / kBY) * ((s.W + kBX - 1) / kBX);
  dim3 grid(bricks, s.Hkv);
  local_bwd_dkv_kernel<T><<<grid, 2 * kBSites, smem, st>>>(s, g2p, (const T*)qr, (const T*)kr, (const T*)vl,
                                                           (const T*)dout, gate, stats, (T*)dk, (T*)dv);
  return cudaGetLastError();
}

template <typename T>
cudaError_t summaries_bwd_t(const Shape& s, const int32_t* coords, const int32_t* members, const void* kc,
                            const void* vc, const float* scores, const float* dks, const float* dvs, void* dkc,
                            void* dvc, float* dsc, cudaStream_t st) {
  if (s.v > kMaxBlockVolume) return cudaErrorInvalidValue;
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = set_table_smem((const void*)summaries_bwd_kernel<T>, smem);
  if (e != cudaSuccess) return e;
  const long warps = (long)s.M * s.Hkv;
  const long per_cta = kSbThreads / 32;
  summaries_bwd_kernel<T><<<(unsigned)((warps + per_cta - 1) / per_cta), kSbThreads, smem, st>>>(
      s, coords, members, (const T*)kc, (const T*)vc, scores, dks, dvs, (T*)dkc, (T*)dvc, dsc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_summary_bwd_dq(const Shape& s, int dtype, const void* qr, const void* ks, const void* vs,
                                  const void* dout, const float* gate, const float* stats, float* dqr,
                                  cudaStream_t st) {
  if (dtype == PACK3D_BF16) return bwd_dq_t<__nv_bfloat16>(s, qr, ks, vs, dout, gate, stats, dqr, st);
  return bwd_dq_t<float>(s, qr, ks, vs, dout, gate, stats, dqr, st);
}

cudaError_t launch_summary_bwd_dkv(const Shape& s, int dtype, const void* qr, const void* ks, const void* vs,
                                   const void* dout, const float* gate, const float* stats, float* dks,
                                   float* dvs, cudaStream_t st) {
  if (dtype == PACK3D_BF16) return bwd_dkv_t<__nv_bfloat16>(s, qr, ks, vs, dout, gate, stats, dks, dvs, st);
  return bwd_dkv_t<float>(s, qr, ks, vs, dout, gate, stats, dks, dvs, st);
}

cudaError_t launch_local_bwd_dq(const Shape& s, int dtype, const int32_t* g2p, const void* qr, const void* kr,
                                const void* vl, const void* dout, const float* gate, const float* stats,
                                const float* dqr, void* dq, cudaStream_t st) {
  if (dtype == PACK3D_BF16) return local_dq_g<__nv_bfloat16>(s, g2p, qr, kr, vl, dout, gate, stats, dqr, dq, st);
  return local_dq_g<float>(s, g2p, qr, kr, vl, dout, gate, stats, dqr, dq, st);
}

cudaError_t launch_local_bwd_dkv(const Shape& s, int dtype, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, const void* dout, const float* gate, const float* stats,
                                 void* dk, void* dv, cudaStream_t st) {
  if (dtype == PACK3D_BF16) return local_dkv_t<__nv_bfloat16>(s, g2p, qr, kr, vl, dout, gate, stats, dk, dv, st);
  return local_dkv_t<float>(s, g2p, qr, kr, vl, dout, gate, stats, dk, dv, st);
}

cudaError_t launch_local_bwd_finalize(const Shape& s, int dtype, const int32_t* coords, const float* dqr,
                                      const float* dka, const float* dva, void* dq, void* dk, void* dv,
                                      cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  dim3 grid(148 * 8, 3);
  if (dtype == PACK3D_BF16) {
    cudaError_t e = set_table_smem((const void*)local_bwd_finalize_kernel<__nv_bfloat16>, smem);
    if (e != cudaSuccess) return e;
    local_bwd_finalize_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(
        s, coords, dqr, dka, dva, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv);
  } else {
    cudaError_t e = set_table_smem((const void*)local_bwd_finalize_kernel<float>, smem);
    if (e != cudaSuccess) return e;
    local_bwd_finalize_kernel<float><<<grid, 256, smem, st>>>(s, coords, dqr, dka, dva, (float*)dq, (float*)dk,
                                                              (float*)dv);
  }
  return cudaGetLastError();
}

cudaError_t launch_summaries_bwd(const Shape& s, int dtype, const int32_t* coords, const int32_t* members,
                                 const void* kc, const void* vc, const float* scores, const float* dks,
                                 const float* dvs, void* dkc, void* dvc, float* dsc, cudaStream_t st) {
  if (dtype == PACK3D_BF16)
    return summaries_bwd_t<__nv_bfloat16>(s, coords, members, kc, vc, scores, dks, dvs, dkc, dvc, dsc, st);
  return summaries_bwd_t<float>(s, coords, members, kc, vc, scores, dks, dvs, dkc, dvc, dsc, st);
}

}  // namespace pack3d
