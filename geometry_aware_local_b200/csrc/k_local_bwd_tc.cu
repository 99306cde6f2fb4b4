// Backward of the exact local attention branch on sm_100a tensor cores
// ("Geometry Matters in Packed 3D Attention", Key design 3: softmax attention
// of each token over its clipped lattice box), for the training block.
//
// The CTA covers the same unit as the forward kernel: one 2 x 4 x 4 brick of
// query sites of one kv head with its G = 4 q heads stacked, 128 rows (row =
// site * 4 + head), and the brick's halo keys one lattice z-plane at a time
// (a plane of (4 + 2ry) x (4 + 2rx) <= 100 sites padded to NP <= 112 rows,
// gathered through the index map with cp.async; outside keys zero-filled).
// With lse2 the row's saved log-sum-exp (base 2), gamma0 its local gate
// weight and D = <gamma0 dout, o_loc>, per plane:
//   S  = Q K^T,  dP = dout V^T                      (M=128, N=NP, K=64)
//   P  = 2^(c S - lse2) on the row's box mask, else 0; dS = P (gamma0 dP - D)
//   dQ += dS K                                      (M=128, N=64, K=NP; A = dS
//                                                     from tensor memory)
//   dK_plane = dS^T Q,  dV_plane = (gamma0 P)^T dout (M=128 keys, N=64, K=128
//                                                     rows; A MN-major from
//                                                     shared memory)
// One pass over the columns suffices: the log-sum-exp is known, so there is
// no running maximum.  Each plane's dK / dV rows are added to float
// accumulators (a key lies in the halo of several bricks) with vector
// atomics; dQ (every row owned by one CTA) is added to the float query
// gradient the compressed branch wrote.  A separate streaming kernel applies
// R(c)^T and converts.  Tensor memory: S 0-127, dP 128-255, dS 256-319
// (packed bf16), dQ 320-383, dK_plane 384-447, dV_plane 448-511; one CTA per
// SM.  Supported: bf16, G = 4, rz = 1, ry <= 3, rx <= 3, as the forward.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace pack3d {
namespace {

constexpr int kRows = 128;
// Warpgroups: each covers the CTA's 128 rows (a warp serves the tensor-memory
// lanes of its index mod 4); they split the softmax's column units, the
// per-plane dK / dV flush and the dQ epilogue.  Warpgroup 0 also does the
// gathers.  Measured on B200, forward+backward at 65k / 262k: one warpgroup
// 4.436 / 52.30 ms, two 4.399 / 52.58, four 4.416 / 51.90 (no clear gain).
#ifndef PACK3D_LBWD_WG
#define PACK3D_LBWD_WG 1
#endif
constexpr int kWG = PACK3D_LBWD_WG;
constexpr int kThreads = 128 * kWG;
constexpr int kMaxKeys = 112;                     // padded keys per plane
constexpr int kMaxPlanes = 4;                     // 2 brick layers + r_z = 1 on each side
constexpr int kRowTileBytes = kRows * kDh * 2;    // 16 KiB
constexpr int kPlaneTileBytes = kMaxKeys * kDh * 2;   // 14 KiB, a multiple of 1 KiB
constexpr int kQOff = 0, kDOOff = kRowTileBytes;
constexpr int kBufOff = 2 * kRowTileBytes;        // plane buffers: K at +0, V at +kPlaneTileBytes
constexpr int kBufs = 2;
constexpr int kBufBytes = 2 * kPlaneTileBytes;
constexpr int kDSOff = kBufOff + kBufs * kBufBytes;   // dS^T: keys 0-63 and 64-127 halves, 16 KiB each
constexpr int kPWOff = kDSOff + 2 * kRowTileBytes;    // (gamma0 P)^T, same layout
constexpr int kBarOff = kPWOff + 2 * kRowTileBytes;
constexpr int kSmemBytes = kBarOff + 64 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr int kColS = 0, kColDP = 128, kColDS = 256, kColDQ = 320, kColDK = 384, kColDV = 448;
constexpr uint32_t kIdescDQ = ptx::idesc_bf16_f32(kRows, kDh, true);             // B = K plane, MN-major
constexpr uint32_t kIdescKV = ptx::idesc_bf16_f32_ab(kRows, kDh, true, true);    // A, B MN-major

struct LocalBwdArgs {
  int Z, H, W, Hq, Hkv;
  int ry, rx, PH, PW, NP;
  float scale_log2, scale;
  const int32_t* g2p;
  const __nv_bfloat16* q;      // rotated queries
  const __nv_bfloat16* k;      // rotated local keys
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  const float* gate;
  const float* stats;
  float* dqr;                  // [N, Hq, 64]: += scale * dQ
  float* dk_acc;               // [N, Hkv, 64]: += scale * dK (rotated frame)
  float* dv_acc;               // [N, Hkv, 64]
  int32_t* err;
  unsigned long long wait_ns;  // limit of every pipeline wait
  int stall;                   // diagnostic: the S / dP MMAs of the last plane are never issued
};

// One 128-byte row into a 128-byte-swizzled tile at row r (zeros if src == nullptr).
__device__ __forceinline__ void gather_row(uint32_t tile, int r, const __nv_bfloat16* src,
                                           const __nv_bfloat16* any_valid) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t dst = tile + r * 128 + ((c ^ (r & 7)) << 4);
    if (src)
      ptx::cp_async16(dst, src + c * 8, 16);
    else
      ptx::cp_async16(dst, any_valid, 0);
  }
}

// Packed index of row r of the padded plane zp, or -1.
__device__ __forceinline__ int plane_row_index(const LocalBwdArgs& a, int r, int zp, int y0, int x0) {
  if (r >= a.PH * a.PW) return -1;
  const int y = y0 - a.ry + r / a.PW, x = x0 - a.rx + r % a.PW;
  if (y < 0 || y >= a.H || x < 0 || x >= a.W) return -1;
  return __ldg(a.g2p + ((size_t)zp * a.H + y) * a.W + x);
}

__device__ __forceinline__ void gather_plane(const LocalBwdArgs& a, int r, uint32_t kt, int g, int j) {
  if (r >= a.NP) return;
  gather_row(kt, r, j >= 0 ? a.k + ((size_t)j * a.Hkv + g) * kDh : nullptr, a.k);
  gather_row(kt + kPlaneTileBytes, r, j >= 0 ? a.v + ((size_t)j * a.Hkv + g) * kDh : nullptr, a.v);
}

__global__ void __launch_bounds__(kThreads, 1) local_bwd_tc_kernel(const LocalBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t s_full = sbase + kBarOff;        // S and dP of the current plane are in tensor memory
  const uint32_t mma_done = sbase + kBarOff + 8;  // dQ / dK / dV MMAs of the last issued plane completed
  const uint32_t drain = sbase + kBarOff + 16;    // abort path: every MMA issued so far has completed
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + 24);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 24 + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kRows - 1), wg = tid >> 7;   // tensor-memory lane and warpgroup
  const int g = blockIdx.y;

  const int nbx = (a.W + 3) / 4, nby = (a.H + 3) / 4;
  const int b = blockIdx.x;
  const int x0 = (b % nbx) * 4, y0 = ((b / nbx) % nby) * 4, z0 = (b / (nbx * nby)) * 2;
  const int site = row >> 2, hh = row & 3;
  const int lz = site >> 4, ly = (site >> 2) & 3, lx = site & 3;
  const int qz = z0 + lz, qy = y0 + ly, qx = x0 + lx;
  const bool qvalid = qz < a.Z && qy < a.H && qx < a.W;
  const int h = g * 4 + hh;

  if (tid == 0) {
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(mma_done, 1);
    ptx::mbar_init(drain, 1);
    ctl->abort = 0;
    ctl->limit_ns = a.wait_ns;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }

  const int zlo = max(0, z0 - 1), zhi = min(a.Z - 1, z0 + 2);
  const int nplanes = zhi - zlo + 1;
  const int qi = qvalid ? __ldg(a.g2p + ((size_t)qz * a.H + qy) * a.W + qx) : -1;
  int gi[kMaxPlanes];
#pragma unroll
  for (int p = 0; p < kMaxPlanes; ++p) gi[p] = p < nplanes ? plane_row_index(a, row, zlo + p, y0, x0) : -1;

  auto kt_of = [&](int p) { return sbase + kBufOff + (p % kBufs) * kBufBytes; };
  const size_t orow = qi >= 0 ? (size_t)qi * a.Hq + h : 0;
  if (wg == 0) {
    gather_row(sbase + kQOff, row, qi >= 0 ? a.q + orow * kDh : nullptr, a.q);
    gather_row(sbase + kDOOff, row, qi >= 0 ? a.dout + orow * kDh : nullptr, a.dout);
    gather_plane(a, row, kt_of(0), g, gi[0]);
    if (nplanes > 1) gather_plane(a, row, kt_of(1), g, gi[1]);
  }
  ptx::cp_async_commit();

  // Row statistics; rows of sites outside the volume keep P = 0 through an empty mask.
  const float lse2 = qi >= 0 ? a.stats[4 * orow] : 0.f;
  const float delta = qi >= 0 ? a.stats[4 * orow + 2] : 0.f;
  const float w0 = qi >= 0 ? gate_weights(a.gate, orow).x : 0.f;

  // Lattice-box mask of this row over the padded plane (bit k = key k allowed).
  uint32_t mask[4];
  {
    uint32_t xvalid = 0;
    for (int kx = 0; kx < a.PW; ++kx) {
      const int x = x0 - a.rx + kx;
      if (x >= 0 && x < a.W) xvalid |= 1u << kx;
    }
    const uint32_t xbits = (((1u << (2 * a.rx + 1)) - 1u) << lx) & xvalid;
    unsigned __int128 m = 0;
    if (qi >= 0)
      for (int dy = 0; dy <= 2 * a.ry; ++dy) {
        const int ky = ly + dy, y = y0 - a.ry + ky;
        if (y >= 0 && y < a.H) m |= (unsigned __int128)xbits << (ky * a.PW);
      }
    mask[0] = (uint32_t)m;
    mask[1] = (uint32_t)(m >> 32);
    mask[2] = (uint32_t)(m >> 64);
    mask[3] = (uint32_t)(m >> 96);
  }

  ptx::cp_async_wait_all();
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const uint32_t idescS = ptx::idesc_bf16_f32(kRows, a.NP, false);
  const float2 c2 = make_float2(a.scale_log2, a.scale_log2), nl2 = make_float2(-lse2, -lse2);
  const float2 w2 = make_float2(w0, w0), nd2 = make_float2(-delta, -delta);

  auto issue_sdp = [&](int p) {
    const uint32_t kt = kt_of(p), vt = kt + kPlaneTileBytes;
#pragma unroll
    for (int kk = 0; kk < kDh / 16; ++kk)
      ptx::mma_ss(tmem + kColS, ptx::smem_desc_sw128(sbase + kQOff + kk * 32, 16, 1024),
                  ptx::smem_desc_sw128(kt + kk * 32, 16, 1024), idescS, kk > 0);
#pragma unroll
    for (int kk = 0; kk < kDh / 16; ++kk)
      ptx::mma_ss(tmem + kColDP, ptx::smem_desc_sw128(sbase + kDOOff + kk * 32, 16, 1024),
                  ptx::smem_desc_sw128(vt + kk * 32, 16, 1024), idescS, kk > 0);
    ptx::tc_commit(s_full);
  };
  auto issue_grads = [&](int p) {
    const uint32_t kt = kt_of(p);
    for (int kk = 0; kk < a.NP / 16; ++kk)
      ptx::mma_ts(tmem + kColDQ, tmem + kColDS + kk * 8, ptx::smem_desc_sw128(kt + kk * 2048, 8192, 1024), kIdescDQ,
                  (p > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < kRows / 16; ++kk)
      ptx::mma_ss(tmem + kColDK, ptx::smem_desc_sw128(sbase + kDSOff + kk * 2048, 2 * 8192, 1024),
                  ptx::smem_desc_sw128(sbase + kQOff + kk * 2048, 8192, 1024), kIdescKV, kk > 0);
#pragma unroll
    for (int kk = 0; kk < kRows / 16; ++kk)
      ptx::mma_ss(tmem + kColDV, ptx::smem_desc_sw128(sbase + kPWOff + kk * 2048, 2 * 8192, 1024),
                  ptx::smem_desc_sw128(sbase + kDOOff + kk * 2048, 8192, 1024), kIdescKV, kk > 0);
    ptx::tc_commit(mma_done);
  };
  // Adds plane p's dK / dV rows (tensor-memory lane = key row of the plane) to
  // the accumulators; the warpgroups share the 128 columns (dK 64, then dV 64).
  auto flush_plane = [&](int p) {
    const int j = gi[p];
    const bool mine = row < a.NP && j >= 0;
    constexpr int kCols = 2 * kDh / kWG;          // 128, 64 or 32
    constexpr int kLoad = kCols < 64 ? kCols : 64;
#pragma unroll
    for (int part = 0; part < kCols / kLoad; ++part) {
      const int col0 = wg * kCols + part * kLoad;   // in [0, 128): dK below 64, dV from 64
      uint32_t r[kLoad];
      if constexpr (kLoad == 64)
        ptx::tmem_ld64_sync(trow + kColDK + col0, r);
      else
        ptx::tmem_ld32_sync(trow + kColDK + col0, r);
      if (mine) {
        const bool is_k = col0 < kDh;
        const float f = is_k ? a.scale : 1.f;
        float4* dst = reinterpret_cast<float4*>((is_k ? a.dk_acc : a.dv_acc) + ((size_t)j * a.Hkv + g) * kDh +
                                                (col0 % kDh));
#pragma unroll
        for (int q = 0; q < kLoad / 4; ++q)
          atomicAdd(dst + q, make_float4(f * __uint_as_float(r[4 * q]), f * __uint_as_float(r[4 * q + 1]),
                                         f * __uint_as_float(r[4 * q + 2]), f * __uint_as_float(r[4 * q + 3])));
      }
    }
  };

  // (PACK3D_FLAG_DIAG_STALL withholds the S / dP MMAs of the last plane.)
  if (tid == 0 && !(a.stall && nplanes == 1)) issue_sdp(0);
  bool ok = true;
  for (int p = 0; p < nplanes; ++p) {
    const int zp = zlo + p;
    const bool uses = zp >= z0 + lz - 1 && zp <= z0 + lz + 1;   // warp-uniform (layer = warp / 2)
    bool w_ok = __all_sync(0xffffffffu, wait(s_full, p & 1));
    if (w_ok && p > 0) w_ok = __all_sync(0xffffffffu, wait(mma_done, (p - 1) & 1));
    if (!(ok = __syncthreads_and(w_ok))) break;
    ptx::tc_fence_after();
    if (p > 0) {
      flush_plane(p - 1);
      // Plane p-1's buffer is free again (its MMAs completed): gather plane p+1 into it.
      if (p + 1 < nplanes && wg == 0) gather_plane(a, row, kt_of(p + 1), g, gi[p + 1]);
      ptx::cp_async_commit();
    }
    // One pass over the plane's columns, 16 at a time, units split over the warpgroups.
    for (int u = wg; u < a.NP / 16; u += kWG) {
      uint32_t sv[16], dv[16];
      ptx::tmem_ld16x2_sync(trow + kColS + 16 * u, trow + kColDP + 16 * u, sv, dv);
      const uint32_t bits = uses ? (mask[u >> 1] >> ((u & 1) * 16)) & 0xffffu : 0u;
      uint32_t pd[8], pw[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
        const float2 t = __ffma2_rn(make_float2(__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])), w2, nd2);
        float2 pr = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
        if (!((bits >> (2 * k)) & 1u)) pr.x = 0.f;
        if (!((bits >> (2 * k + 1)) & 1u)) pr.y = 0.f;
        const float2 ds = __fmul2_rn(pr, t);
        const float2 pwv = __fmul2_rn(pr, w2);
        pd[k] = pack_bf16x2(ds.x, ds.y);
        pw[k] = pack_bf16x2(pwv.x, pwv.y);
      }
      ptx::tmem_st8(trow + kColDS + 8 * u, pd);
      // keys 16u .. 16u+15: chunks ((16u) % 64) / 8 and +1 of half (16u) / 64, this row
      const uint32_t half = (uint32_t)(16 * u) >> 6, e0 = (uint32_t)(16 * u) & 63u;
      const uint32_t o0 = half * kRowTileBytes + ptx::sw128_offset((uint32_t)row, e0);
      const uint32_t o1 = half * kRowTileBytes + ptx::sw128_offset((uint32_t)row, e0 + 8);
      ptx::st_shared_v4(sbase + kDSOff + o0, pd[0], pd[1], pd[2], pd[3]);
      ptx::st_shared_v4(sbase + kDSOff + o1, pd[4], pd[5], pd[6], pd[7]);
      ptx::st_shared_v4(sbase + kPWOff + o0, pw[0], pw[1], pw[2], pw[3]);
      ptx::st_shared_v4(sbase + kPWOff + o1, pw[4], pw[5], pw[6], pw[7]);
    }
    ptx::tmem_wait_st();
    ptx::cp_async_wait_all();
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      issue_grads(p);
      if (p + 1 < nplanes && !(a.stall && p + 2 == nplanes)) issue_sdp(p + 1);
    }
  }

  if (ok) ok = __syncthreads_and(__all_sync(0xffffffffu, wait(mma_done, (nplanes - 1) & 1)));
  if (ok) {
    ptx::tc_fence_after();
    flush_plane(nplanes - 1);
    constexpr int kQCols = kDh / kWG;             // 64, 32 or 16 columns of dQ per warpgroup
    uint32_t r[kQCols];
    if constexpr (kQCols == 64)
      ptx::tmem_ld64_sync(trow + kColDQ, r);
    else if constexpr (kQCols == 32)
      ptx::tmem_ld32_sync(trow + kColDQ + wg * 32, r);
    else
      ptx::tmem_ld16_sync(trow + kColDQ + wg * 16, r);
    if (qi >= 0) {
      float4* dst = reinterpret_cast<float4*>(a.dqr + orow * kDh + wg * kQCols);
#pragma unroll
      for (int q = 0; q < kQCols / 4; ++q) {
        float4 v = dst[q];
        v.x = fmaf(a.scale, __uint_as_float(r[4 * q]), v.x);
        v.y = fmaf(a.scale, __uint_as_float(r[4 * q + 1]), v.y);
        v.z = fmaf(a.scale, __uint_as_float(r[4 * q + 2]), v.z);
        v.w = fmaf(a.scale, __uint_as_float(r[4 * q + 3]), v.w);
        dst[q] = v;
      }
    }
  }
  ptx::cp_async_wait_all();
  ptx::tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    // The flag is final here: the MMAs thread 0 issued complete before
    // tensor memory is released.
    if (tid == 0) {
      ptx::tc_commit(drain);
      ptx::mbar_wait_drain(drain, 0, ctl->limit_ns);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && ctl->abort) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_local_bwd_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr, const void* vl,
                                const void* dout, const float* gate, const float* stats, float* dqr, float* dk_acc,
                                float* dv_acc, int32_t* err, cudaStream_t st) {
  LocalBwdArgs a;
  a.Z = s.Z; a.H = s.H; a.W = s.W; a.Hq = s.Hq; a.Hkv = s.Hkv;
  a.ry = s.ry; a.rx = s.rx;
  a.PH = 4 + 2 * s.ry; a.PW = 4 + 2 * s.rx;
  a.NP = (a.PH * a.PW + 15) / 16 * 16;
  a.scale_log2 = s.scale_log2;
  a.scale = s.scale;
  a.g2p = g2p;
  a.q = (const __nv_bfloat16*)qr;
  a.k = (const __nv_bfloat16*)kr;
  a.v = (const __nv_bfloat16*)vl;
  a.dout = (const __nv_bfloat16*)dout;
  a.gate = gate;
  a.stats = stats;
  a.dqr = dqr;
  a.dk_acc = dk_acc;
  a.dv_acc = dv_acc;
  a.err = err;
  a.wait_ns = s.wait_ns;
  a.stall = s.stall;
  cudaError_t e = cudaFuncSetAttribute(local_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(((s.Z + 1) / 2) * ((s.H + 3) / 4) * ((s.W + 3) / 4)), s.Hkv);
  local_bwd_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace pack3d
