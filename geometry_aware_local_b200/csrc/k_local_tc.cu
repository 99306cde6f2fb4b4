// Exact local attention on sm_100a tensor cores ("Geometry Matters in Packed 3D
// Attention", Key design 3: softmax attention of each token over the tokens of
// its clipped lattice box, found through the grid-to-packed map, with no
// gathered neighbour tensor in global memory).
//
// One CTA = one 2 x 4 x 4 brick of query sites of one kv head; with the G = 4
// query heads of a kv head stacked, that is 128 rows = one tcgen05 M tile
// (row = site * 4 + head, sites z-major, so rows 0-63 are the brick's first
// z layer and rows 64-127 its second).  The keys of the brick's halo are
// processed one lattice z-plane at a time: a plane of (4 + 2ry) x (4 + 2rx) <=
// 10 x 10 sites, padded to NP <= 112 rows, is gathered through the index map
// with cp.async (keys outside the volume are zero-filled) into a 128-byte-
// swizzled K tile and V tile, double-buffered.  Per plane:
//   S = Q K^T  (M=128, N=NP, K=64; A, B from shared memory)
//   softmax on the rows whose z window contains the plane (the other layer's
//   warps write P = 0): the lattice-box mask is a per-row bit mask, the
//   running maximum moves lazily (only by more than 2^8) and O is rescaled in
//   tensor memory when it does;
//   O += P V   (M=128, N=64, K=NP; A = P from tensor memory, B = V from
//   shared memory, MN-major).
// Two CTAs share an SM (256 tensor-memory columns each: S 0-111, P 128-183,
// O 192-255), so one CTA's softmax overlaps the other's gathers and MMAs.
// Supported: bf16, G = 4, rz = 1, ry <= 3, rx <= 3 (the SIMT kernel covers the
// rest).  Every mbarrier wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace pack3d {
namespace {

constexpr int kRows = 128;
constexpr int kThreads = 128;
constexpr int kMaxKeys = 112;                     // padded keys per plane
constexpr int kTileBytes = kMaxKeys * kDh * 2;    // 14 KiB, a multiple of 1 KiB
constexpr int kQOff = 0;                          // 16 KiB query tile
constexpr int kKV0 = kRows * kDh * 2;             // plane buffers: K at +0, V at +kTileBytes
constexpr int kBufBytes = 2 * kTileBytes;
constexpr int kBarOff = kKV0 + 2 * kBufBytes;
// Requesting more than a third of the SM's shared memory keeps at most two
// CTAs per SM, matching the 2 x 256 tensor-memory columns.
constexpr int kSmemBytes = 80 * 1024;
static_assert(kBarOff + 64 + 1024 <= kSmemBytes, "shared memory plan");
constexpr float kRescaleThreshold = 8.0f;

struct LocalArgs {
  int Z, H, W, Hq, Hkv;
  int ry, rx, PH, PW, NP;  // plane height/width and padded key count
  float scale_log2;
  const int32_t* g2p;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  float* oloc;
  int32_t* err;
};

// Copies one 128-byte row into a 128-byte-swizzled tile at row r (zeros if src == nullptr).
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

__device__ __forceinline__ void gather_plane(const LocalArgs& a, uint32_t kt, uint32_t vt, int g, int zp, int y0,
                                             int x0) {
  // 128 threads x NP rows x 2 tensors; each thread takes rows tid, tid+128, ...
  // (NP <= 112 < 128: one row per thread, threads >= NP write nothing).
  const int r = threadIdx.x;
  if (r >= a.NP) return;
  const __nv_bfloat16* ks = nullptr;
  const __nv_bfloat16* vs = nullptr;
  if (r < a.PH * a.PW) {
    const int y = y0 - a.ry + r / a.PW, x = x0 - a.rx + r % a.PW;
    if (y >= 0 && y < a.H && x >= 0 && x < a.W) {
      const int j = __ldg(a.g2p + ((size_t)zp * a.H + y) * a.W + x);
      if (j >= 0) {
        ks = a.k + ((size_t)j * a.Hkv + g) * kDh;
        vs = a.v + ((size_t)j * a.Hkv + g) * kDh;
      }
    }
  }
  gather_row(kt, r, ks, a.k);
  gather_row(vt, r, vs, a.v);
}

__global__ void __launch_bounds__(kThreads, 2) local_attn_tc_kernel(const LocalArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar = sbase + kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + 12);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int g = blockIdx.y;

  // Brick origin.
  const int nbx = (a.W + 3) / 4, nby = (a.H + 3) / 4;
  const int b = blockIdx.x;
  const int x0 = (b % nbx) * 4, y0 = ((b / nbx) % nby) * 4, z0 = (b / (nbx * nby)) * 2;

  // This thread's row: site (lz, ly, lx) of the brick, head hh.
  const int site = tid >> 2, hh = tid & 3;
  const int lz = site >> 4, ly = (site >> 2) & 3, lx = site & 3;
  const int qz = z0 + lz, qy = y0 + ly, qx = x0 + lx;
  const bool qvalid = qz < a.Z && qy < a.H && qx < a.W;
  const int h = g * 4 + hh;

  if (tid == 0) {
    ptx::mbar_init(bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 256);
    ptx::tmem_relinquish();
  }

  // Query row gather (own row).
  int qi = -1;
  if (qvalid) qi = __ldg(a.g2p + ((size_t)qz * a.H + qy) * a.W + qx);
  gather_row(sbase + kQOff, tid, qi >= 0 ? a.q + ((size_t)qi * a.Hq + h) * kDh : nullptr, a.q);

  // Planes z0-1 .. z0+2 inside the volume.  cp.async groups: {Q, plane 0},
  // {plane 1}, then one group per loop iteration (plane p + 2, possibly empty),
  // so waiting until at most one group is pending always lands plane p.
  const int zlo = max(0, z0 - 1), zhi = min(a.Z - 1, z0 + 2);
  const int nplanes = zhi - zlo + 1;
  gather_plane(a, sbase + kKV0, sbase + kKV0 + kTileBytes, g, zlo, y0, x0);
  ptx::cp_async_commit();
  if (nplanes > 1) gather_plane(a, sbase + kKV0 + kBufBytes, sbase + kKV0 + kBufBytes + kTileBytes, g, zlo + 1, y0, x0);
  ptx::cp_async_commit();

  // Lattice-box mask of this row over the padded plane (bit k = key k
  // allowed): the row's x run [lx, lx + 2rx] limited to in-volume columns,
  // repeated on the plane rows [ly, ly + 2ry] that lie inside the volume.
  uint32_t mask[4];
  {
    uint32_t xvalid = 0;
    for (int kx = 0; kx < a.PW; ++kx) {
      const int x = x0 - a.rx + kx;
      if (x >= 0 && x < a.W) xvalid |= 1u << kx;
    }
    const uint32_t xbits = (((1u << (2 * a.rx + 1)) - 1u) << lx) & xvalid;
    unsigned __int128 m = 0;
    for (int dy = 0; dy <= 2 * a.ry; ++dy) {
      const int ky = ly + dy, y = y0 - a.ry + ky;
      if (y >= 0 && y < a.H) m |= (unsigned __int128)xbits << (ky * a.PW);
    }
    mask[0] = (uint32_t)m;
    mask[1] = (uint32_t)(m >> 32);
    mask[2] = (uint32_t)(m >> 64);
    mask[3] = (uint32_t)(m >> 96);
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const uint32_t tS = trow, tP = trow + 128, tO = trow + 192;
  const uint32_t idescS = ptx::idesc_bf16_f32(kRows, a.NP, false);
  const uint32_t idescPV = ptx::idesc_bf16_f32(kRows, kDh, true);
  const float c = a.scale_log2;

  float m_used = -INFINITY, l = 0.f;
  uint32_t phase = 0;
  bool ok = true;
  for (int p = 0; p < nplanes && ok; ++p) {
    const int zp = zlo + p;
    const uint32_t kt = sbase + kKV0 + (p & 1) * kBufBytes, vt = kt + kTileBytes;
    ptx::cp_async_wait_one();
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kDh / 16; ++kk)
        ptx::mma_ss(tS, ptx::smem_desc_sw128(sbase + kQOff + kk * 32, 16, 1024),
                    ptx::smem_desc_sw128(kt + kk * 32, 16, 1024), idescS, kk > 0);
      ptx::tc_commit(bar);
    }
    __syncwarp();
    if (!(ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar, phase, abort_flag)))) break;
    phase ^= 1;
    ptx::tc_fence_after();

    const bool uses = zp >= z0 + lz - 1 && zp <= z0 + lz + 1;  // warp-uniform (layer = warp / 2)
    if (uses) {
      uint32_t sv[kMaxKeys];
#pragma unroll
      for (int q = 0; q < kMaxKeys / 16; ++q)
        if (q * 16 < a.NP) ptx::tmem_ld16_sync(tS + 16 * q, sv + 16 * q);
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < kMaxKeys; ++k) {
        const float sk = (mask[k >> 5] >> (k & 31)) & 1u ? __uint_as_float(sv[k]) : -INFINITY;
        sv[k] = __float_as_uint(sk);
        mx = fmaxf(mx, sk);
      }
      const float mxs = mx * c;
      float f = 1.f;
      if (m_used == -INFINITY) {
        m_used = mxs;            // first plane this row sees: its O row is still zero
      } else if (mxs > m_used + kRescaleThreshold) {
        f = ptx::ex2(m_used - mxs);
        m_used = mxs;
      }
      // A row with no allowed key yet (only rows of sites outside the volume)
      // keeps P = 0 instead of exp2(-inf + inf).
      const float nm = m_used == -INFINITY ? 0.f : -m_used;
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxKeys / 16; ++q) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(sv[16 * q + 2 * k]), c, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(sv[16 * q + 2 * k + 1]), c, nm));
          rs += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        if (q * 16 < a.NP) ptx::tmem_st8(tP + 8 * q, pk);
      }
      if (__any_sync(0xffffffffu, f != 1.f)) {
        // PV of the previous plane completed before this plane's gather was
        // waited on, so O is stable.
        uint32_t r[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          ptx::tmem_ld32_sync(tO + 32 * q, r);
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
          ptx::tmem_st32(tO + 32 * q, r);
        }
      }
      l = l * f + rs;
    } else {
      uint32_t zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < kMaxKeys / 16; ++q)
        if (q * 16 < a.NP) ptx::tmem_st8(tP + 8 * q, zero);
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      for (int kk = 0; kk < a.NP / 16; ++kk)
        ptx::mma_ts(tO, tmem + 128 + kk * 8, ptx::smem_desc_sw128(vt + kk * 2048, 8192, 1024), idescPV,
                    (p > 0 || kk > 0) ? 1u : 0u);
      ptx::tc_commit(bar);
    }
    __syncwarp();
    if (!(ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar, phase, abort_flag)))) break;
    phase ^= 1;
    ptx::tc_fence_after();
    // The buffer this plane used is free again: prefetch plane p + 2 into it.
    if (p + 2 < nplanes) gather_plane(a, kt, vt, g, zlo + p + 2, y0, x0);
    ptx::cp_async_commit();
  }

  if (ok) {
    uint32_t r[2][32];
    ptx::tmem_ld64_sync(tO, &r[0][0]);
    if (qi >= 0) {
      const float inv = 1.f / l;
      float4* o = reinterpret_cast<float4*>(a.oloc + ((size_t)qi * a.Hq + h) * kDh);
#pragma unroll
      for (int q = 0; q < kDh / 4; ++q)
        o[q] = make_float4(__uint_as_float(r[q / 8][(4 * q) % 32]) * inv,
                           __uint_as_float(r[q / 8][(4 * q + 1) % 32]) * inv,
                           __uint_as_float(r[q / 8][(4 * q + 2) % 32]) * inv,
                           __uint_as_float(r[q / 8][(4 * q + 3) % 32]) * inv);
    }
  }
  ptx::cp_async_wait_all();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
  if (tid == 0 && *abort_flag) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_local(const Shape& s, int dtype, int flags, const int32_t* g2p, const void* qr,
                         const void* kr, const void* vl, float* oloc, int32_t* err, cudaStream_t st) {
  if (!(flags & PACK3D_FLAG_SIMT_LOCAL) && local_attn_tc_supported(s, dtype))
    return launch_local_attn_tc(s, g2p, qr, kr, vl, oloc, err, st);
  return launch_local_attn(s, dtype, g2p, qr, kr, vl, oloc, st);
}

bool local_attn_tc_supported(const Shape& s, int dtype) {
  return dtype == PACK3D_BF16 && s.G == 4 && s.rz == 1 && s.ry <= 3 && s.rx <= 3;
}

cudaError_t launch_local_attn_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, float* oloc, int32_t* err, cudaStream_t st) {
  LocalArgs a;
  a.Z = s.Z; a.H = s.H; a.W = s.W; a.Hq = s.Hq; a.Hkv = s.Hkv;
  a.ry = s.ry; a.rx = s.rx;
  a.PH = 4 + 2 * s.ry; a.PW = 4 + 2 * s.rx;
  a.NP = (a.PH * a.PW + 15) / 16 * 16;
  a.scale_log2 = s.scale_log2;
  a.g2p = g2p;
  a.q = (const __nv_bfloat16*)qr;
  a.k = (const __nv_bfloat16*)kr;
  a.v = (const __nv_bfloat16*)vl;
  a.oloc = oloc;
  a.err = err;
  cudaError_t e = cudaFuncSetAttribute(local_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(((s.Z + 1) / 2) * ((s.H + 3) / 4) * ((s.W + 3) / 4)), s.Hkv);
  local_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace pack3d
