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
// swizzled K tile and V tile.  Per plane:
//   S = Q K^T  (M=128, N=NP, K=64; A, B from shared memory)
//   softmax on the rows whose z window contains the plane (the other layer's
//   warps write P = 0): the lattice-box mask is a per-row bit mask, the
//   running maximum moves lazily (only by more than 2^8) and O is rescaled in
//   tensor memory when it does;
//   O += P V   (M=128, N=64, K=NP; A = P from tensor memory, B = V from
//   shared memory, MN-major).
// Pipelining inside the CTA: every index-map lookup of the CTA (its query row
// and its gather row of each plane) is issued at the start; three plane
// buffers hold planes 0-2 from the start and plane 3 once plane 0's MMAs are
// done; S of plane p+1 is issued as soon as every warp has read S of plane p
// into registers, so it runs under plane p's exponentials.  Two CTAs share an
// SM (256 tensor-memory columns each: S 0-111, P 128-183, O 192-255).
// Supported: bf16, G = 4, rz = 1, ry <= 3, rx <= 3 (the SIMT kernel covers the
// rest).  Every mbarrier wait is bounded, and the CTA leaves the plane loop
// only all together (barrier votes).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace pack3d {
namespace {

constexpr int kRows = 128;
constexpr int kThreads = 128;
constexpr int kMaxKeys = 112;                     // padded keys per plane
constexpr int kMaxPlanes = 4;                     // 2 brick layers + r_z = 1 on each side
constexpr int kTileBytes = kMaxKeys * kDh * 2;    // 14 KiB, a multiple of 1 KiB
constexpr int kQOff = 0;                          // 16 KiB query tile
constexpr int kKV0 = kRows * kDh * 2;             // plane buffers: K at +0, V at +kTileBytes
constexpr int kBufs = 3;
constexpr int kBufBytes = 2 * kTileBytes;
constexpr int kBarOff = kKV0 + kBufs * kBufBytes;
constexpr int kSmemBytes = kBarOff + 64 + 1024;   // + barriers and flags, + alignment slack
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");
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
  float* stats;            // nullable: lse2 of each row to stats[4 row]
  int32_t* err;
  unsigned long long wait_ns;  // limit of every pipeline wait
  int stall;               // diagnostic: the score MMA of the last plane is never issued
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

// Packed index of this thread's gather row (row r = threadIdx.x of the padded
// plane) in lattice plane zp, or -1 (padding or outside the volume).
__device__ __forceinline__ int plane_row_index(const LocalArgs& a, int zp, int y0, int x0) {
  const int r = threadIdx.x;
  if (r >= a.PH * a.PW) return -1;
  const int y = y0 - a.ry + r / a.PW, x = x0 - a.rx + r % a.PW;
  if (y < 0 || y >= a.H || x < 0 || x >= a.W) return -1;
  return __ldg(a.g2p + ((size_t)zp * a.H + y) * a.W + x);
}

// K and V rows of this thread's gather row into plane buffer (kt, vt).
__device__ __forceinline__ void gather_plane(const LocalArgs& a, uint32_t kt, uint32_t vt, int g, int j) {
  const int r = threadIdx.x;
  if (r >= a.NP) return;
  gather_row(kt, r, j >= 0 ? a.k + ((size_t)j * a.Hkv + g) * kDh : nullptr, a.k);
  gather_row(vt, r, j >= 0 ? a.v + ((size_t)j * a.Hkv + g) * kDh : nullptr, a.v);
}

__global__ void __launch_bounds__(kThreads, 2) local_attn_tc_kernel(const LocalArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t s_full = sbase + kBarOff;        // S of the current plane is in tensor memory
  const uint32_t pv_done = sbase + kBarOff + 8;   // O += P V of the last issued plane has completed
  const uint32_t drain = sbase + kBarOff + 16;    // abort path: every MMA issued so far has completed
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + 24);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 24 + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };
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
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(pv_done, 1);
    ptx::mbar_init(drain, 1);
    ctl->abort = 0;
    ctl->limit_ns = a.wait_ns;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 256);
    ptx::tmem_relinquish();
  }

  // Every index-map lookup of the CTA at once: the query row and this
  // thread's gather row of each plane z0-1 .. z0+2 inside the volume.
  const int zlo = max(0, z0 - 1), zhi = min(a.Z - 1, z0 + 2);
  const int nplanes = zhi - zlo + 1;
  const int qi = qvalid ? __ldg(a.g2p + ((size_t)qz * a.H + qy) * a.W + qx) : -1;
  int gi[kMaxPlanes];
#pragma unroll
  for (int p = 0; p < kMaxPlanes; ++p) gi[p] = p < nplanes ? plane_row_index(a, zlo + p, y0, x0) : -1;

  // cp.async groups: {Q, plane 0}, {plane 1}, {plane 2} (possibly empty), and
  // later {plane 3} into plane 0's buffer.
  auto kt_of = [&](int p) { return sbase + kKV0 + (p % kBufs) * kBufBytes; };
  gather_row(sbase + kQOff, tid, qi >= 0 ? a.q + ((size_t)qi * a.Hq + h) * kDh : nullptr, a.q);
  gather_plane(a, kt_of(0), kt_of(0) + kTileBytes, g, gi[0]);
  ptx::cp_async_commit();
  if (nplanes > 1) gather_plane(a, kt_of(1), kt_of(1) + kTileBytes, g, gi[1]);
  ptx::cp_async_commit();
  if (nplanes > 2) gather_plane(a, kt_of(2), kt_of(2) + kTileBytes, g, gi[2]);
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

  auto issue_s = [&](int p) {
    ptx::tc_fence_after();
    const uint32_t kt = kt_of(p);
#pragma unroll
    for (int kk = 0; kk < kDh / 16; ++kk)
      ptx::mma_ss(tmem, ptx::smem_desc_sw128(sbase + kQOff + kk * 32, 16, 1024),
                  ptx::smem_desc_sw128(kt + kk * 32, 16, 1024), idescS, kk > 0);
    ptx::tc_commit(s_full);
  };

  // S of plane 0 once Q and plane 0 are in shared memory (group 0 of 3).
  ptx::cp_async_wait_two();
  ptx::fence_proxy_async_smem();
  __syncthreads();
  // (PACK3D_FLAG_DIAG_STALL withholds the score MMA of the last plane.)
  if (tid == 0 && !(a.stall && nplanes == 1)) issue_s(0);

  float m_used = -INFINITY, l = 0.f;
  bool ok = true;
  for (int p = 0; p < nplanes; ++p) {
    const int zp = zlo + p;
    const bool uses = zp >= z0 + lz - 1 && zp <= z0 + lz + 1;  // warp-uniform (layer = warp / 2)
    // S of plane p; each using warp keeps its rows in registers.
    bool w_ok = __all_sync(0xffffffffu, wait(s_full, p & 1));
    uint32_t sv[kMaxKeys];
    if (w_ok) {
      ptx::tc_fence_after();
      if (uses) {
        ptx::tmem_ld64_sync(tS, sv);
        ptx::tmem_ld48_sync(tS + 64, sv + 64);
      }
    }
    // Plane p+1 landed (groups: after plane 0 one more may be pending, later none).
    if (p == 0) ptx::cp_async_wait_one(); else ptx::cp_async_wait_all();
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    if (!(ok = __syncthreads_and(w_ok))) break;
    // Every warp has read S(p): S(p+1) may overwrite it and run under this
    // plane's exponentials.
    if (tid == 0 && p + 1 < nplanes && !(a.stall && p + 2 == nplanes)) issue_s(p + 1);

    float f = 1.f, rs = 0.f;
    if (uses) {
      // Masked row maximum: 8 independent max3 chains.
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
      for (int k = 0; k < kMaxKeys; k += 2) {
        const float s0 = (mask[k >> 5] >> (k & 31)) & 1u ? __uint_as_float(sv[k]) : -INFINITY;
        const float s1 = (mask[(k + 1) >> 5] >> ((k + 1) & 31)) & 1u ? __uint_as_float(sv[k + 1]) : -INFINITY;
        sv[k] = __float_as_uint(s0);
        sv[k + 1] = __float_as_uint(s1);
        float& mq = m8[(k >> 1) & 7];
        asm("max.f32 %0, %0, %1, %2;" : "+f"(mq) : "f"(s0), "f"(s1));
      }
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mxs = mx * c;
      if (m_used == -INFINITY) {
        m_used = mxs;            // first plane this row sees: its O row is still zero
      } else if (mxs > m_used + kRescaleThreshold) {
        f = ptx::ex2(m_used - mxs);
        m_used = mxs;
      }
    }
    // P and O are free again once O += P V of plane p-1 has completed.
    if (p > 0) {
      w_ok = __all_sync(0xffffffffu, wait(pv_done, (p - 1) & 1));
      if (w_ok) ptx::tc_fence_after();
    }
    if (p == 1 && nplanes > 3 && w_ok) {
      // Plane 0's buffer (read by S(0) and O += P V of plane 0, both done) takes plane 3.
      gather_plane(a, kt_of(3), kt_of(3) + kTileBytes, g, gi[3]);
    }
    if (p == 1) ptx::cp_async_commit();
    if (uses && w_ok) {
      // A row with no allowed key yet (only rows of sites outside the volume)
      // keeps P = 0 instead of exp2(-inf + inf).
      const float nm = m_used == -INFINITY ? 0.f : -m_used;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(nm, nm);
      float2 r2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int q = 0; q < kMaxKeys / 16; ++q) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int i = 16 * q + 2 * k;
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2, nm2);
          const float2 pe = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
          r2[k & 1] = __fadd2_rn(r2[k & 1], pe);
          pk[k] = pack_bf16x2(pe.x, pe.y);
        }
        ptx::tmem_st8(tP + 8 * q, pk);
      }
      rs = (r2[0].x + r2[0].y) + (r2[1].x + r2[1].y);
      if (__any_sync(0xffffffffu, f != 1.f)) {
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
    } else if (w_ok) {
      uint32_t zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < kMaxKeys / 16; ++q) ptx::tmem_st8(tP + 8 * q, zero);
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    if (!(ok = __syncthreads_and(w_ok))) break;
    if (tid == 0) {
      ptx::tc_fence_after();
      const uint32_t vt = kt_of(p) + kTileBytes;
      for (int kk = 0; kk < a.NP / 16; ++kk)
        ptx::mma_ts(tO, tmem + 128 + kk * 8, ptx::smem_desc_sw128(vt + kk * 2048, 8192, 1024), idescPV,
                    (p > 0 || kk > 0) ? 1u : 0u);
      ptx::tc_commit(pv_done);
    }
  }

  if (ok) ok = __all_sync(0xffffffffu, wait(pv_done, (nplanes - 1) & 1));
  if (ok) {
    ptx::tc_fence_after();
    uint32_t r[2][32];
    ptx::tmem_ld64_sync(tO, &r[0][0]);
    if (qi >= 0) {
      const float inv = 1.f / l;
      if (a.stats) a.stats[4 * ((size_t)qi * a.Hq + h)] = m_used + log2f(l);
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
  if (ctl->abort) {
    // The flag is final here (every thread has left the plane loop).  The
    // MMAs thread 0 issued complete before tensor memory is released.
    if (tid == 0) {
      ptx::tc_commit(drain);
      ptx::mbar_wait_drain(drain, 0, ctl->limit_ns);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
  if (tid == 0 && ctl->abort) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_local(const Shape& s, int dtype, int flags, const int32_t* g2p, const void* qr,
                         const void* kr, const void* vl, float* oloc, int32_t* err, cudaStream_t st,
                         float* stats) {
  if (!(flags & PACK3D_FLAG_SIMT_LOCAL) && local_attn_tc_supported(s, dtype))
    return launch_local_attn_tc(s, g2p, qr, kr, vl, oloc, err, st, stats);
  return launch_local_attn(s, dtype, g2p, qr, kr, vl, oloc, st, stats);
}

bool local_attn_tc_supported(const Shape& s, int dtype) {
  return dtype == PACK3D_BF16 && s.G == 4 && s.rz == 1 && s.ry <= 3 && s.rx <= 3;
}

cudaError_t launch_local_attn_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, float* oloc, int32_t* err, cudaStream_t st, float* stats) {
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
  a.stats = stats;
  a.err = err;
  a.wait_ns = s.wait_ns;
  a.stall = s.stall;
  cudaError_t e = cudaFuncSetAttribute(local_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(((s.Z + 1) / 2) * ((s.H + 3) / 4) * ((s.W + 3) / 4)), s.Hkv);
  local_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace pack3d
