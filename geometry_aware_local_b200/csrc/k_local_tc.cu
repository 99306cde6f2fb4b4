// Exact local attention on sm_100a tensor cores ("Geometry Matters in Packed 3D
// Attention", Key design 3: softmax attention of each token over the tokens of
// its clipped lattice box, found through the grid-to-packed map, with no
// gathered neighbour tensor in global memory).
//
// Work item = one 2 x 4 x 4 brick of query sites and one kv head; with the
// G = 4 query heads of a kv head stacked, that is 128 rows = one tcgen05 M tile
// (row = site * 4 + head, sites z-major, so rows 0-63 are the brick's first
// z layer and rows 64-127 its second).  The keys of the brick's halo are
// taken one key unit at a time: half of a lattice z-plane of the halo, i.e.
// (2 + ry) rows of (4 + 2rx) sites (at most 5 x 10 = 50 keys), padded to
// NU <= 64 keys.  Per unit:
//   S = Q K^T  (M=128, N=NU, K=64; A, B from shared memory) into one of three
//   S / P buffers of tensor memory;
//   softmax on the rows whose z window contains the unit's plane (the other
//   layer's warps write P = 0): the lattice-box mask is a per-row bit mask of
//   the unit (the same for every plane of the brick), the running maximum
//   moves lazily (only by more than 2^8) and O is rescaled in tensor memory
//   when it does; P (packed bf16) is written over the columns S occupied;
//   O += P V  (M=128, N=64, K=NU; A = P from tensor memory, B = V from shared
//   memory, MN-major).
// The kernel is persistent: CTA c takes items c, c + grid, c + 2 grid, ...,
// and the units of its items form one stream, so the gathers and MMAs of the
// next item start while the current one's last units and epilogue run.  The
// query tile is triple-buffered.  One O accumulator suffices: the softmax warps
// read an item's O out (and signal o_free) before they write the next item's
// first P, which its first O += P V needs anyway.
// Warp roles (224 threads, two CTAs per SM):
//   * warps 0-3, softmax: thread = row = tensor-memory lane;
//   * warp 4, S: issues S of unit t+3 once O += P V of unit t has freed its
//     S / P buffer and the unit's keys (and, at an item's first unit, its query
//     tile) have landed;
//   * warp 5, P V: issues O += P V of unit t once P(t) is written, never held
//     up by the S of a later item;
//   * warp 6, gather: the next item's query rows at the start of each item,
//     then each unit's K and V rows, through the index map into shared memory
//     with cp.async (keys outside the volume and padding zero-filled, 128-byte
//     swizzle), completion signalled on mbarriers; a K / V slot is refilled
//     once O += P V has read it.
// An item's output rows leave through its own query tile (no longer read by
// then): each softmax warp stages its 32 rows there, half a row at a time, and
// writes them back as whole 128-byte segments, instead of every thread
// storing its own 256-byte row (32 cache lines per warp instruction); the
// gather warp refills a query tile once q_out says its output has left.
// Tensor memory: S / P buffers at columns 0, 64 and 128, O at 192.
// Supported: bf16, G = 4, rz = 1, ry <= 3, rx <= 3 (the SIMT kernel covers the
// rest).  Every mbarrier wait is bounded; a CTA that gives up lets its issued
// copies and MMAs complete before it frees tensor memory.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace pack3d {
namespace {

constexpr int kRows = 128;
constexpr int kSWarp = 4, kPVWarp = 5, kGatherWarp = 6;
constexpr int kThreads = 32 * 7;
constexpr int kUnitKeys = 64;                     // padded keys per unit (half a halo plane)
constexpr int kTileBytes = kUnitKeys * kDh * 2;   // 8 KiB
constexpr int kSlots = 3;                         // K / V unit slots
constexpr int kQBufs = 3;                         // query tiles
constexpr int kQBytes = kRows * kDh * 2;          // 16 KiB query tile
constexpr int kSlotOff = kQBufs * kQBytes;        // slot s: K at kSlotOff + 2 s kTileBytes, V after it
constexpr int kBarOff = kSlotOff + kSlots * 2 * kTileBytes;
constexpr int kSP = 3;                            // S / P buffers in tensor memory
// barriers: q_full[3], q_free[3], kv_full[kSlots], slot_free[kSlots], s_full[kSP], p_full[kSP],
// pv_done[kSP], o_free, q_out[kQBufs], drain[2]
constexpr int kNumBars = 2 * kQBufs + 2 * kSlots + 3 * kSP + 1 + kQBufs + 2;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;   // + barriers, wait control, alignment slack
constexpr int kCtasPerSm = 2;
static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");
constexpr int kTmemCols = 256;                    // S / P buffer b at 64 b, O at 192
constexpr int kColO = 64 * kSP;
constexpr float kRescaleThreshold = 8.0f;

struct LocalArgs {
  int Z, H, W, Hq, Hkv;
  int ry, rx, PW;          // window radii in y and x, halo plane width (4 + 2rx)
  int UR, UK, NU;          // plane rows per unit (2 + ry), keys per unit, padded to NU (multiple of 16)
  int nitems;              // bricks x kv heads
  float scale_log2;
  const int32_t* g2p;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  float* oloc;
  float* stats;            // nullable: lse2 of each row to stats[4 row]
  int32_t* err;
  unsigned long long wait_ns;  // limit of every pipeline wait
  int stall;               // diagnostic: the score MMA of the CTA's last unit is never issued
};

// One work item: brick origin, kv head, the in-volume planes z0-1 .. z0+2 of
// its halo (unit u = half u % 2 of plane zlo + u / 2).
struct Item {
  int g, x0, y0, z0, zlo, nunits;
};

__device__ __forceinline__ Item decode_item(const LocalArgs& a, int i) {
  Item it;
  it.g = i % a.Hkv;
  const int b = i / a.Hkv;
  const int nbx = (a.W + 3) / 4, nby = (a.H + 3) / 4;
  it.x0 = (b % nbx) * 4;
  it.y0 = ((b / nbx) % nby) * 4;
  it.z0 = (b / (nbx * nby)) * 2;
  it.zlo = max(0, it.z0 - 1);
  it.nunits = 2 * (min(a.Z - 1, it.z0 + 2) - it.zlo + 1);
  return it;
}

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

// Packed index of query row `row` of an item (site row / 4 of the brick), or -1 outside the volume.
__device__ __forceinline__ int query_index(const LocalArgs& a, const Item& it, int row) {
  const int site = row >> 2;
  const int qz = it.z0 + (site >> 4), qy = it.y0 + ((site >> 2) & 3), qx = it.x0 + (site & 3);
  return (qz < a.Z && qy < a.H && qx < a.W) ? __ldg(a.g2p + ((size_t)qz * a.H + qy) * a.W + qx) : -1;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm) local_attn_tc_kernel(const LocalArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + kBarOff;
  constexpr int kB = 2 * kQBufs + 2 * kSlots;
  auto q_full = [&](int c) { return bar0 + 8 * c; };                   // query tile c loaded
  auto q_free = [&](int c) { return bar0 + 8 * (kQBufs + c); };        // S MMAs done reading tile c
  auto kv_full = [&](int s) { return bar0 + 8 * (2 * kQBufs + s); };   // slot s holds K and V
  auto slot_free = [&](int s) { return bar0 + 8 * (2 * kQBufs + kSlots + s); };  // O += P V read slot s
  auto s_full = [&](int b) { return bar0 + 8 * (kB + b); };                 // S in buffer b
  auto p_full = [&](int b) { return bar0 + 8 * (kB + kSP + b); };           // P in buffer b, O rescaled
  auto pv_done = [&](int b) { return bar0 + 8 * (kB + 2 * kSP + b); };      // O += P V from buffer b done
  auto o_free = [&]() { return bar0 + 8 * (kB + 3 * kSP); };                // the item's O read out
  auto q_out = [&](int c) { return bar0 + 8 * (kB + 3 * kSP + 1 + c); };    // query tile c's output stored
  auto drain = [&](int w) { return bar0 + 8 * (kB + 3 * kSP + 1 + kQBufs + w); };  // abort path: warp w's MMAs completed
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + 8 * kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * kNumBars + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int c = 0; c < kQBufs; ++c) {
      ptx::mbar_init(q_full(c), 32);           // one cp.async arrival per gather thread
      ptx::mbar_init(q_free(c), 1);
    }
    for (int c = 0; c < kSP; ++c) {
      ptx::mbar_init(s_full(c), 1);
      ptx::mbar_init(p_full(c), 4);            // one arrival per softmax warp
      ptx::mbar_init(pv_done(c), 1);
    }
    ptx::mbar_init(o_free(), 4);
    for (int c = 0; c < kQBufs; ++c) ptx::mbar_init(q_out(c), 4);
    for (int s = 0; s < kSlots; ++s) {
      ptx::mbar_init(kv_full(s), 32);
      ptx::mbar_init(slot_free(s), 1);
    }
    ptx::mbar_init(drain(0), 1);
    ptx::mbar_init(drain(1), 1);
    ctl->abort = 0;
    ctl->issued = 0;
    ctl->limit_ns = a.wait_ns;
    ptx::fence_mbar_init();
  }
  if (warp == kSWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto q_tile = [&](int k) { return sbase + (k % kQBufs) * kQBytes; };
  auto k_tile = [&](int t) { return sbase + kSlotOff + (t % kSlots) * 2 * kTileBytes; };

  if (warp == kGatherWarp) {
    // ---------------- gather: query rows lane + 32 i, K / V rows lane and lane + 32 ----------------
    int r[2], kyr[2], kxo[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      r[i] = lane + 32 * i;
      kyr[i] = r[i] / a.PW;
      kxo[i] = r[i] % a.PW;
    }
    auto key_index = [&](const Item& it, int u, int i) {
      const int y = it.y0 - a.ry + (u & 1) * a.UR + kyr[i];
      const int x = it.x0 - a.rx + kxo[i];
      return (r[i] < a.UK && x >= 0 && x < a.W && y >= 0 && y < a.H)
                 ? __ldg(a.g2p + ((size_t)(it.zlo + (u >> 1)) * a.H + y) * a.W + x)
                 : -1;
    };
    // Query rows of item k (lane + 32 rr) into query tile k % kQBufs, once the S
    // MMAs of item k - kQBufs have finished reading that tile.
    auto load_query = [&](int k, int i) {
      // The tile's previous item: its S MMAs are done and its output has left the tile.
      if (k >= kQBufs && !(wait(q_free(k % kQBufs), ((k / kQBufs) - 1) & 1) &&
                           wait(q_out(k % kQBufs), ((k / kQBufs) - 1) & 1)))
        return false;
      const Item it = decode_item(a, i);
      int qi[4];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) qi[rr] = query_index(a, it, lane + 32 * rr);
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int row = lane + 32 * rr;
        const int h = it.g * 4 + (row & 3);
        gather_row(q_tile(k), row, qi[rr] >= 0 ? a.q + ((size_t)qi[rr] * a.Hq + h) * kDh : nullptr, a.q);
      }
      ptx::cp_async_mbar_arrive(q_full(k % kQBufs));
      return true;
    };
    bool ok = blockIdx.x < a.nitems ? load_query(0, blockIdx.x) : true;
    int t = 0;
    for (int k = 0, i = blockIdx.x; ok && i < a.nitems; ++k, i += gridDim.x) {
      const Item it = decode_item(a, i);
      int j[2] = {key_index(it, 0, 0), key_index(it, 0, 1)};
      if (i + gridDim.x < a.nitems && !(ok = load_query(k + 1, i + gridDim.x))) break;
      for (int u = 0; u < it.nunits; ++u, ++t) {
        if (t >= kSlots && !(ok = wait(slot_free(t % kSlots), ((t / kSlots) - 1) & 1))) break;
        const uint32_t kt = k_tile(t), vt = kt + kTileBytes;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          gather_row(kt, r[q], j[q] >= 0 ? a.k + ((size_t)j[q] * a.Hkv + it.g) * kDh : nullptr, a.k);
          gather_row(vt, r[q], j[q] >= 0 ? a.v + ((size_t)j[q] * a.Hkv + it.g) * kDh : nullptr, a.v);
        }
        ptx::cp_async_mbar_arrive(kv_full(t % kSlots));
        if (u + 1 < it.nunits) {
          j[0] = key_index(it, u + 1, 0);
          j[1] = key_index(it, u + 1, 1);
        }
      }
    }
  } else if (warp == kSWarp || warp == kPVWarp) {
    // ---------------- MMA issue (lane 0 of the S warp and of the P V warp) ----------------
    if (lane == 0) {
      const uint32_t idescS = ptx::idesc_bf16_f32(kRows, a.NU, false);
      const uint32_t idescPV = ptx::idesc_bf16_f32(kRows, kDh, true);
      // Cursor over the CTA's unit stream: item number k, item index i, unit u, global unit t.
      int k = 0, i = blockIdx.x, u = 0, t = 0;
      int n = i < a.nitems ? decode_item(a, i).nunits : 0;
      auto next = [&]() {
        ++t;
        if (++u == n) {
          ++k;
          i += gridDim.x;
          u = 0;
          n = i < a.nitems ? decode_item(a, i).nunits : 0;
        }
      };
      int total = 0;
      for (int ii = blockIdx.x; ii < a.nitems; ii += gridDim.x) total += decode_item(a, ii).nunits;
      bool ok = true;
      if (warp == kSWarp) {
        // S(t) into buffer t % 3 once K(t) (and, at an item's first unit, its query tile) has
        // landed and O += P V(t-3) has read that buffer's P.  (PACK3D_FLAG_DIAG_STALL
        // withholds the S of the CTA's last unit.)
        const int s_units = a.stall ? total - 1 : total;
        for (; ok && t < s_units; next()) {
          if (!(ok = wait(kv_full(t % kSlots), (t / kSlots) & 1))) break;
          if (u == 0 && !(ok = wait(q_full(k % kQBufs), (k / kQBufs) & 1))) break;
          if (t >= kSP && !(ok = wait(pv_done(t % kSP), ((t / kSP) - 1) & 1))) break;
          ptx::tc_fence_after();
          ptx::fence_proxy_async_smem();   // the gathered tiles were written by cp.async
          const uint32_t kt = k_tile(t), qt = q_tile(k);
#pragma unroll
          for (int kk = 0; kk < kDh / 16; ++kk)
            ptx::mma_ss(tmem + 64 * (t % kSP), ptx::smem_desc_sw128(qt + kk * 32, 16, 1024),
                        ptx::smem_desc_sw128(kt + kk * 32, 16, 1024), idescS, kk > 0);
          ptx::tc_commit(s_full(t % kSP));
          if (u == n - 1) ptx::tc_commit(q_free(k % kQBufs));   // the item's last read of its query tile
        }
      } else {
        // O(item) += P(t) V(t) once the softmax warps have written P(t); an item's first unit
        // starts O afresh once the softmax warps have read out the previous item's.
        for (; ok && t < total; next()) {
          if (!(ok = wait(p_full(t % kSP), (t / kSP) & 1))) break;
          if (u == 0 && k >= 1 && !(ok = wait(o_free(), (k - 1) & 1))) break;
          ptx::tc_fence_after();
          ptx::fence_proxy_async_smem();   // the gathered V tile was written by cp.async
          const uint32_t vt = k_tile(t) + kTileBytes;
          const uint32_t tO = tmem + kColO;
          for (int kk = 0; kk < a.NU / 16; ++kk)
            ptx::mma_ts(tO, tmem + 64 * (t % kSP) + kk * 8, ptx::smem_desc_sw128(vt + kk * 2048, 8192, 1024),
                        idescPV, (u > 0 || kk > 0) ? 1u : 0u);
          ptx::tc_commit(pv_done(t % kSP));
          ptx::tc_commit(slot_free(t % kSlots));
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: thread = row = tensor-memory lane ----------------
    const int site = tid >> 2, hh = tid & 3;
    const int lz = site >> 4, ly = (site >> 2) & 3, lx = site & 3;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const float c = a.scale_log2;
    bool ok = true;
    int t = 0, sb = 0, sph = 0;   // unit count, its S / P buffer and that buffer's phase
    for (int k = 0, i = blockIdx.x; ok && i < a.nitems; ++k, i += gridDim.x) {
      const Item it = decode_item(a, i);
      const int qi = query_index(a, it, tid);   // where this row's output goes (read at the item's end)
      const bool qvalid = it.z0 + lz < a.Z && it.y0 + ly < a.H && it.x0 + lx < a.W;
      // Lattice-box mask of this row over each half's unit (bit k = key k of the
      // unit allowed): plane row ky = half * UR + k / PW and column kx = k % PW
      // must lie in [ly, ly + 2ry] x [lx, lx + 2rx] and inside the volume.  It is
      // the same for every plane of the brick.
      uint32_t mask0[2], mask1[2];   // half 0 / half 1 of a plane, bits 0-31 and 32-63
      {
        uint32_t xvalid = 0;
        for (int kx = 0; kx < a.PW; ++kx) {
          const int x = it.x0 - a.rx + kx;
          if (x >= 0 && x < a.W) xvalid |= 1u << kx;
        }
        const uint32_t xbits = qvalid ? (((1u << (2 * a.rx + 1)) - 1u) << lx) & xvalid : 0u;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint64_t m = 0;
          for (int kr = 0; kr < a.UR; ++kr) {
            const int ky = half * a.UR + kr, y = it.y0 - a.ry + ky;
            if (ky >= ly && ky <= ly + 2 * a.ry && y >= 0 && y < a.H) m |= (uint64_t)xbits << (kr * a.PW);
          }
          (half ? mask1 : mask0)[0] = (uint32_t)m;
          (half ? mask1 : mask0)[1] = (uint32_t)(m >> 32);
        }
      }
      const uint32_t tO = trow + kColO;
      float m_used = -INFINITY, l = 0.f;
      for (int u = 0; u < it.nunits; ++u, ++t) {
        const int zp = it.zlo + (u >> 1);
        const bool uses = zp >= it.z0 + lz - 1 && zp <= it.z0 + lz + 1;  // warp-uniform (layer = warp / 2)
        const uint32_t tS = trow + 64 * sb;
        if (!(ok = __all_sync(0xffffffffu, wait(s_full(sb), sph)))) break;
        ptx::tc_fence_after();
        if (uses) {
          uint32_t sv[kUnitKeys];
          ptx::tmem_ld64_sync(tS, sv);
          // Masked row maximum: 8 independent max3 chains.
          const uint32_t mk[2] = {(u & 1) ? mask1[0] : mask0[0], (u & 1) ? mask1[1] : mask0[1]};
          float m8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
          for (int kk = 0; kk < kUnitKeys; kk += 2) {
            const float s0 = (mk[kk >> 5] >> (kk & 31)) & 1u ? __uint_as_float(sv[kk]) : -INFINITY;
            const float s1 = (mk[kk >> 5] >> ((kk + 1) & 31)) & 1u ? __uint_as_float(sv[kk + 1]) : -INFINITY;
            sv[kk] = __float_as_uint(s0);
            sv[kk + 1] = __float_as_uint(s1);
            float& mq = m8[(kk >> 1) & 7];
            asm("max.f32 %0, %0, %1, %2;" : "+f"(mq) : "f"(s0), "f"(s1));
          }
          const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          const float mxs = mx * c;
          float f = 1.f;
          if (m_used == -INFINITY) {
            m_used = mxs;            // first unit this row sees a key in: its O row is still zero
          } else if (mxs > m_used + kRescaleThreshold) {
            f = ptx::ex2(m_used - mxs);
            m_used = mxs;
          }
          // A row with no allowed key yet (only rows of sites outside the volume)
          // keeps P = 0 instead of exp2(-inf + inf).
          const float nm = m_used == -INFINITY ? 0.f : -m_used;
          const float2 c2 = make_float2(c, c), nm2 = make_float2(nm, nm);
          float2 r2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int q = 0; q < kUnitKeys / 16; ++q) {
            uint32_t pk[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const int e = 16 * q + 2 * kk;
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2, nm2);
              const float2 pe = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
              r2[kk & 1] = __fadd2_rn(r2[kk & 1], pe);
              pk[kk] = pack_bf16x2(pe.x, pe.y);
            }
            ptx::tmem_st8(tS + 8 * q, pk);   // P over the S columns this warp has read
          }
          if (__any_sync(0xffffffffu, f != 1.f)) {
            // O is rescaled once O += P V of the item's previous unit has completed,
            // before this unit's O += P V is issued.
            if (!(ok = __all_sync(0xffffffffu, wait(pv_done(sb == 0 ? kSP - 1 : sb - 1), sb == 0 ? sph ^ 1 : sph)))) break;
            ptx::tc_fence_after();
            uint32_t o[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              ptx::tmem_ld32_sync(tO + 32 * q, o);
#pragma unroll
              for (int kk = 0; kk < 32; ++kk) o[kk] = __float_as_uint(__uint_as_float(o[kk]) * f);
              ptx::tmem_st32(tO + 32 * q, o);
            }
          }
          l = l * f + ((r2[0].x + r2[0].y) + (r2[1].x + r2[1].y));
        } else {
          const uint32_t zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
          for (int q = 0; q < kUnitKeys / 16; ++q) ptx::tmem_st8(tS + 8 * q, zero);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full(sb));
        if (++sb == kSP) {   // the S / P buffer and its phase of the next unit
          sb = 0;
          sph ^= 1;
        }
      }
      if (!ok) break;
      // The item's output: its last O += P V has completed.
      if (!(ok = __all_sync(0xffffffffu, wait(pv_done(sb == 0 ? kSP - 1 : sb - 1), sb == 0 ? sph ^ 1 : sph)))) break;
      ptx::tc_fence_after();
      uint32_t o[2][32];
      ptx::tmem_ld64_sync(tO, &o[0][0]);
      // O is in registers: the next item's first O += P V may overwrite it.
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(o_free());
      const float inv = 1.f / l;
      if (a.stats && qi >= 0) a.stats[4 * ((size_t)qi * a.Hq + it.g * 4 + hh)] = m_used + log2f(l);
      // Rows 32 warp .. 32 warp + 31 of the item's query tile hold this warp's
      // staging: row r, 16-byte chunk c at r * 128 + (c ^ (r % 8)) * 16.
      const uint32_t stg = q_tile(k) + warp * 32 * 128;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          ptx::st_shared_v4(stg + lane * 128 + ((cc ^ (lane & 7)) << 4),
                            __float_as_uint(__uint_as_float(o[half][4 * cc]) * inv),
                            __float_as_uint(__uint_as_float(o[half][4 * cc + 1]) * inv),
                            __float_as_uint(__uint_as_float(o[half][4 * cc + 2]) * inv),
                            __float_as_uint(__uint_as_float(o[half][4 * cc + 3]) * inv));
        __syncwarp();
        // Four rows per instruction: lanes 8 r' .. 8 r' + 7 write row 4 s + r' of the warp.
#pragma unroll
        for (int s4 = 0; s4 < 8; ++s4) {
          const int rw = 4 * s4 + (lane >> 3), cc = lane & 7;
          const int dst_i = __shfl_sync(0xffffffffu, qi, rw);
          const uint4 v = ptx::ld_shared_v4(stg + rw * 128 + ((cc ^ (rw & 7)) << 4));
          if (dst_i >= 0)
            *reinterpret_cast<uint4*>(a.oloc + ((size_t)dst_i * a.Hq + it.g * 4 + (rw & 3)) * kDh + 32 * half +
                                      4 * cc) = v;
        }
        __syncwarp();
      }
      if (lane == 0) ptx::mbar_arrive(q_out(k % kQBufs));   // the query tile may be refilled
    }
  }

  ptx::cp_async_wait_all();            // the gather warp's copies
  ptx::tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    // The flag is final here (every role has finished).  The MMAs each issuing
    // warp started complete before tensor memory is released.
    if ((warp == kSWarp || warp == kPVWarp) && lane == 0) {
      ptx::tc_commit(drain(warp - kSWarp));
      ptx::mbar_wait_drain(drain(warp - kSWarp), 0, ctl->limit_ns);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == kSWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
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
  a.PW = 4 + 2 * s.rx;
  a.UR = 2 + s.ry;                        // half of the 4 + 2ry plane rows
  a.UK = a.UR * a.PW;                     // <= 50 keys
  a.NU = (a.UK + 15) / 16 * 16;           // <= 64
  a.nitems = ((s.Z + 1) / 2) * ((s.H + 3) / 4) * ((s.W + 3) / 4) * s.Hkv;
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
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = min(a.nitems, kCtasPerSm * max(1, sms));
  local_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace pack3d
