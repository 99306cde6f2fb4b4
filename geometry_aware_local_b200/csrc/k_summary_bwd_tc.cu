// Backward of the query x summary branch on sm_100a tensor cores.
//
// "Geometry Matters in Packed 3D Attention", Key design 3 (every query against
// all M summaries with its own softmax), differentiated for the training
// block.  With c = scale * log2(e), lse2 the row's saved log-sum-exp (base 2),
// gamma1 the row's compressed gate weight and D = <gamma1 dout, o_cmp>:
//   P  = 2^(c S - lse2),  S = Q k~^T          (recomputed, never stored)
//   dP = dout v~^T                            (gamma1 applied per row)
//   dS = P (gamma1 dP - D)
//   dQ_rot += scale dS k~,  dk~ += scale dS^T Q_rot,  dv~ += (gamma1 P)^T dout.
// Two kernels, neither with an [N, M] tensor in memory:
//
// summary_bwd_dq_tc_kernel (query side): one 128-row query tile per CTA (rows
//   are (token, q head) pairs of one kv group, as in the forward), 64 summaries
//   per step, two CTAs per SM.  Per step the MMA warp issues S = Q k~^T and
//   dP = dout v~^T (M=128, N=64, K=64) into tensor memory; the softmax warps
//   (thread = row) read both, write dS as packed bf16 into tensor memory, and
//   the MMA warp accumulates dQ += dS k~ (A = dS from tensor memory, B = the
//   same k~ tile read MN-major).  k~ / v~ tiles stream through a TMA ring.
//
// summary_bwd_dkv_tc_kernel (summary side): one 128-summary tile per CTA and a
//   range of the kv group's query rows, 128 rows per step, one CTA per SM.
//   Per step S = Q k~^T and dP = dout v~^T (M=128 rows, N=128 summaries) go to
//   tensor memory; four softmax warpgroups (one per 32-summary chunk) write
//   dS and gamma1 P as bf16 into shared memory in the 128-byte-swizzled
//   MN-major layout, and a second MMA warp accumulates dk~ += dS^T Q and
//   dv~ += (gamma1 P)^T dout (M=128 summaries, N=64, K=128 rows; A MN-major
//   from shared memory, B = the Q / dout tiles read MN-major) in tensor memory.  Each CTA adds its partial dk~ / dv~ to
//   the float outputs with vector atomics.
//
// Every mbarrier wait is bounded; a CTA that gives up raises
// PACK3D_DEVERR_TIMEOUT and drains its issued work before releasing tensor
// memory.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace pack3d {
namespace {

constexpr int kRowsPerTile = 128;
constexpr int kQTileBytes = kRowsPerTile * kDh * 2;   // 16 KiB: 128 rows x 64 bf16

struct BwdArgs {
  int M, G, Hq;
  long rows;           // query rows of one kv group: N * G
  long rows_per_split; // summary side: rows per CTA along grid.z (a multiple of 128)
  float scale_log2;
  float scale;
  const float* gate;
  const float* stats;
  float* dqr;          // query side output  [N, Hq, 64] float
  float* dks;          // summary side outputs [M, Hkv, 64] float (accumulated)
  float* dvs;
  int32_t* err;
  unsigned long long wait_ns;  // limit of every pipeline wait
  int stall;                   // diagnostic: the last operand tile is never loaded
};

// Row of the kv group's row space -> (token * Hq + head).
__device__ __forceinline__ size_t orow_of(long r, int g, int G, int Hq) {
  return (size_t)(r / G) * Hq + g * G + (int)(r % G);
}

__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  ptx::tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

// ============================================================================
// Query side
// ============================================================================
namespace q_side {

// Summaries per step: 64 (two CTAs per SM, 256 tensor-memory columns each)
// or 128 (one CTA per SM, 512 columns; S and dP as N=128 MMAs).  Measured on
// B200, forward+backward: 65k 4.82 ms (64) vs 5.39 ms (128); 262k 56.8 vs
// 65.5 ms: two CTAs that hide each other's softmax win over wider MMAs.
#ifndef PACK3D_BQ_BN
#define PACK3D_BQ_BN 64
#endif
constexpr int kBN = PACK3D_BQ_BN;
constexpr int kCtasPerSm = kBN == 64 ? 2 : 1;
constexpr int kThreads = 192;                   // 4 softmax warps, MMA warp, TMA warp
constexpr int kMmaWarp = 4, kTmaWarp = 5;
constexpr int kColS = 0, kColDP = kBN, kColDS = 2 * kBN, kColDQ = 2 * kBN + kBN / 2;
constexpr int kTmemCols = kBN == 64 ? 256 : 512;
static_assert(kColDQ + kDh <= kTmemCols, "tensor memory plan");
constexpr int kKVBytes = kBN * kDh * 2;         // 8 or 16 KiB
constexpr int kStages = 4;
constexpr int kQOff = 0, kDOOff = kQTileBytes, kStageOff = 2 * kQTileBytes;
constexpr int kStageBytes = 2 * kKVBytes;       // k~ at +0, v~ at +kKVBytes
constexpr int kBarOff = kStageOff + kStages * kStageBytes;
// barriers: full[S], empty[S], qfull, s_full, s_free, p_full, p_free, o_final, drain
constexpr int kNumBars = 2 * kStages + 7;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;
static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "CTAs per SM");
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kRowsPerTile, kBN, false);  // S, dP: N = 64 summaries
constexpr uint32_t kIdescDQ = ptx::idesc_bf16_f32(kRowsPerTile, kDh, true);  // dQ: N = 64 dims, k~ MN-major

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
summary_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                         const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int tile = blockIdx.x;
  const int T = (a.M + kBN - 1) / kBN;
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + kBarOff;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  const uint32_t qfull = bar0 + 8 * (2 * kStages);
  const uint32_t s_full = qfull + 8, s_free = qfull + 16, p_full = qfull + 24, p_free = qfull + 32,
                 o_final = qfull + 40, drain = qfull + 48;
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + kNumBars * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8 + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    ptx::mbar_init(qfull, 1);
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(s_free, 4);
    ptx::mbar_init(p_full, 4);
    ptx::mbar_init(p_free, 1);
    ptx::mbar_init(o_final, 1);
    ptx::mbar_init(drain, 1);
    ctl->abort = 0;
    ctl->limit_ns = a.wait_ns;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;   // producer: summary tiles whose loads were issued

  if (warp == kTmaWarp) {
    if (lane == 0) {
      ptx::tma_prefetch(&tmQ);
      ptx::tma_prefetch(&tmO);
      ptx::tma_prefetch(&tmK);
      ptx::tma_prefetch(&tmV);
      const int tok0 = tile * (kRowsPerTile / a.G);
      ptx::mbar_expect_tx(qfull, 2 * kQTileBytes);
      ptx::tma_load_4d(sbase + kQOff, &tmQ, 0, 0, g, tok0, qfull);
      ptx::tma_load_4d(sbase + kDOOff, &tmO, 0, 0, g, tok0, qfull);
      const int T_load = a.stall ? T - 1 : T;
      for (int j = 0; j < T_load; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !wait(empty(st), ((j / kStages) - 1) & 1)) break;
        const uint32_t dst = sbase + kStageOff + st * kStageBytes;
        ptx::mbar_expect_tx(full(st), kStageBytes);
        ptx::tma_load_3d(dst, &tmK, 0, g, j * kBN, full(st));
        ptx::tma_load_3d(dst + kKVBytes, &tmV, 0, g, j * kBN, full(st));
        issued = j + 1;
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t tS = tmem + kColS, tDP = tmem + kColDP, tDS = tmem + kColDS, tDQ = tmem + kColDQ;
      auto issue_sdp = [&](int j) {
        const uint32_t kaddr = sbase + kStageOff + (j % kStages) * kStageBytes;
        const uint32_t vaddr = kaddr + kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          ptx::mma_ss(tS, ptx::smem_desc_sw128(sbase + kQOff + kk * 32, 16, 1024),
                      ptx::smem_desc_sw128(kaddr + kk * 32, 16, 1024), kIdescS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          ptx::mma_ss(tDP, ptx::smem_desc_sw128(sbase + kDOOff + kk * 32, 16, 1024),
                      ptx::smem_desc_sw128(vaddr + kk * 32, 16, 1024), kIdescS, kk > 0);
        ptx::tc_commit(s_full);
      };
      auto issue_dq = [&](int j) {
        const uint32_t kaddr = sbase + kStageOff + (j % kStages) * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          ptx::mma_ts(tDQ, tDS + kk * 8, ptx::smem_desc_sw128(kaddr + kk * 2048, 8192, 1024), kIdescDQ,
                      (j > 0 || kk > 0) ? 1u : 0u);
        ptx::tc_commit(p_free);
        ptx::tc_commit(empty(j % kStages));
        if (j == T - 1) ptx::tc_commit(o_final);
      };
      bool ok = wait(qfull, 0) && wait(full(0), 0);
      if (ok) {
        ptx::tc_fence_after();
        issue_sdp(0);
      }
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          if (!(ok = wait(s_free, j & 1) && wait(full((j + 1) % kStages), ((j + 1) / kStages) & 1))) break;
          ptx::tc_fence_after();
          issue_sdp(j + 1);
        }
        if (!(ok = wait(p_full, j & 1))) break;
        ptx::tc_fence_after();
        issue_dq(j);
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: thread = row = tensor-memory lane ----------------
    const int lane_base = warp * 32;
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16);
    const long grow = (long)tile * kRowsPerTile + lane_base + lane;
    const bool valid = grow < a.rows;
    const size_t orow = valid ? orow_of(grow, g, a.G, a.Hq) : 0;
    // Rows past the end read zeros through TMA: with lse2 = D = gamma1 = 0 their dS is 0.
    const float lse2 = valid ? a.stats[4 * orow + 1] : 0.f;
    const float delta = valid ? a.stats[4 * orow + 3] : 0.f;
    const float w1 = valid ? gate_weights(a.gate, orow).y : 0.f;
    const float2 c2 = make_float2(a.scale_log2, a.scale_log2), nl2 = make_float2(-lse2, -lse2);
    const float2 w2 = make_float2(w1, w1), nd2 = make_float2(-delta, -delta);
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!(ok = __all_sync(0xffffffffu, wait(s_full, j & 1)))) break;
      ptx::tc_fence_after();
      // 64 columns of S and dP at a time; the tensor memory is released after
      // the last chunk is read.
#pragma unroll
      for (int h = 0; h < kBN / 64; ++h) {
        uint32_t sv[64], dv[64];
        ptx::tmem_ld64_sync(trow + kColS + 64 * h, sv);
        ptx::tmem_ld64_sync(trow + kColDP + 64 * h, dv);
        if (h == kBN / 64 - 1) warp_arrive(s_free);
        const int lim = a.M - j * kBN - 64 * h;   // columns >= lim are past the last summary
        uint32_t pk[32];
        if (lim >= 64) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])), w2, nd2);
            const float2 ds = __fmul2_rn(make_float2(ptx::ex2(x.x), ptx::ex2(x.y)), t);
            pk[k] = pack_bf16x2(ds.x, ds.y);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])), w2, nd2);
            float2 ds = __fmul2_rn(make_float2(ptx::ex2(x.x), ptx::ex2(x.y)), t);
            if (2 * k >= lim) ds.x = 0.f;
            if (2 * k + 1 >= lim) ds.y = 0.f;
            pk[k] = pack_bf16x2(ds.x, ds.y);
          }
        }
        // dS of the previous step is read by its dQ MMAs until p_free: wait
        // only now, so this step's exponentials overlap them.
        if (h == 0 && j > 0) {
          if (!(ok = __all_sync(0xffffffffu, wait(p_free, (j - 1) & 1)))) break;
          ptx::tc_fence_after();
        }
        ptx::tmem_st16(trow + kColDS + 32 * h, pk);
        ptx::tmem_st16(trow + kColDS + 32 * h + 16, pk + 16);
      }
      if (!ok) break;
      ptx::tmem_wait_st();
      warp_arrive(p_full);
    }
    if (ok && __all_sync(0xffffffffu, wait(o_final, 0))) {
      ptx::tc_fence_after();
      uint32_t r[kDh];
      ptx::tmem_ld64_sync(trow + kColDQ, r);
      if (valid) {
        float4* dst = reinterpret_cast<float4*>(a.dqr + orow * kDh);
#pragma unroll
        for (int q = 0; q < kDh / 4; ++q)
          dst[q] = make_float4(a.scale * __uint_as_float(r[4 * q]), a.scale * __uint_as_float(r[4 * q + 1]),
                               a.scale * __uint_as_float(r[4 * q + 2]), a.scale * __uint_as_float(r[4 * q + 3]));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    // Final once every role has finished: the MMAs and loads this CTA
    // started complete before its tensor and shared memory are released.
    if (warp == kMmaWarp && lane == 0) {
      ptx::tc_commit(drain);
      ptx::mbar_wait_drain(drain, 0, ctl->limit_ns);
    }
    if (warp == kTmaWarp && lane == 0) {
      ptx::mbar_wait_drain(qfull, 0, ctl->limit_ns);
      for (int j = max(0, issued - kStages); j < issued; ++j)
        ptx::mbar_wait_drain(full(j % kStages), (j / kStages) & 1, ctl->limit_ns);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && ctl->abort) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
}

}  // namespace q_side

// ============================================================================
// Summary side
// ============================================================================
namespace k_side {

constexpr int kBS = 128;                        // summaries per CTA (M of the dk~ / dv~ accumulators)
// Softmax warpgroups first (warpgroup w covers 32-summary chunks of the tile;
// a warp reads the tensor-memory lanes of its warp index mod 4), then two MMA
// warps and the TMA warp.
// Two MMA warps: the first issues each step's S and dP, the second its
// dk~ / dv~ accumulation, so that S and dP of the next step never queue
// behind the slower accumulation issue.
#ifndef PACK3D_BKV_SMWARPS
#define PACK3D_BKV_SMWARPS 16
#endif
// Softmax warps: 16 (four warpgroups, one 32-summary chunk per thread and
// step) or 8 (two chunks).  Measured on B200, forward+backward: 65k 4.45 ms
// (16) vs 4.62 ms (8); 262k 52.6 vs 55.4 ms.  With two warps per
// sub-partition the softmax's waits were exposed.
constexpr int kSoftmaxWarps = PACK3D_BKV_SMWARPS;
constexpr int kWarpgroups = kSoftmaxWarps / 4;
constexpr int kChunksPerWg = 4 / kWarpgroups;      // 32-summary chunks per thread and step
constexpr int kThreads = 32 * (kSoftmaxWarps + 3);
constexpr int kMmaWarp = kSoftmaxWarps, kMmaWarp2 = kSoftmaxWarps + 1, kTmaWarp = kSoftmaxWarps + 2;
constexpr int kColS = 0, kColDP = 128, kColDK = 256, kColDV = 320, kTmemCols = 512;
constexpr int kSumTileBytes = kBS * kDh * 2;    // 16 KiB
// Operand buffers: buffer b holds dS^T (two 16 KiB halves: summaries 0-63,
// 64-127) and then (gamma1 P)^T; step t uses buffer t % kOpBufs.  With two
// buffers a step's softmax writes while the previous step's dk~ / dv~ MMAs
// still read; with one, shared memory holds two more Q / dout stages (four).
// Measured on B200, forward+backward: 65k 4.86 ms (two) vs 4.81 ms (one);
// 262k 56.8 vs 56.6 ms.
#ifndef PACK3D_BKV_OPBUFS
#define PACK3D_BKV_OPBUFS 1
#endif
constexpr int kOpBufs = PACK3D_BKV_OPBUFS;
constexpr int kOpBytes = 4 * kQTileBytes;
constexpr int kPInOp = 2 * kQTileBytes;
constexpr int kKOff = 0, kVOff = kSumTileBytes;
constexpr int kStageOff = 2 * kSumTileBytes;
constexpr int kStageBytes = 2 * kQTileBytes;    // Q at +0, dout at +kQTileBytes
constexpr int kStages = (224 * 1024 - kStageOff - kOpBufs * kOpBytes) / kStageBytes;
constexpr int kOpOff = kStageOff + kStages * kStageBytes;
constexpr int kBarOff = kOpOff + kOpBufs * kOpBytes;
// barriers: full[S], empty[S], kvfull, o_final, s_full, s_free, p_full[kOpBufs], p_free[kOpBufs],
// drain[2] (the abort path's MMA drain of each issuing warp)
constexpr int kNumBars = 2 * kStages + 6 + 2 * kOpBufs;
static_assert(kStages >= 2, "at least two Q / dout stages");
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kRowsPerTile, kBS, false);        // S, dP: N = 128 summaries
constexpr uint32_t kIdescKV = ptx::idesc_bf16_f32_ab(kBS, kDh, true, true);        // dk~, dv~: A, B MN-major

__global__ void __launch_bounds__(kThreads, 1)
summary_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int stile = blockIdx.x;
  const long r0 = (long)blockIdx.z * a.rows_per_split;
  const long r1 = min(a.rows, r0 + a.rows_per_split);
  const int nsteps = (int)((r1 - r0 + kRowsPerTile - 1) / kRowsPerTile);
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + kBarOff;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  const uint32_t kvfull = bar0 + 8 * (2 * kStages);
  const uint32_t o_final = kvfull + 8, s_full = kvfull + 16, s_free = kvfull + 24;
  auto p_full = [&](int b) { return kvfull + 32 + 8 * b; };
  auto p_free = [&](int b) { return kvfull + 32 + 8 * kOpBufs + 8 * b; };
  auto drain = [&](int i) { return kvfull + 32 + 16 * kOpBufs + 8 * i; };
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + kNumBars * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8 + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    ptx::mbar_init(kvfull, 1);
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(s_free, kSoftmaxWarps);
    ptx::mbar_init(o_final, 1);
    for (int b = 0; b < kOpBufs; ++b) {
      ptx::mbar_init(p_full(b), kSoftmaxWarps);
      ptx::mbar_init(p_free(b), 1);
    }
    ptx::mbar_init(drain(0), 1);
    ptx::mbar_init(drain(1), 1);
    ctl->abort = 0;
    ctl->limit_ns = a.wait_ns;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;   // producer: steps whose Q / dout loads were issued

  if (warp == kTmaWarp) {
    if (lane == 0) {
      ptx::tma_prefetch(&tmQ);
      ptx::tma_prefetch(&tmO);
      ptx::tma_prefetch(&tmK);
      ptx::tma_prefetch(&tmV);
      ptx::mbar_expect_tx(kvfull, 2 * kSumTileBytes);
      ptx::tma_load_3d(sbase + kKOff, &tmK, 0, g, stile * kBS, kvfull);
      ptx::tma_load_3d(sbase + kVOff, &tmV, 0, g, stile * kBS, kvfull);
      const int nsteps_load = a.stall ? nsteps - 1 : nsteps;
      for (int t = 0; t < nsteps_load; ++t) {
        const int st = t % kStages;
        if (t >= kStages && !wait(empty(st), ((t / kStages) - 1) & 1)) break;
        const uint32_t dst = sbase + kStageOff + st * kStageBytes;
        const int tok0 = (int)((r0 + (long)t * kRowsPerTile) / a.G);
        ptx::mbar_expect_tx(full(st), kStageBytes);
        ptx::tma_load_4d(dst, &tmQ, 0, 0, g, tok0, full(st));
        ptx::tma_load_4d(dst + kQTileBytes, &tmO, 0, 0, g, tok0, full(st));
        issued = t + 1;
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    if (lane == 0) {
      const uint32_t tS = tmem + kColS, tDP = tmem + kColDP, tDK = tmem + kColDK, tDV = tmem + kColDV;
      auto issue_sdp = [&](int t) {
        const uint32_t qaddr = sbase + kStageOff + (t % kStages) * kStageBytes;
        const uint32_t oaddr = qaddr + kQTileBytes;
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          ptx::mma_ss(tS, ptx::smem_desc_sw128(qaddr + kk * 32, 16, 1024),
                      ptx::smem_desc_sw128(sbase + kKOff + kk * 32, 16, 1024), kIdescS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          ptx::mma_ss(tDP, ptx::smem_desc_sw128(oaddr + kk * 32, 16, 1024),
                      ptx::smem_desc_sw128(sbase + kVOff + kk * 32, 16, 1024), kIdescS, kk > 0);
        ptx::tc_commit(s_full);
      };
      auto issue_dkv = [&](int t) {
        const uint32_t qaddr = sbase + kStageOff + (t % kStages) * kStageBytes;
        const uint32_t oaddr = qaddr + kQTileBytes;
        const uint32_t op = sbase + kOpOff + (t % kOpBufs) * kOpBytes;
#pragma unroll
        for (int kk = 0; kk < kRowsPerTile / 16; ++kk)
          ptx::mma_ss(tDK, ptx::smem_desc_sw128(op + kk * 2048, 2 * 8192, 1024),
                      ptx::smem_desc_sw128(qaddr + kk * 2048, 8192, 1024), kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kRowsPerTile / 16; ++kk)
          ptx::mma_ss(tDV, ptx::smem_desc_sw128(op + kPInOp + kk * 2048, 2 * 8192, 1024),
                      ptx::smem_desc_sw128(oaddr + kk * 2048, 8192, 1024), kIdescKV, (t > 0 || kk > 0) ? 1u : 0u);
        ptx::tc_commit(p_free(t % kOpBufs));
        ptx::tc_commit(empty(t % kStages));
        if (t == nsteps - 1) ptx::tc_commit(o_final);
      };
      bool ok = true;
      if (warp == kMmaWarp) {
        ok = wait(kvfull, 0);
        for (int t = 0; ok && t < nsteps; ++t) {
          // S and dP of step t: stage t landed, and step t-1's softmax read S and dP.
          if (!(ok = wait(full(t % kStages), (t / kStages) & 1))) break;
          if (t > 0 && !(ok = wait(s_free, (t - 1) & 1))) break;
          ptx::tc_fence_after();
          issue_sdp(t);
        }
      } else {
        for (int t = 0; ok && t < nsteps; ++t) {
          if (!(ok = wait(p_full(t % kOpBufs), (t / kOpBufs) & 1))) break;
          ptx::tc_fence_after();
          issue_dkv(t);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: thread = query row of the step ----------------
    const int wg = warp >> 2;                    // summary chunks [kChunksPerWg wg, +kChunksPerWg) of the tile
    const int lane_base = (warp & 3) * 32;
    const int rl = lane_base + lane;             // row inside the step's tile
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16);
    const float2 c2 = make_float2(a.scale_log2, a.scale_log2);
    bool ok = true;
    for (int t = 0; t < nsteps; ++t) {
      const long grow = r0 + (long)t * kRowsPerTile + rl;
      const bool valid = grow < r1;
      const size_t orow = valid ? orow_of(grow, g, a.G, a.Hq) : 0;
      const float lse2 = valid ? a.stats[4 * orow + 1] : 0.f;
      const float delta = valid ? a.stats[4 * orow + 3] : 0.f;
      // Rows outside this CTA's range contribute nothing: gamma1 = 0 zeroes gamma1 P and dS.
      const float w1 = valid ? gate_weights(a.gate, orow).y : 0.f;
      const float2 nl2 = make_float2(-lse2, -lse2), w2 = make_float2(w1, w1), nd2 = make_float2(-delta, -delta);
      if (!(ok = __all_sync(0xffffffffu, wait(s_full, t & 1)))) break;
      ptx::tc_fence_after();
      for (int cc = 0; cc < kChunksPerWg; ++cc) {
        const int c = kChunksPerWg * wg + cc;    // 32-summary chunk of the tile
        uint32_t sv[32], dv[32];
        ptx::tmem_ld32x2_sync(trow + kColS + 32 * c, trow + kColDP + 32 * c, sv, dv);
        if (cc == kChunksPerWg - 1) warp_arrive(s_free);
        uint32_t pd[16], pp[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
          const float2 tt = __ffma2_rn(make_float2(__uint_as_float(dv[2 * k]), __uint_as_float(dv[2 * k + 1])), w2, nd2);
          const float2 p = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
          const float2 ds = __fmul2_rn(p, tt);
          const float2 pw = __fmul2_rn(p, w2);
          pd[k] = pack_bf16x2(ds.x, ds.y);
          pp[k] = pack_bf16x2(pw.x, pw.y);
        }
        // Step (t - kOpBufs)'s dk~ / dv~ MMAs read this buffer: wait for them
        // only now, so this step's first exponentials overlap them.
        if (cc == 0 && t >= kOpBufs) {
          if (!(ok = __all_sync(0xffffffffu, wait(p_free(t % kOpBufs), ((t / kOpBufs) - 1) & 1)))) break;
        }
        // Row rl of the MN-major operands: summaries 32c .. 32c+31 are 16-byte
        // chunks (c & 1) * 4 + m of half c / 2.
        const uint32_t op = sbase + kOpOff + (t % kOpBufs) * kOpBytes + (uint32_t)(c >> 1) * kQTileBytes;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t off = ptx::sw128_offset((uint32_t)rl, (uint32_t)(((c & 1) * 4 + m) * 8));
          ptx::st_shared_v4(op + off, pd[4 * m], pd[4 * m + 1], pd[4 * m + 2], pd[4 * m + 3]);
          ptx::st_shared_v4(op + kPInOp + off, pp[4 * m], pp[4 * m + 1], pp[4 * m + 2], pp[4 * m + 3]);
        }
      }
      if (!ok) break;
      ptx::fence_proxy_async_smem();
      warp_arrive(p_full(t % kOpBufs));
    }
    if (ok && __all_sync(0xffffffffu, wait(o_final, 0))) {
      ptx::tc_fence_after();
      // Accumulator lane = summary of this tile.  The warpgroups share the
      // 128 accumulator columns (dk~ 64, then dv~ 64) evenly.
      const int j = stile * kBS + rl;
      constexpr int kCols = 2 * kDh / kWarpgroups;   // 64 or 32
      const int col0 = wg * kCols;                   // in [0, 128): dk~ below 64, dv~ from 64
      const bool is_k = col0 < kDh;
      uint32_t r[kCols];
      if constexpr (kCols == 64)
        ptx::tmem_ld64_sync(trow + kColDK + col0, r);
      else
        ptx::tmem_ld32_sync(trow + kColDK + col0, r);
      if (j < a.M) {
        const float f = is_k ? a.scale : 1.f;
        float4* dst = reinterpret_cast<float4*>((is_k ? a.dks : a.dvs) + ((size_t)j * gridDim.y + g) * kDh +
                                                (col0 % kDh));
#pragma unroll
        for (int q = 0; q < kCols / 4; ++q)
          atomicAdd(dst + q, make_float4(f * __uint_as_float(r[4 * q]), f * __uint_as_float(r[4 * q + 1]),
                                         f * __uint_as_float(r[4 * q + 2]), f * __uint_as_float(r[4 * q + 3])));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    // Final once every role has finished: the MMAs of both issuing warps and
    // the producer's loads complete before tensor and shared memory are released.
    if ((warp == kMmaWarp || warp == kMmaWarp2) && lane == 0) {
      const uint32_t d = drain(warp - kMmaWarp);
      ptx::tc_commit(d);
      ptx::mbar_wait_drain(d, 0, ctl->limit_ns);
    }
    if (warp == kTmaWarp && lane == 0) {
      ptx::mbar_wait_drain(kvfull, 0, ctl->limit_ns);
      for (int t = max(0, issued - kStages); t < issued; ++t)
        ptx::mbar_wait_drain(full(t % kStages), (t / kStages) & 1, ctl->limit_ns);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && ctl->abort) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
}

}  // namespace k_side

// ---- host side ----------------------------------------------------------------

// Q-shaped bf16 tensor [N][Hq][64] viewed as [N][Hkv][G][64]: a box of 128/G
// tokens x G heads x 64 dims of one kv head is one 128-row tile.
bool map_rows(CUtensorMap* m, const Shape& s, const void* base) {
  const cuuint64_t dims[4] = {(cuuint64_t)kDh, (cuuint64_t)s.G, (cuuint64_t)s.Hkv, (cuuint64_t)s.N};
  const cuuint64_t strides[3] = {(cuuint64_t)kDh * 2, (cuuint64_t)s.G * kDh * 2, (cuuint64_t)s.Hq * kDh * 2};
  const cuuint32_t box[4] = {(cuuint32_t)kDh, (cuuint32_t)s.G, 1, (cuuint32_t)(kRowsPerTile / s.G)};
  return tma::encode_bf16_sw128(m, base, 4, dims, strides, box);
}

// Summary tensor [M][Hkv][64], boxes of `rows` summaries of one kv head.
bool map_sums(CUtensorMap* m, const Shape& s, const void* base, int rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)kDh, (cuuint64_t)s.Hkv, (cuuint64_t)s.M};
  const cuuint64_t strides[2] = {(cuuint64_t)kDh * 2, (cuuint64_t)s.Hkv * kDh * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kDh, 1, (cuuint32_t)rows};
  return tma::encode_bf16_sw128(m, base, 3, dims, strides, box);
}

BwdArgs make_args(const Shape& s, const float* gate, const float* stats, int32_t* err) {
  BwdArgs a;
  a.M = s.M;
  a.G = s.G;
  a.Hq = s.Hq;
  a.rows = (long)s.N * s.G;
  a.rows_per_split = a.rows;
  a.scale_log2 = s.scale_log2;
  a.scale = s.scale;
  a.gate = gate;
  a.stats = stats;
  a.dqr = nullptr;
  a.dks = a.dvs = nullptr;
  a.err = err;
  a.wait_ns = s.wait_ns;
  a.stall = s.stall;
  return a;
}

}  // namespace

cudaError_t launch_summary_bwd_dq_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                     const void* dout, const float* gate, const float* stats, float* dqr,
                                     int32_t* err, cudaStream_t st) {
  CUtensorMap tq, to, tk, tv;
  if (!map_rows(&tq, s, qr) || !map_rows(&to, s, dout) || !map_sums(&tk, s, ks, q_side::kBN) ||
      !map_sums(&tv, s, vs, q_side::kBN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(q_side::summary_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       q_side::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a = make_args(s, gate, stats, err);
  a.dqr = dqr;
  dim3 grid((unsigned)((a.rows + kRowsPerTile - 1) / kRowsPerTile), s.Hkv);
  q_side::summary_bwd_dq_tc_kernel<<<grid, q_side::kThreads, q_side::kSmemBytes, st>>>(tq, to, tk, tv, a);
  return cudaGetLastError();
}

cudaError_t launch_summary_bwd_dkv_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                      const void* dout, const float* gate, const float* stats, float* dks,
                                      float* dvs, int32_t* err, cudaStream_t st) {
  CUtensorMap tq, to, tk, tv;
  if (!map_rows(&tq, s, qr) || !map_rows(&to, s, dout) || !map_sums(&tk, s, ks, k_side::kBS) ||
      !map_sums(&tv, s, vs, k_side::kBS))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_side::summary_bwd_dkv_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, k_side::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a = make_args(s, gate, stats, err);
  a.dks = dks;
  a.dvs = dvs;
  // Split the kv group's rows over grid.z: at least four CTAs per SM over
  // the grid, each CTA keeping at least eight 128-row steps, and among the
  // split counts up to twice that, the one whose last wave of CTAs leaves the
  // fewest SMs idle.
  int dev = 0, sm_count = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev);
  const long sms = max(1, sm_count);
  const int tiles = (s.M + k_side::kBS - 1) / k_side::kBS;
  const long steps = (a.rows + kRowsPerTile - 1) / kRowsPerTile;
  const long units = (long)tiles * s.Hkv;
  const long lo = max(1L, min((4L * sms + units - 1) / units, steps / 8));
  long splits = lo;
  double best = 2.0;
  for (long c = lo; c <= max(lo, min(2 * lo, steps / 8)); ++c) {
    const long per = (steps + c - 1) / c;
    const long used = (steps + per - 1) / per;          // splits that get rows
    const long ctas = units * used;
    const double idle = (double)((ctas + sms - 1) / sms * sms - ctas) / (double)ctas;
    if (idle < best - 1e-9) {
      best = idle;
      splits = c;
    }
  }
  const long per_steps = (steps + splits - 1) / splits;
  a.rows_per_split = per_steps * kRowsPerTile;
  splits = (a.rows + a.rows_per_split - 1) / a.rows_per_split;
  dim3 grid((unsigned)tiles, s.Hkv, (unsigned)splits);
  k_side::summary_bwd_dkv_tc_kernel<<<grid, k_side::kThreads, k_side::kSmemBytes, st>>>(tq, to, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace pack3d
