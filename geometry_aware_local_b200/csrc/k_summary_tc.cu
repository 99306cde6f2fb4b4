// Query x summary attention with the tokenwise gate on sm_100a tensor cores.
//
// "Geometry Matters in Packed 3D Attention", Key design 3: every query attends
// to all M block summaries with its own softmax, streamed with an online
// softmax so that no [N, M] score tensor exists; the overall framework's
// tokenwise two-way softmax gate mixes the result with the local branch.
//
// One CTA = kGroups 128-row query tiles of one kv head sharing every summary
// tile (rows are (token, q head) pairs of the kv group: 128/G tokens x G
// heads); the default is two tiles and 128-summary tiles (the one-tile build,
// k_summary_tc_one.cu, uses 96-summary tiles and two P buffers).
//   * the last warp streams k~ / v~ tiles (kBN summaries x 64 dims, bf16,
//     128-byte swizzle) through a TMA ring; the Q tiles are loaded once.
//   * one warp per group issues that group's tcgen05.mma: S = Q k~^T (M=128,
//     N=kBN, K=64) into tensor memory and O += P v~ (M=128, N=64, K=kBN) with P
//     read from tensor memory.  An SM accepts about one tcgen05.mma per 50
//     clocks whichever warp issues it (so the N=64 steps of O += P v~ are
//     issue bound); a warp per group lets each group's MMAs follow its own
//     barriers instead of queueing behind the other group's waits.
//   * warps 0 .. 4*kGroups-1 are the softmax warpgroups, one per query tile,
//     thread = row = TMEM lane.
// At d_h = 64 each exponential pairs with only 256 MMA flops, so the softmax
// sets the pace: packed f32x2 FMA/add, a three-input max and MUFU.ex2 (the
// one-tile build evaluates 2 of every 16 exponential pairs on the FMA pipe
// instead, which unloads MUFU).  O is
// rescaled lazily (only when a row maximum grows by more than
// 2^8).  Tensor memory, group w at w*kGroupCols: S, P (packed bf16; one or two
// buffers), O.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

// The file is compiled twice: as the two-tile kernel (namespace sa_two, the
// default) and, from k_summary_tc_one.cu, as the one-tile kernel run two
// CTAs per SM (namespace sa_one); k_summary_dispatch.cu picks per launch.
#ifndef PACK3D_SA_NS
#define PACK3D_SA_NS sa_two
#endif

namespace pack3d {
namespace PACK3D_SA_NS {
namespace {

// Compile-time shape of the pipeline: query tiles (softmax warpgroups) per
// CTA and summaries per tile.  Tensor memory per group: S (kBN columns), P
// (kBN/2 per buffer), O (64), i.e. 256 columns for (2, 128) with one P buffer
// and for (1, 96) with two.
#ifndef PACK3D_SA_GROUPS
#define PACK3D_SA_GROUPS 2
#endif
#ifndef PACK3D_SA_BN
#define PACK3D_SA_BN 128
#endif
// P buffers per group: with two, the exponentials of tile j are written while
// O += P v~ of tile j-1 still reads the other buffer (tensor memory per group:
// S kBN + 2 x kBN/2 + O 64, i.e. 256 columns at kBN = 96).
#ifndef PACK3D_SA_PBUFS
#define PACK3D_SA_PBUFS 1
#endif
// Of every 16 pairs of exponentials, this many are evaluated on the FMA pipe
// (exp2_fma) instead of MUFU, spread evenly over the pairs.
#ifndef PACK3D_SA_POLY
#define PACK3D_SA_POLY 0
#endif
constexpr int kBM = 128;                      // rows per query tile
constexpr int kBN = PACK3D_SA_BN;             // summaries per tile
constexpr int kGroups = PACK3D_SA_GROUPS;     // query tiles (softmax warpgroups) per CTA
constexpr int kMmaWarp = 4 * kGroups;          // first MMA warp; one per group
constexpr int kTmaWarp = kMmaWarp + kGroups;
constexpr int kThreads = 32 * (kTmaWarp + 1);
constexpr int kPBufs = PACK3D_SA_PBUFS;
constexpr int kColS = 0, kColP = kBN, kColO = kBN + kPBufs * (kBN / 2);
constexpr int kGroupCols = kColO + kDh;       // tensor-memory columns per group
constexpr int kQBytes = kBM * kDh * 2;        // 16 KiB
constexpr int kKVBytes = kBN * kDh * 2;
// CTAs per SM: one CTA of two tiles, or two CTAs of one tile each (then an
// SM runs two independent pipelines, each with half the tensor memory and
// shared memory).
constexpr int kCtasPerSm = kGroups == 1 ? 2 : 1;
constexpr int kSmemBudget = kCtasPerSm == 1 ? 192 * 1024 : 110 * 1024;
constexpr int kStages = ((kSmemBudget - kGroups * kQBytes) / (2 * kKVBytes)) < 8
                            ? ((kSmemBudget - kGroups * kQBytes) / (2 * kKVBytes)) : 8;
constexpr int kTmemCols = kGroups == 1 ? 256 : 512;
constexpr int kQOff = 0;
constexpr int kStageOff = kGroups * kQBytes;  // stage s: k~ at +0, v~ at +kKVBytes
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kBarOff = kStageOff + kStages * kStageBytes;
// P can be handed between the softmax warps and the MMA warp in kPChunks
// column chunks, so that O += P v~ for one chunk runs while the exponentials
// of the next are computed.  Measured on B200 at 65k tokens: 1 chunk 0.81 ms,
// 2 chunks 0.82 ms, 4 chunks 0.86 ms (the extra barriers cost more than the
// overlap gains), so the default is a single hand-off per tile.
#ifndef PACK3D_SA_PCHUNKS
#define PACK3D_SA_PCHUNKS 1
#endif
constexpr int kPChunks = PACK3D_SA_PCHUNKS;
constexpr int kPairsPerChunk = kBN / 2 / kPChunks;   // packed P columns per chunk
constexpr int kMmasPerChunk = kBN / 16 / kPChunks;   // K = 16 steps of O += P v~ per chunk
static_assert(kPairsPerChunk % 16 == 0, "P chunks are stored 16 columns at a time");
// barriers: full[S], empty[S], qfull, then per group: s_full, s_free, o_final,
// p_full[kPSlots], p_free[kPSlots] (per P chunk, or per P buffer), drain (the
// abort path's MMA drain)
static_assert(kPBufs == 1 || kPChunks == 1, "P buffers or P chunks, not both");
constexpr int kPSlots = kPChunks * kPBufs;           // p_full / p_free barriers per group
constexpr int kGroupBars = 4 + 2 * kPSlots;
constexpr int kNumBars = 2 * kStages + 1 + kGroups * kGroupBars;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr int kPoly = PACK3D_SA_POLY;
__host__ __device__ constexpr bool poly_pair(int k) { return kPoly > 0 && ((k % 16) * kPoly) % 16 < kPoly; }
static_assert(kGroups * kGroupCols <= kTmemCols, "tensor memory plan");

constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, kBN, false);      // S: N = kBN summaries
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBM, kDh, true);     // O: N = 64 dims, v~ MN-major

struct TcArgs {
  int M;             // summaries
  int G;             // q heads per kv head
  int Hq;
  long rows;         // rows of this launch end here (token end * G)
  int tile_base;     // first 128-row tile of this launch
  float scale_log2;  // softmax scale * log2(e)
  const float* oloc;
  const float* gate;
  __nv_bfloat16* out;
  float* stats;                 // training: row statistics (nullable)
  const __nv_bfloat16* dout;    // training: output gradient
  float* dgate;                 // training: gate gradient
  int32_t* err;
  unsigned long long wait_ns;   // limit of every pipeline wait
  int stall;                    // diagnostic: the last summary tile is never loaded
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// kTrain: the training block's forward (row statistics and dgate in the
// epilogue); a separate instantiation so the plain forward's code is unchanged.
template <bool kTrain>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
summary_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int tile0 = a.tile_base + blockIdx.x * kGroups;
  const int T = (a.M + kBN - 1) / kBN;

  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + kBarOff;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  const uint32_t qfull = bar0 + 8 * (2 * kStages);
  auto gbar = [&](int w, int i) { return bar0 + 8 * (2 * kStages + 1 + w * kGroupBars + i); };
  auto s_full = [&](int w) { return gbar(w, 0); };
  auto s_free = [&](int w) { return gbar(w, 1); };
  auto o_final = [&](int w) { return gbar(w, 2); };
  auto p_full = [&](int w, int c) { return gbar(w, 3 + c); };
  auto p_free = [&](int w, int c) { return gbar(w, 3 + kPSlots + c); };
  auto drain = [&](int w) { return gbar(w, 3 + 2 * kPSlots); };
  volatile ptx::WaitCtl* ctl = reinterpret_cast<volatile ptx::WaitCtl*>(smem + kBarOff + kNumBars * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8 + sizeof(ptx::WaitCtl));
  auto wait = [&](uint32_t bar, uint32_t parity) { return ptx::mbar_wait(bar, parity, ctl); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kGroups);   // one commit per group's MMA warp
    }
    ptx::mbar_init(qfull, 1);
    for (int w = 0; w < kGroups; ++w) {
      ptx::mbar_init(s_full(w), 1);
      ptx::mbar_init(s_free(w), 4);       // one arrival per softmax warp
      ptx::mbar_init(o_final(w), 1);
      ptx::mbar_init(drain(w), 1);
      for (int c = 0; c < kPSlots; ++c) {
        ptx::mbar_init(p_full(w, c), 4);
        ptx::mbar_init(p_free(w, c), 1);
      }
    }
    ctl->abort = 0;
    ctl->issued = 0;
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

  if (warp == kTmaWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::tma_prefetch(&tmQ);
      ptx::tma_prefetch(&tmK);
      ptx::tma_prefetch(&tmV);
      const int tok_per_tile = kBM / a.G;
      ptx::mbar_expect_tx(qfull, kGroups * kQBytes);
      for (int w = 0; w < kGroups; ++w)
        ptx::tma_load_4d(sbase + kQOff + w * kQBytes, &tmQ, 0, 0, g, (tile0 + w) * tok_per_tile, qfull);
      const int T_load = a.stall ? T - 1 : T;
      int issued = 0;
      for (int j = 0; j < T_load; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !wait(empty(st), ((j / kStages) - 1) & 1)) break;
        const uint32_t dst = sbase + kStageOff + st * kStageBytes;
        ptx::mbar_expect_tx(full(st), kStageBytes);
        ptx::tma_load_3d(dst, &tmK, 0, g, j * kBN, full(st));
        ptx::tma_load_3d(dst + kKVBytes, &tmV, 0, g, j * kBN, full(st));
        issued = j + 1;
      }
      ctl->issued = issued;
    }
    __syncwarp();
  } else if (warp >= kMmaWarp) {
    // ---------------- MMA issuers: one warp per group ----------------
    // A single issuing thread cannot keep up (each tcgen05.mma takes longer to
    // issue than a 128 x 64 x 16 step takes to run), so every group has its own.
    // A group's events are ordered (s_free(j), then the P chunks of tile j in
    // column order, then s_free(j+1)), so plain bounded waits in that order
    // suffice.
    const int w = warp - kMmaWarp;
    if (lane == 0) {
      const uint32_t qaddr = sbase + kQOff + w * kQBytes;
      const uint32_t tS = tmem + w * kGroupCols + kColS;
      const uint32_t tP = tmem + w * kGroupCols + kColP;
      const uint32_t tO = tmem + w * kGroupCols + kColO;
      auto issue_s = [&](int j) {
        const uint32_t kaddr = sbase + kStageOff + (j % kStages) * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          ptx::mma_ss(tS, ptx::smem_desc_sw128(qaddr + kk * 32, 16, 1024),
                      ptx::smem_desc_sw128(kaddr + kk * 32, 16, 1024), kIdesc, kk > 0);
        ptx::tc_commit(s_full(w));
      };
      auto issue_pv = [&](int j, int c) {
        const uint32_t vaddr = sbase + kStageOff + (j % kStages) * kStageBytes + kKVBytes;
        const int pb = j % kPBufs;                       // this tile's P buffer
#pragma unroll
        for (int i = 0; i < kMmasPerChunk; ++i) {
          const int kk = c * kMmasPerChunk + i;
          ptx::mma_ts(tO, tP + pb * (kBN / 2) + kk * 8, ptx::smem_desc_sw128(vaddr + kk * 2048, 8192, 1024),
                      kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::tc_commit(p_free(w, c + pb));
        if (c == kPChunks - 1) {
          ptx::tc_commit(empty(j % kStages));
          if (j == T - 1) ptx::tc_commit(o_final(w));
        }
      };
      bool ok = wait(qfull, 0) && wait(full(0), 0);
      if (ok) {
        ptx::tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          if (!(ok = wait(s_free(w), j & 1) && wait(full((j + 1) % kStages), ((j + 1) / kStages) & 1)))
            break;
          ptx::tc_fence_after();
          issue_s(j + 1);
        }
        for (int c = 0; ok && c < kPChunks; ++c) {
          if (!(ok = wait(p_full(w, c + j % kPBufs), (j / kPBufs) & 1))) break;
          ptx::tc_fence_after();
          issue_pv(j, c);
        }
      }
      if (!ok) {
        // Gave up: let this warp's MMAs complete now (phase 0 of drain(w);
        // the end of the kernel then finds it done and skips its own drain).
        ptx::tc_commit(drain(w));
        ptx::mbar_wait_drain(drain(w), 0, ctl->limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warpgroups ----------------
    const int w = warp >> 2;
    const int lane_base = (warp & 3) * 32;
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16) + w * kGroupCols;
    const uint32_t tP = trow + kColP, tO = trow + kColO;
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // Online softmax with a lazily moved maximum: m_used (log2 units) only
    // moves when a tile's row maximum exceeds it by more than 8, so P stays
    // below 2^8 and O is rescaled in tensor memory on few tiles.  S is read
    // into registers and released at once, so S for the next tile runs on the
    // tensor core while this tile's exponentials are computed.
    auto load_s = [&](uint32_t* sv, int j) {
#pragma unroll
      for (int q = 0; q < kBN / 64; ++q) ptx::tmem_ld64_sync(trow + kColS + 64 * q, sv + 64 * q);
      if constexpr (kBN % 64 == 32) ptx::tmem_ld32_sync(trow + kColS + kBN - 32, sv + kBN - 32);
      if ((j + 1) * kBN > a.M) {
        const int lim = a.M - j * kBN;
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (k >= lim) sv[k] = __float_as_uint(-INFINITY);
      }
    };
    // Row maximum over the kBN columns: 8 independent max3 chains, each chain
    // covering one column pair of every 16-column group.
    auto row_max = [&](const uint32_t* sv) {
      static_assert(kBN % 16 == 0, "row_max walks 16-column groups");
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = fmaxf(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1]));
#pragma unroll
      for (int k = 16; k < kBN; k += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          m8[q] = max3(m8[q], __uint_as_float(sv[k + 2 * q]), __uint_as_float(sv[k + 2 * q + 1]));
      return max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
    };
    // Exponentials of chunk cc of one S row, written to the P buffer 16 packed
    // columns at a time; the (unrounded) values are added to rs.
    auto exps_chunk = [&](const uint32_t* sv, int cc, float2* rs, uint32_t tPb) {
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_used, -m_used);
#pragma unroll
      for (int q = 0; q < kPairsPerChunk / 16; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int pair = cc * kPairsPerChunk + q * 16 + k;
          const float2 x =
              __ffma2_rn(make_float2(__uint_as_float(sv[2 * pair]), __uint_as_float(sv[2 * pair + 1])), c2, nm2);
          const float2 p = poly_pair(pair) ? exp2_fma(x) : make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
          rs[k & 1] = __fadd2_rn(rs[k & 1], p);
          pk[k] = pack_bf16x2(p.x, p.y);
        }
        ptx::tmem_st16(tPb + cc * kPairsPerChunk + 16 * q, pk);
      }
    };
    // One arrival per warp: every lane's tensor-memory accesses are complete
    // (waited and fenced) before the warp converges and lane 0 arrives (one
    // arrival instead of 32 per warp took 0.92 -> 0.81 ms at 65k tokens).
    auto warp_arrive = [&](uint32_t bar) {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar);
    };
    for (int j = 0; j < T; ++j) {
      if (!(ok = __all_sync(0xffffffffu, wait(s_full(w), j & 1)))) break;
      ptx::tc_fence_after();
      float f = 1.f;
      float2 rs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      {
        uint32_t sv[kBN];
        load_s(sv, j);
        warp_arrive(s_free(w));
        const float mxs = row_max(sv) * c;
        if (j == 0) m_used = mxs;
        else if (mxs > m_used + kRescaleThreshold) {
          f = ptx::ex2(m_used - mxs);
          m_used = mxs;
        }
        const bool rescale = j > 0 && __any_sync(0xffffffffu, f != 1.f);
        const int pb = j % kPBufs;                       // this tile's P buffer
#pragma unroll
        for (int cc = 0; cc < kPChunks; ++cc) {
          if (j >= kPBufs) {
            // The buffer's previous tile (j - kPBufs) has been read by its O += P v~.
            if (!(ok = __all_sync(0xffffffffu, wait(p_free(w, cc + pb), ((j / kPBufs) - 1) & 1)))) break;
            ptx::tc_fence_after();
          }
          exps_chunk(sv, cc, rs, tP + pb * (kBN / 2));
          if (cc == 0 && rescale) {
            // O is rescaled before this tile's first O += P v~ is issued and
            // after the previous tile's last one has completed (its commit
            // covers all earlier MMAs of the group).
            const int pj = j - 1;
            if (!(ok = __all_sync(0xffffffffu, wait(p_free(w, kPChunks - 1 + pj % kPBufs), (pj / kPBufs) & 1))))
              break;
            ptx::tc_fence_after();
            uint32_t r[16];
#pragma unroll
            for (int q = 0; q < kDh / 16; ++q) {
              ptx::tmem_ld16_sync(tO + 16 * q, r);
#pragma unroll
              for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
              ptx::tmem_st16(tO + 16 * q, r);
            }
          }
          ptx::tmem_wait_st();
          warp_arrive(p_full(w, cc + pb));
        }
        if (!ok) break;
      }
      l = l * f + ((rs[0].x + rs[0].y) + (rs[1].x + rs[1].y));
    }
    if (ok && __all_sync(0xffffffffu, wait(o_final(w), 0))) {
      ptx::tc_fence_after();
      uint32_t r[2][32];
      ptx::tmem_ld64_sync(tO, &r[0][0]);
      const long grow = (long)(tile0 + w) * kBM + lane_base + lane;
      if (grow < a.rows) {
        const long tok = grow / a.G;
        const int h = g * a.G + (int)(grow % a.G);
        const size_t orow = (size_t)tok * a.Hq + h;
        const float inv = 1.f / l;
        float o[kDh];
#pragma unroll
        for (int e = 0; e < kDh; ++e) o[e] = __uint_as_float(r[e >> 5][e & 31]) * inv;
        if constexpr (kTrain)
          train_epilogue_row(o, a.gate, a.oloc, a.dout, orow, m_used + log2f(l), a.stats, a.dgate);
        if (a.gate != nullptr) {
          const float g0 = __ldg(a.gate + 2 * orow), g1 = __ldg(a.gate + 2 * orow + 1);
          const float gm = fmaxf(g0, g1);
          const float e0 = expf(g0 - gm), e1 = expf(g1 - gm);
          const float w0 = e0 / (e0 + e1), w1 = e1 / (e0 + e1);
          const float4* lo = reinterpret_cast<const float4*>(a.oloc + orow * kDh);
#pragma unroll
          for (int q = 0; q < kDh / 4; ++q) {
            const float4 v = __ldg(lo + q);
            o[4 * q] = w0 * v.x + w1 * o[4 * q];
            o[4 * q + 1] = w0 * v.y + w1 * o[4 * q + 1];
            o[4 * q + 2] = w0 * v.z + w1 * o[4 * q + 2];
            o[4 * q + 3] = w0 * v.w + w1 * o[4 * q + 3];
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(a.out + orow * kDh);
#pragma unroll
        for (int q = 0; q < kDh / 8; ++q)
          dst[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                              pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    // Every role has finished, so the flag is final and the same for all
    // threads.  Before tensor memory and shared memory are released, the MMAs
    // each issuing warp started and the loads the producer started complete.
    if (warp >= kMmaWarp && warp < kTmaWarp && lane == 0 && !ptx::mbar_test_wait(drain(warp - kMmaWarp), 0)) {
      ptx::tc_commit(drain(warp - kMmaWarp));
      ptx::mbar_wait_drain(drain(warp - kMmaWarp), 0, ctl->limit_ns);
    }
    if (warp == kTmaWarp && lane == 0) {
      ptx::mbar_wait_drain(qfull, 0, ctl->limit_ns);
      const int issued = ctl->issued;
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

// ---- host side -------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

long token_quantum(const Shape& s) { return (long)kGroups * kBM / s.G; }

cudaError_t launch(const Shape& s, const void* qr, const void* ks, const void* vs, const float* oloc,
                   const float* gate, void* out, int32_t* err, cudaStream_t st, long tok_begin, long tok_end,
                   const Train* tr) {
  if (tok_end < 0) tok_end = s.N;
  if (tok_begin < 0 || tok_begin >= tok_end || tok_end > s.N || tok_begin % token_quantum(s))
    return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  // Q viewed as [N][Hkv][G][64]: a box of 128/G tokens x G heads x 64 dims is one 128-row tile.
  const cuuint64_t qd[4] = {(cuuint64_t)kDh, (cuuint64_t)s.G, (cuuint64_t)s.Hkv, (cuuint64_t)s.N};
  const cuuint64_t qs[3] = {(cuuint64_t)kDh * 2, (cuuint64_t)s.G * kDh * 2, (cuuint64_t)s.Hq * kDh * 2};
  const cuuint32_t qb[4] = {(cuuint32_t)kDh, (cuuint32_t)s.G, 1, (cuuint32_t)(kBM / s.G)};
  const cuuint64_t kd[3] = {(cuuint64_t)kDh, (cuuint64_t)s.Hkv, (cuuint64_t)s.M};
  const cuuint64_t kst[2] = {(cuuint64_t)kDh * 2, (cuuint64_t)s.Hkv * kDh * 2};
  const cuuint32_t kb[3] = {(cuuint32_t)kDh, 1, (cuuint32_t)kBN};
  if (!encode(&tq, qr, 4, qd, qs, qb) || !encode(&tk, ks, 3, kd, kst, kb) || !encode(&tv, vs, 3, kd, kst, kb))
    return cudaErrorInvalidValue;
  const bool train = tr != nullptr && tr->stats != nullptr;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, TcArgs) =
      train ? summary_attn_tc_kernel<true> : summary_attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  TcArgs a;
  a.M = s.M;
  a.G = s.G;
  a.Hq = s.Hq;
  a.rows = tok_end * s.G;
  a.tile_base = (int)(tok_begin * s.G / kBM);
  a.scale_log2 = s.scale_log2;
  a.oloc = oloc;
  a.gate = gate;
  a.out = (__nv_bfloat16*)out;
  a.stats = tr ? tr->stats : nullptr;
  a.dout = tr ? (const __nv_bfloat16*)tr->dout : nullptr;
  a.dgate = tr ? tr->dgate : nullptr;
  a.err = err;
  a.wait_ns = s.wait_ns;
  a.stall = s.stall;
  const long tiles = (a.rows - tok_begin * s.G + kBM - 1) / kBM;
  dim3 grid((unsigned)((tiles + kGroups - 1) / kGroups), s.Hkv);
  kern<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace PACK3D_SA_NS
}  // namespace pack3d
