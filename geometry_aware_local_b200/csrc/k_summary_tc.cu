// Query x summary attention with the tokenwise gate on sm_100a tensor cores.
//
// "Geometry Matters in Packed 3D Attention", Key design 3: every query attends
// to all M block summaries with its own softmax, streamed with an online
// softmax so that no [N, M] score tensor exists; the overall framework's
// tokenwise two-way softmax gate mixes the result with the local branch.
//
// Design (one CTA = two 128-row query tiles of one kv head, sharing every
// summary tile):
//   * rows are (token, q head) pairs of one kv group, G = Hq/Hkv heads per
//     token, so a 128-row tile is 128/G tokens x G heads and one k~/v~ tile
//     serves all of them;
//   * warp 9 streams k~ and v~ tiles (128 summaries x 64 dims, bf16, 128-byte
//     swizzle) through a 4-stage TMA ring; Q tiles are loaded once;
//   * warp 8 issues tcgen05.mma: S = Q k~^T into tensor memory (128 x 128
//     float) and O += P v~ with P read back from tensor memory (bf16);
//   * warps 0-3 and 4-7 are two softmax warpgroups, one per query tile; each
//     thread owns one row (one TMEM lane).  While one group turns S into P,
//     the tensor core works on the other group's tiles (ping-pong).
//   * O is rescaled lazily: the running maximum used for P only moves when a
//     row's new maximum exceeds it by more than 2^8, so most tiles skip the
//     rescale.  P values stay below 256, well inside bf16 range.
// Tensor memory (512 columns): group w owns columns [256w, 256w+256): S at +0
// (128 cols), P at +128 (64 cols of packed bf16 pairs), O at +192 (64 cols).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace pack3d {
namespace {

constexpr int kBM = 128;          // rows per query tile
constexpr int kBN = 128;          // summaries per tile
constexpr int kStages = 4;
constexpr int kThreads = 320;     // 8 softmax warps + MMA warp + TMA warp
constexpr int kTileBytes = kBM * kDh * 2;  // 16 KiB bf16 tile
constexpr int kQOff = 0;                   // two Q tiles
constexpr int kKVOff = 2 * kTileBytes;     // stage s: k~ at +0, v~ at +16 KiB
constexpr int kBarOff = kKVOff + kStages * 2 * kTileBytes;
constexpr int kNumBars = 2 * kStages + 1 + 2 + 2 + 2 + 2;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // + slack for 1 KiB alignment
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kBM, kBN, false);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBM, kDh, true);

struct TcArgs {
  int M;             // summaries
  int G;             // q heads per kv head
  int Hq;
  long rows;         // N * G rows per kv head
  float scale_log2;  // softmax scale * log2(e)
  const float* oloc;
  const float* gate;
  __nv_bfloat16* out;
  int32_t* err;
};

__global__ void __launch_bounds__(kThreads, 1)
summary_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int tile0 = blockIdx.x * 2;
  const int T = (a.M + kBN - 1) / kBN;

  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + kBarOff;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  const uint32_t qfull = bar0 + 8 * (2 * kStages);
  auto s_full = [&](int w) { return bar0 + 8 * (2 * kStages + 1 + w); };
  auto s_free = [&](int w) { return bar0 + 8 * (2 * kStages + 3 + w); };
  auto p_full = [&](int w) { return bar0 + 8 * (2 * kStages + 5 + w); };
  auto o_final = [&](int w) { return bar0 + 8 * (2 * kStages + 7 + w); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    ptx::mbar_init(qfull, 1);
    for (int w = 0; w < 2; ++w) {
      ptx::mbar_init(s_full(w), 1);
      ptx::mbar_init(s_free(w), kBM);
      ptx::mbar_init(p_full(w), kBM);
      ptx::mbar_init(o_final(w), 1);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 8) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::tma_prefetch(&tmQ);
      ptx::tma_prefetch(&tmK);
      ptx::tma_prefetch(&tmV);
      const int tok_per_tile = kBM / a.G;
      ptx::mbar_expect_tx(qfull, 2 * kTileBytes);
      ptx::tma_load_4d(sbase + kQOff, &tmQ, 0, 0, g, tile0 * tok_per_tile, qfull);
      ptx::tma_load_4d(sbase + kQOff + kTileBytes, &tmQ, 0, 0, g, (tile0 + 1) * tok_per_tile, qfull);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !ptx::mbar_wait(empty(st), ((j / kStages) - 1) & 1, abort_flag)) break;
        const uint32_t kdst = sbase + kKVOff + st * 2 * kTileBytes;
        ptx::mbar_expect_tx(full(st), 2 * kTileBytes);
        ptx::tma_load_3d(kdst, &tmK, 0, g, j * kBN, full(st));
        ptx::tma_load_3d(kdst + kTileBytes, &tmV, 0, g, j * kBN, full(st));
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's shared memory is released.
        for (int j = max(0, issued - kStages); j < issued; ++j)
          ptx::mbar_wait(full(j % kStages), (j / kStages) & 1, abort_flag);
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t qaddr[2] = {sbase + kQOff, sbase + kQOff + kTileBytes};
      auto issue_s = [&](int w, int st) {
        const uint32_t kaddr = sbase + kKVOff + st * 2 * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(qaddr[w] + kk * 32, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(kaddr + kk * 32, 16, 1024);
          ptx::mma_ss(tmem + w * 256, ad, bd, kIdescS, kk > 0);
        }
        ptx::tc_commit(s_full(w));
      };
      auto issue_pv = [&](int w, int st, bool first) {
        const uint32_t vaddr = sbase + kKVOff + st * 2 * kTileBytes + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = ptx::smem_desc_sw128(vaddr + kk * 2048, 8192, 1024);
          ptx::mma_ts(tmem + w * 256 + 192, tmem + w * 256 + 128 + kk * 8, bd, kIdescPV,
                      (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = ptx::mbar_wait(qfull, 0, abort_flag) && ptx::mbar_wait(full(0), 0, abort_flag);
      if (ok) {
        ptx::tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % kStages;
        for (int w = 0; w < 2 && ok; ++w) {
          if (!(ok = ptx::mbar_wait(p_full(w), j & 1, abort_flag))) break;
          ptx::tc_fence_after();
          issue_pv(w, st, j == 0);
          if (j == T - 1) ptx::tc_commit(o_final(w));
          if (w == 1) ptx::tc_commit(empty(st));
          if (j + 1 < T) {
            const int st1 = (j + 1) % kStages;
            if (!(ok = ptx::mbar_wait(full(st1), ((j + 1) / kStages) & 1, abort_flag))) break;
            if (!(ok = ptx::mbar_wait(s_free(w), j & 1, abort_flag))) break;
            ptx::tc_fence_after();
            issue_s(w, st1);
          }
        }
      }
      if (!ok) {
        // Drain whatever was issued before tensor memory is released.
        ptx::tc_commit(o_final(0));
        ptx::mbar_wait(o_final(0), 0, abort_flag);
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax warpgroups ----------------
    const int w = warp >> 2;
    const int lane_base = (warp & 3) * 32;
    const uint32_t trow = tmem + ((uint32_t)lane_base << 16) + w * 256;
    const uint32_t tS = trow, tP = trow + 128, tO = trow + 192;
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!(ok = __all_sync(0xffffffffu, ptx::mbar_wait(s_full(w), j & 1, abort_flag)))) break;
      ptx::tc_fence_after();
      uint32_t sv[kBN];
#pragma unroll
      for (int q = 0; q < kBN / 32; ++q) ptx::tmem_ld32(tS + 32 * q, sv + 32 * q);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(s_free(w));
      if ((j + 1) * kBN > a.M) {
        const int lim = a.M - j * kBN;
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (k >= lim) sv[k] = __float_as_uint(-INFINITY);
      }
      float mx = __uint_as_float(sv[0]);
#pragma unroll
      for (int k = 1; k < kBN; ++k) mx = fmaxf(mx, __uint_as_float(sv[k]));
      const float mxs = mx * c;
      // Lazy rescale: the maximum used for P moves only when this tile's row
      // maximum exceeds it by more than the threshold.
      float f = 1.f;
      if (j == 0) {
        m_used = mxs;
      } else if (mxs > m_used + kRescaleThreshold) {
        f = ptx::ex2(m_used - mxs);
        m_used = mxs;
      }
      const float nm = -m_used;
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < kBN / 32; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(sv[32 * q + 2 * k]), c, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(sv[32 * q + 2 * k + 1]), c, nm));
          rs += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        ptx::tmem_st16(tP + 16 * q, pk);
      }
      if (__any_sync(0xffffffffu, f != 1.f)) {
        // O holds P_0..P_{j-1} v~ relative to the old maximum.  PV_{j-1}
        // completed before S_j was committed, and PV_j waits for p_full, so O
        // is stable here.
        uint32_t r[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          ptx::tmem_ld32(tO + 32 * q, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
          ptx::tmem_st32(tO + 32 * q, r);
        }
      }
      l = l * f + rs;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(p_full(w));
    }
    if (ok && __all_sync(0xffffffffu, ptx::mbar_wait(o_final(w), 0, abort_flag))) {
      ptx::tc_fence_after();
      float o[kDh];
      {
        uint32_t r[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          ptx::tmem_ld32(tO + 32 * q, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[32 * q + k] = __uint_as_float(r[k]);
        }
      }
      const long grow = (long)(tile0 + w) * kBM + lane_base + lane;
      if (grow < a.rows) {
        const long tok = grow / a.G;
        const int h = g * a.G + (int)(grow % a.G);
        const size_t orow = (size_t)tok * a.Hq + h;
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < kDh; ++e) o[e] *= inv;
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
  if (warp == 8) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(a.err, PACK3D_DEVERR_TIMEOUT);
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

cudaError_t launch_summary_attn_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                   const float* oloc, const float* gate, void* out, int32_t* err,
                                   cudaStream_t st) {
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
  cudaError_t e = cudaFuncSetAttribute(summary_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  TcArgs a;
  a.M = s.M;
  a.G = s.G;
  a.Hq = s.Hq;
  a.rows = (long)s.N * s.G;
  a.scale_log2 = s.scale_log2;
  a.oloc = oloc;
  a.gate = gate;
  a.out = (__nv_bfloat16*)out;
  a.err = err;
  const long tiles = (a.rows + kBM - 1) / kBM;
  dim3 grid((unsigned)((tiles + 1) / 2), s.Hkv);
  summary_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace pack3d
