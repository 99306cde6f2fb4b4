// Memory-bound stages of the PACK3D forward pass on sm_100a:
//   - the grid-to-packed index map and block membership,
//   - axial grid RoPE on Q and K ("Geometry Matters in Packed 3D Attention",
//     Key design 1, equation R(c)),
//   - rotate-before-compress block summaries (Key design 2, equations k~_j^R
//     and v~_j).
// All three stream 16-byte chunks with several loads in flight per thread; the
// RoPE and summary kernels first build the per-axis cos/sin tables in shared
// memory so that no transcendental is evaluated per element.
#include "common.cuh"
#include "internal.h"

namespace pack3d {

// ---- index map ---------------------------------------------------------

__global__ void fill_i32_kernel(int32_t* __restrict__ p, int n, int32_t v) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

// One thread per token: scatter its packed index to its lattice site and to
// its slot in its block.  A repeated site is caught by the exchange returning
// a previous owner.
__global__ void index_kernel(Shape s, const int32_t* __restrict__ coords, int32_t* __restrict__ g2p,
                             int32_t* __restrict__ members, int32_t* err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= s.N) return;
  const int z = coords[3 * i], y = coords[3 * i + 1], x = coords[3 * i + 2];
  if (z < 0 || z >= s.Z || y < 0 || y >= s.H || x < 0 || x >= s.W) {
    set_err(err, PACK3D_DEVERR_COORD_RANGE);
    return;
  }
  const int site = (z * s.H + y) * s.W + x;
  if (atomicExch(&g2p[site], i) != -1) set_err(err, PACK3D_DEVERR_DUPLICATE);
  const int j = ((z / s.bz) * s.nby + y / s.by) * s.nbx + x / s.bx;
  const int t = ((z % s.bz) * s.by + y % s.by) * s.bx + x % s.bx;
  members[j * s.v + t] = i;
}

cudaError_t launch_build_index(const Shape& s, const int32_t* coords, int32_t* g2p,
                               int32_t* members, int32_t* err, cudaStream_t st) {
  // Both maps start at -1 so that a slot no valid token claims (bad input)
  // is recognisable downstream and never dereferenced.
  fill_i32_kernel<<<min((s.N + 255) / 256, 148 * 8), 256, 0, st>>>(g2p, s.N, -1);
  fill_i32_kernel<<<min((s.M * s.v + 255) / 256, 148 * 8), 256, 0, st>>>(members, s.M * s.v, -1);
  index_kernel<<<(s.N + 255) / 256, 256, 0, st>>>(s, coords, g2p, members, err);
  return cudaGetLastError();
}

// ---- axial RoPE ----------------------------------------------------------

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;

// One tensor of the RoPE launch.  Each thread keeps one 16-byte chunk position
// ct of a token row (so the planes it rotates, and their table entries, are
// fixed) and walks the tokens; the threads of a block cover whole contiguous
// token rows, so every load and store is fully coalesced.
template <typename T>
__device__ __forceinline__ void rope_tensor(const Shape& s, const float2* tab, const int32_t* __restrict__ coords,
                                            const T* x, T* y, int heads) {
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int CPR = kDh / NE;  // chunks per head row
  constexpr int NP = NE / 2;     // rotary planes per chunk
  const int CPT = heads * CPR;   // chunks per token
  if (CPT <= (int)blockDim.x) {
    const int tpb = blockDim.x / CPT;
    const int tl = threadIdx.x / CPT, ct = threadIdx.x % CPT;
    if (tl >= tpb) return;
    PlaneLut<NP> lut;
    lut.init(s, (ct % CPR) * NP);
    const int tstride = gridDim.x * tpb;
    for (int t0 = blockIdx.x * tpb + tl; t0 < s.N; t0 += kRopeUnroll * tstride) {
      uint4 u[kRopeUnroll];
      int cz[kRopeUnroll], cy[kRopeUnroll], cx[kRopeUnroll];
#pragma unroll
      for (int k = 0; k < kRopeUnroll; ++k) {
        const int t = t0 + k * tstride;
        if (t < s.N) {
          u[k] = *reinterpret_cast<const uint4*>(x + ((size_t)t * CPT + ct) * NE);
          // Clamped so that a bad coordinate (reported by the index map) cannot
          // index outside the tables.
          cz[k] = min(max(__ldg(coords + 3 * t), 0), s.Z - 1);
          cy[k] = min(max(__ldg(coords + 3 * t + 1), 0), s.H - 1);
          cx[k] = min(max(__ldg(coords + 3 * t + 2), 0), s.W - 1);
        }
      }
#pragma unroll
      for (int k = 0; k < kRopeUnroll; ++k) {
        const int t = t0 + k * tstride;
        if (t >= s.N) continue;
        float f[NE];
        chunk_to_float(u[k], f, T());
        lut.rotate(f, tab, cz[k], cy[k], cx[k]);
        stg16(y + ((size_t)t * CPT + ct) * NE, float_to_chunk(f, T()));
      }
    }
  } else {
    // Rows wider than a block: plain strided walk over all chunks.
    const unsigned total = (unsigned)s.N * CPT;
    for (unsigned c = blockIdx.x * blockDim.x + threadIdx.x; c < total; c += gridDim.x * blockDim.x) {
      const unsigned t = c / CPT;
      PlaneLut<NP> lut;
      lut.init(s, (int)(c % CPR) * NP);
      float f[NE];
      chunk_to_float(*reinterpret_cast<const uint4*>(x + (size_t)c * NE), f, T());
      lut.rotate(f, tab, min(max(__ldg(coords + 3 * t), 0), s.Z - 1), min(max(__ldg(coords + 3 * t + 1), 0), s.H - 1),
                 min(max(__ldg(coords + 3 * t + 2), 0), s.W - 1));
      stg16(y + (size_t)c * NE, float_to_chunk(f, T()));
    }
  }
}

// Rotates up to two tensors (e.g. Q and K_loc) in one launch; y may alias x
// (each chunk is read and written by the same thread).
template <typename T>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(Shape s, const int32_t* __restrict__ coords,
                                                            const T* x0, T* y0, int h0,
                                                            const T* x1, T* y1, int h1) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  rope_tensor(s, tab, coords, x0, y0, h0);
  if (x1 != nullptr) rope_tensor(s, tab, coords, x1, y1, h1);
}

static int rope_grid(const Shape& s, int heads, int chunk_elems) {
  long chunks = (long)s.N * heads * (kDh / chunk_elems);
  long want = (chunks + kRopeThreads * kRopeUnroll - 1) / (kRopeThreads * kRopeUnroll);
  return (int)max(1L, min(want, 148L * 4));
}

template <typename T>
static cudaError_t rope_t(const Shape& s, const int32_t* coords, const void* x0, void* y0, int h0,
                          const void* x1, void* y1, int h1, cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  cudaError_t e = cudaFuncSetAttribute(rope_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int grid = rope_grid(s, h0 + (x1 ? h1 : 0), Elem<T>::kPerChunk);
  rope_kernel<T><<<grid, kRopeThreads, smem, st>>>(
      s, coords, (const T*)x0, (T*)y0, h0, (const T*)x1, (T*)y1, h1);
  return cudaGetLastError();
}

cudaError_t launch_rope(const Shape& s, int dtype, const int32_t* coords, const void* x0, void* y0,
                        int h0, const void* x1, void* y1, int h1, cudaStream_t st) {
  if (dtype == PACK3D_BF16) return rope_t<__nv_bfloat16>(s, coords, x0, y0, h0, x1, y1, h1, st);
  return rope_t<float>(s, coords, x0, y0, h0, x1, y1, h1, st);
}

// ---- rotate-before-compress summaries ----------------------------------

constexpr int kSumThreads = 256;

// Fast path (block volume <= U): a unit of U = 2 * (kDh / NE) lanes owns one
// (block j, kv head g).  Lane t first holds member t: it loads that member's
// score once, and the unit's softmax weights come from shuffle reductions.
// Then lane l accumulates one 16-byte chunk of k~ (lanes 0 .. U/2-1, rotating
// each member row before pooling) or of v~ (the other half) over the members,
// with every member row read as a whole 128-byte line by U/2 lanes and four
// rows in flight per lane.  V > 0 fixes the block volume at compile time;
// V = 0 reads it from the shape.
template <typename T, int V>
__global__ void __launch_bounds__(kSumThreads) summaries_kernel(
    Shape s, const int32_t* __restrict__ members, const T* __restrict__ kc,
    const T* __restrict__ vc, const float* __restrict__ scores, T* __restrict__ ks,
    T* __restrict__ vs) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int LPT = kDh / NE;          // lanes per tensor row
  constexpr int U = 2 * LPT;             // lanes per unit (16 bf16, 32 float)
  constexpr int NP = NE / 2;
  constexpr int VMAX = V > 0 ? V : U;
  const int vol = V > 0 ? V : s.v;
  const int lu = threadIdx.x % U;
  const int is_v = lu >= LPT;
  const int part = lu % LPT;
  const unsigned umask = U == 32 ? 0xffffffffu : (0xffffu << (threadIdx.x & 16));
  PlaneLut<NP> lut;
  lut.init(s, part * NP);
  const long units = (long)s.M * s.Hkv;
  const long ustride = (long)gridDim.x * (kSumThreads / U);
  const T* src = is_v ? vc : kc;
  for (long u = (long)blockIdx.x * (kSumThreads / U) + threadIdx.x / U; u < units; u += ustride) {
    const int g = (int)(u % s.Hkv);
    const int j = (int)(u / s.Hkv);
    // a_{j,t}: softmax over the block's members of their scores for kv head g.
    const int m = lu < vol ? __ldg(members + (size_t)j * vol + lu) : -1;
    const float sc = m >= 0 ? __ldg(scores + (size_t)m * s.Hkv + g) : -INFINITY;
    float mx = sc;
#pragma unroll
    for (int o = U / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(umask, mx, o, U));
    const float e = m >= 0 ? expf(sc - mx) : 0.f;
    float den = e;
#pragma unroll
    for (int o = U / 2; o > 0; o >>= 1) den += __shfl_xor_sync(umask, den, o, U);
    const float a = den > 0.f ? e / den : 0.f;
    const int jx = j % s.nbx, jy = (j / s.nbx) % s.nby, jz = j / (s.nbx * s.nby);
    float acc[NE];
#pragma unroll
    for (int k = 0; k < NE; ++k) acc[k] = 0.f;
    // Members in batches of kBatch rows in flight per lane.
    constexpr int kBatch = 4;
#pragma unroll 1
    for (int t0 = 0; t0 < VMAX; t0 += kBatch) {
      uint4 rowc[kBatch];
      int mts[kBatch];
      float ats[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int t = t0 + b;
        mts[b] = __shfl_sync(umask, m, t & (U - 1), U);
        ats[b] = __shfl_sync(umask, a, t & (U - 1), U);
        if (t < vol && mts[b] >= 0) rowc[b] = ldg16(src + ((size_t)mts[b] * s.Hkv + g) * kDh + part * NE);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int t = t0 + b;
        if (t >= vol || mts[b] < 0) continue;
        float f[NE];
        chunk_to_float(rowc[b], f, T());
        if (!is_v && !s.center) {
          const int tz = t / (s.by * s.bx), ty = (t / s.bx) % s.by, tx = t % s.bx;
          lut.rotate(f, tab, jz * s.bz + tz, jy * s.by + ty, jx * s.bx + tx);
        }
#pragma unroll
        for (int k = 0; k < NE; ++k) acc[k] = fmaf(ats[b], f[k], acc[k]);
      }
    }
    if (!is_v && s.center)
      rotate_at<NP>(acc, s, part * NP, s.origin[0] + jz * s.bz + 0.5 * (s.bz - 1),
                    s.origin[1] + jy * s.by + 0.5 * (s.by - 1), s.origin[2] + jx * s.bx + 0.5 * (s.bx - 1));
    T* dst = is_v ? vs : ks;
    stg16(dst + ((size_t)j * s.Hkv + g) * kDh + part * NE, float_to_chunk(acc, T()));
  }
}

// A unit is (block j, kv head g, K or V); kDh/NE lanes share a unit, each lane
// owning one 16-byte chunk of the 64 dims.  Member t of block j sits at the
// t-th raster site of the block, so its coordinates follow from (j, t).
template <typename T>
__global__ void __launch_bounds__(kSumThreads) summaries_generic_kernel(
    Shape s, const int32_t* __restrict__ members, const T* __restrict__ kc,
    const T* __restrict__ vc, const float* __restrict__ scores, T* __restrict__ ks,
    T* __restrict__ vs) {
  extern __shared__ float2 tab[];
  build_rope_table(tab, s);
  __syncthreads();
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int LPU = kDh / NE;
  const int units_per_cta = kSumThreads / LPU;
  const long units = (long)s.M * s.Hkv * 2;
  const int part = threadIdx.x % LPU;
  for (long ub = (long)blockIdx.x * units_per_cta; ub < units; ub += (long)gridDim.x * units_per_cta) {
    const long u = ub + threadIdx.x / LPU;
    if (u >= units) continue;
    const int is_v = (int)(u & 1);
    const long jg = u >> 1;
    const int g = (int)(jg % s.Hkv);
    const int j = (int)(jg / s.Hkv);
    const int32_t* mem = members + (size_t)j * s.v;
    const int jx = j % s.nbx, jy = (j / s.nbx) % s.nby, jz = j / (s.nbx * s.nby);
    // a_{j,u}: softmax of the block's scores for kv head g.
    // Members left at -1 (only possible for coordinates that are not a
    // bijection, which the index map reports) are skipped.
    float smax = -INFINITY;
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m >= 0) smax = fmaxf(smax, __ldg(scores + (size_t)m * s.Hkv + g));
    }
    float den = 0.f;
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m >= 0) den += expf(__ldg(scores + (size_t)m * s.Hkv + g) - smax);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const T* src = is_v ? vc : kc;
    float acc[NE];
#pragma unroll
    for (int k = 0; k < NE; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int t = 0; t < s.v; ++t) {
      const int m = __ldg(mem + t);
      if (m < 0) continue;
      const float a = expf(__ldg(scores + (size_t)m * s.Hkv + g) - smax) * inv;
      const uint4 c = ldg16(src + ((size_t)m * s.Hkv + g) * kDh + part * NE);
      float f[NE];
      chunk_to_float(c, f, T());
      if (!is_v && !s.center) {
        const int tz = t / (s.by * s.bx), ty = (t / s.bx) % s.by, tx = t % s.bx;
        PlaneLut<NE / 2> lut;
        lut.init(s, part * (NE / 2));
        lut.rotate(f, tab, jz * s.bz + tz, jy * s.by + ty, jx * s.bx + tx);
      }
#pragma unroll
      for (int k = 0; k < NE; ++k) acc[k] = fmaf(a, f[k], acc[k]);
    }
    if (!is_v && s.center)
      rotate_at<NE / 2>(acc, s, part * (NE / 2), s.origin[0] + jz * s.bz + 0.5 * (s.bz - 1),
                        s.origin[1] + jy * s.by + 0.5 * (s.by - 1), s.origin[2] + jx * s.bx + 0.5 * (s.bx - 1));
    T* dst = is_v ? vs : ks;
    stg16(dst + ((size_t)j * s.Hkv + g) * kDh + part * NE, float_to_chunk(acc, T()));
  }
}

// Warp-per-block path (block volume 16).  One warp owns block j for every kv
// head and both tensors.  Lane l owns chunk slot c of a member's head rows
// (head c / CPR, 16-byte part c % CPR) in BOTH K_cmp and V_cmp, so K and V
// lanes never diverge; when a member has fewer than 32 slots the warp covers
// MPI members per load and the lanes' partial sums are combined at the end.
//
// The rotation is split with R(c_base + d) = R(c_base) R(d) (each plane is a
// 2-D rotation by omega * coordinate, so angles add): member t, at in-block
// offset d_t of the block's first site c_base, is rotated by R(d_t) from a
// small per-CTA table of the 16 offsets x 32 planes, and the pooled key is
// rotated once by R(c_base):  k~_j = R(c_base) sum_t a_t R(d_t) k_t, the same
// sum as sum_t a_t R(c_t) k_t.  Both are evaluated directly (angle reduced in
// double, float sincos), so the kernel needs no whole-volume cos/sin table.
constexpr int kSumWarpThreads = 256;

template <typename T, int HKV>
__global__ void __launch_bounds__(kSumWarpThreads) summaries_warp_kernel(
    Shape s, const int32_t* __restrict__ members, const T* __restrict__ kc,
    const T* __restrict__ vc, const float* __restrict__ scores, T* __restrict__ ks,
    T* __restrict__ vs) {
  constexpr int V = 16;
  static_assert(kMaxPairs == 32, "one rotary plane per lane");
  __shared__ float2 dtab[V][kMaxPairs];   // cos/sin of plane p at member t's in-block offset
  const int lane = threadIdx.x & 31;
  // Lane p holds rotary plane p's axis and frequency.
  const int my_axis = lane < s.npairs ? s.pair_axis[lane] : 3;
  const double my_omega = lane < s.npairs ? s.omega[lane] : 0.0;
  for (int t = threadIdx.x >> 5; t < V; t += kSumWarpThreads / 32) {
    const int d = my_axis == 0 ? t / (s.by * s.bx) : (my_axis == 1 ? (t / s.bx) % s.by : t % s.bx);
    // (Summary-centre variant: members are pooled unrotated.)
    dtab[t][lane] = my_axis < 3 && !s.center ? rope_cos_sin(my_omega * (double)d) : make_float2(1.f, 0.f);
  }
  __syncthreads();
  constexpr int NE = Elem<T>::kPerChunk;
  constexpr int NP = NE / 2;
  constexpr int CPR = kDh / NE;                   // chunks per head row
  constexpr int LPM = HKV * CPR;                  // chunk slots per member and tensor
  constexpr int SPL = LPM >= 32 ? LPM / 32 : 1;   // slots per lane
  constexpr int MPI = LPM >= 32 ? 1 : 32 / LPM;   // members per load instruction
  constexpr int PPL = (V * HKV + 31) / 32;        // (member, head) score pairs per lane
#ifndef PACK3D_SUM_LOADS
#define PACK3D_SUM_LOADS 8
#endif
  // Members per batch: PACK3D_SUM_LOADS K and V chunk pairs in flight per lane.
  constexpr int B = (PACK3D_SUM_LOADS * MPI / SPL) < V ? (PACK3D_SUM_LOADS * MPI / SPL) : V;
  static_assert(V % B == 0 && B % MPI == 0, "member batches");
  const int sub = MPI > 1 ? lane / LPM : 0;
  int head[SPL], part[SPL];
#pragma unroll
  for (int i = 0; i < SPL; ++i) {
    const int c = (lane % LPM) + 32 * i;
    head[i] = c / CPR;
    part[i] = c % CPR;
  }
  const int nwarps = gridDim.x * (kSumWarpThreads / 32);
  int j = blockIdx.x * (kSumWarpThreads / 32) + (threadIdx.x >> 5);
  // Block-grid position of block j, stepped by nwarps blocks per iteration.
  int jx = j % s.nbx, jy = (j / s.nbx) % s.nby, jz = j / (s.nbx * s.nby);
  const int sx = nwarps % s.nbx, sy = (nwarps / s.nbx) % s.nby, sz = nwarps / (s.nbx * s.nby);
  // Member t of block j is held by lanes t and t + 16; the next block's
  // indices are requested while this block is pooled.
  int m_next = j < s.M ? __ldg(members + (size_t)j * V + (lane & 15)) : -1;
  for (; j < s.M; j += nwarps) {
    const int m_l = m_next;
    if (j + nwarps < s.M) m_next = __ldg(members + (size_t)(j + nwarps) * V + (lane & 15));
    // Scores: pair p = lane + 32 i is (member p % 16, head p / 16).
    float sc[PPL];
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
      const int p = lane + 32 * i, h = p >> 4;
      const int mt = __shfl_sync(0xffffffffu, m_l, p & 15);
      sc[i] = (h < HKV && mt >= 0) ? __ldg(scores + (size_t)mt * HKV + h) : -INFINITY;
    }
    float ak[SPL][NE], av[SPL][NE];
#pragma unroll
    for (int i = 0; i < SPL; ++i)
#pragma unroll
      for (int k = 0; k < NE; ++k) ak[i][k] = av[i][k] = 0.f;
    float wa[PPL];
#pragma unroll 1
    for (int t0 = 0; t0 < V; t0 += B) {
      uint4 rk[B / MPI][SPL], rv[B / MPI][SPL];
      int mts[B / MPI];
#pragma unroll
      for (int b = 0; b < B / MPI; ++b) {
        mts[b] = __shfl_sync(0xffffffffu, m_l, t0 + b * MPI + sub);
#pragma unroll
        for (int i = 0; i < SPL; ++i) {
          // A member slot left at -1 (coordinates that are not a bijection,
          // reported by the index map) contributes zero rows with zero weight.
          const size_t off = ((size_t)max(mts[b], 0) * HKV + head[i]) * kDh + part[i] * NE;
          rk[b][i] = mts[b] >= 0 ? ldg16(kc + off) : make_uint4(0u, 0u, 0u, 0u);
          rv[b][i] = mts[b] >= 0 ? ldg16(vc + off) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (t0 == 0) {
        // a_{j,t} = softmax over the block's members of their scores (per
        // head): the 16 pairs of one head sit in one half-warp of a register.
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
          float mx = sc[i];
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float e = sc[i] == -INFINITY ? 0.f : expf(sc[i] - mx);
          float den = e;
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
          wa[i] = den > 0.f ? e / den : 0.f;
        }
      }
      // Weights of (member t, head[i]) for the whole batch first (register
      // head/2, lane (head%2)*16 + t), so the pooling below has no shuffle or
      // branch between members.
      float wt[B / MPI][SPL];
#pragma unroll
      for (int b = 0; b < B / MPI; ++b)
#pragma unroll
        for (int i = 0; i < SPL; ++i) {
          float w = 0.f;
#pragma unroll
          for (int r = 0; r < PPL; ++r) {
            const float x = __shfl_sync(0xffffffffu, wa[r], ((head[i] & 1) << 4) + t0 + b * MPI + sub);
            if (r == head[i] >> 1) w = x;
          }
          wt[b][i] = w;
        }
#pragma unroll
      for (int b = 0; b < B / MPI; ++b) {
        const int t = t0 + b * MPI + sub;
#pragma unroll
        for (int i = 0; i < SPL; ++i) {
          const float w = wt[b][i];
          float fk[NE], fv[NE];
          chunk_to_float(rk[b][i], fk, T());
          chunk_to_float(rv[b][i], fv, T());
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            const float2 cs = dtab[t][part[i] * NP + k];
            const float x0 = fk[2 * k], x1 = fk[2 * k + 1];
            ak[i][2 * k] = fmaf(w, x0 * cs.x - x1 * cs.y, ak[i][2 * k]);
            ak[i][2 * k + 1] = fmaf(w, x0 * cs.y + x1 * cs.x, ak[i][2 * k + 1]);
          }
#pragma unroll
          for (int k = 0; k < NE; ++k) av[i][k] = fmaf(w, fv[k], av[i][k]);
        }
      }
    }
    // Lanes that covered different members of the same slot combine.
#pragma unroll
    for (int o = LPM; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < SPL; ++i)
#pragma unroll
        for (int k = 0; k < NE; ++k) {
          ak[i][k] += __shfl_xor_sync(0xffffffffu, ak[i][k], o);
          av[i][k] += __shfl_xor_sync(0xffffffffu, av[i][k], o);
        }
    // R(c_base): lane p evaluates plane p at the block's first site, and every
    // lane takes the pairs of its own planes by shuffle.
    // (Summary-centre variant: at the block's geometric centre instead.)
    const double half = s.center ? 0.5 : 0.0;
    const double cpos = (my_axis < 3 ? s.origin[my_axis] : 0) +
                        (my_axis == 0 ? jz * s.bz + half * (s.bz - 1)
                                      : (my_axis == 1 ? jy * s.by + half * (s.by - 1) : jx * s.bx + half * (s.bx - 1)));
    const float2 cb = my_axis < 3 ? rope_cos_sin(my_omega * cpos) : make_float2(1.f, 0.f);
#pragma unroll
    for (int i = 0; i < SPL; ++i)
#pragma unroll
      for (int k = 0; k < NP; ++k) {
        const float c = __shfl_sync(0xffffffffu, cb.x, part[i] * NP + k);
        const float sn = __shfl_sync(0xffffffffu, cb.y, part[i] * NP + k);
        const float x0 = ak[i][2 * k], x1 = ak[i][2 * k + 1];
        ak[i][2 * k] = x0 * c - x1 * sn;
        ak[i][2 * k + 1] = x0 * sn + x1 * c;
      }
    if (sub == 0) {
#pragma unroll
      for (int i = 0; i < SPL; ++i) {
        const size_t off = ((size_t)j * HKV + head[i]) * kDh + part[i] * NE;
        stg16(ks + off, float_to_chunk(ak[i], T()));
        stg16(vs + off, float_to_chunk(av[i], T()));
      }
    }
    jx += sx;
    if (jx >= s.nbx) { jx -= s.nbx; ++jy; }
    jy += sy;
    if (jy >= s.nby) { jy -= s.nby; ++jz; }
    jz += sz;
  }
}

template <typename T>
static cudaError_t summaries_t(const Shape& s, const int32_t* members, const void* kc, const void* vc,
                               const float* scores, void* ks, void* vs, cudaStream_t st) {
  const size_t smem = (size_t)s.tab_entries * sizeof(float2);
  const int U = 2 * (kDh / Elem<T>::kPerChunk);
  if (s.v == 16 && (s.Hkv == 1 || s.Hkv == 2 || s.Hkv == 4 || s.Hkv == 8)) {
    auto kern = s.Hkv == 1   ? summaries_warp_kernel<T, 1>
                : s.Hkv == 2 ? summaries_warp_kernel<T, 2>
                : s.Hkv == 4 ? summaries_warp_kernel<T, 4>
                             : summaries_warp_kernel<T, 8>;
    // One persistent wave: every SM holds as many CTAs as fit, each warp walks blocks.
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSumWarpThreads, 0);
    if (e != cudaSuccess) return e;
    const long per_cta = kSumWarpThreads / 32;
    const int grid = (int)max(1L, min((s.M + per_cta - 1) / per_cta, (long)sms * max(per_sm, 1)));
    kern<<<grid, kSumWarpThreads, 0, st>>>(s, members, (const T*)kc, (const T*)vc, scores, (T*)ks, (T*)vs);
    return cudaGetLastError();
  }
  if (s.v <= U) {
    auto kern = summaries_kernel<T, 0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long units = (long)s.M * s.Hkv;
    const long per_cta = kSumThreads / U;
    const int grid = (int)max(1L, min((units + per_cta - 1) / per_cta, 148L * 8));
    kern<<<grid, kSumThreads, smem, st>>>(s, members, (const T*)kc, (const T*)vc, scores, (T*)ks, (T*)vs);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(summaries_generic_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int lpu = kDh / Elem<T>::kPerChunk;
  const long units = (long)s.M * s.Hkv * 2;
  const long per_cta = kSumThreads / lpu;
  const int grid = (int)max(1L, min((units + per_cta - 1) / per_cta, 148L * 8));
  summaries_generic_kernel<T><<<grid, kSumThreads, smem, st>>>(s, members, (const T*)kc, (const T*)vc, scores,
                                                                (T*)ks, (T*)vs);
  return cudaGetLastError();
}

cudaError_t launch_summaries(const Shape& s, int dtype, const int32_t* members, const void* kc,
                             const void* vc, const float* scores, void* ks, void* vs,
                             cudaStream_t st) {
  if (dtype == PACK3D_BF16)
    return summaries_t<__nv_bfloat16>(s, members, kc, vc, scores, ks, vs, st);
  return summaries_t<float>(s, members, kc, vc, scores, ks, vs, st);
}

}  // namespace pack3d
