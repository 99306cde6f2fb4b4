// C ABI of the PACK3D forward pass (see pack3d.h): host-side validation,
// workspace carving and stream-ordered launches.  No entry point allocates
// device memory, frees or synchronises except pack3d_check_status;
// pack3d_forward creates one side stream and two events per device on its
// first call there (kept until the process exits).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <new>

#include "common.cuh"
#include "internal.h"
#include "pack3d.h"

namespace pack3d {

Shape make_shape(const pack3d_config& c) {
  Shape s;
  memset(&s, 0, sizeof(s));
  s.Z = c.Z; s.H = c.H; s.W = c.W;
  s.N = c.Z * c.H * c.W;
  s.Hq = c.Hq; s.Hkv = c.Hkv; s.G = c.Hq / c.Hkv;
  s.bz = c.bz; s.by = c.by; s.bx = c.bx;
  s.v = c.bz * c.by * c.bx;
  s.M = s.N / s.v;
  s.nbz = c.Z / c.bz; s.nby = c.H / c.by; s.nbx = c.W / c.bx;
  s.rz = c.rz; s.ry = c.ry; s.rx = c.rx;
  s.mz = c.m_z; s.my = c.m_y; s.mx = c.m_x;
  s.tab_entries = c.Z * c.m_z + c.H * c.m_y + c.W * c.m_x;
  s.scale = c.softmax_scale;
  s.scale_log2 = (float)((double)c.softmax_scale * 1.4426950408889634);
  s.center = (c.flags & PACK3D_FLAG_SUMMARY_CENTER) ? 1 : 0;
  s.wait_ns = c.wait_limit_us > 0 ? (unsigned long long)c.wait_limit_us * 1000ull : 2000000000ull;
  s.stall = (c.flags & PACK3D_FLAG_DIAG_STALL) ? 1 : 0;
  s.sa_build = (c.flags & PACK3D_FLAG_SUMMARY_ONE_TILE) ? 1 : ((c.flags & PACK3D_FLAG_SUMMARY_TWO_TILE) ? 2 : 0);
  for (int a = 0; a < 3; ++a) s.origin[a] = c.origin[a];
  const int m[3] = {c.m_z, c.m_y, c.m_x};
  const int ext[3] = {c.Z, c.H, c.W};
  int p = 0, off = 0;
  for (int a = 0; a < 3; ++a)
    for (int r = 0; r < m[a]; ++r) {
      // The coordinate scale of the axis folds into the plane's frequency.
      s.omega[p] = pow(c.rope_base, -(double)r / (double)m[a]) * c.coord_scale[a];
      s.pair_axis[p] = a;
      s.pair_off[p] = off;
      off += ext[a];
      ++p;
    }
  s.npairs = p;
  for (; p < kMaxPairs; ++p) s.pair_axis[p] = 3;
  return s;
}

ForwardWs carve_forward(const pack3d_config& c, uintptr_t base) {
  const size_t N = (size_t)c.Z * c.H * c.W;
  const size_t v = (size_t)c.bz * c.by * c.bx;
  const size_t M = N / v;
  const size_t eb = c.dtype == PACK3D_BF16 ? 2 : 4;
  const size_t A = 1024;
  auto up = [&](size_t x) { return (x + A - 1) / A * A; };
  ForwardWs w;
  size_t off = 0;
  w.g2p = reinterpret_cast<int32_t*>(base + off);      off = up(off + N * 4);
  w.members = reinterpret_cast<int32_t*>(base + off);  off = up(off + M * v * 4);
  w.q_rot = reinterpret_cast<void*>(base + off);       off = up(off + N * c.Hq * c.d_h * eb);
  w.k_rot = reinterpret_cast<void*>(base + off);       off = up(off + N * c.Hkv * c.d_h * eb);
  w.k_sum = reinterpret_cast<void*>(base + off);       off = up(off + M * c.Hkv * c.d_h * eb);
  w.v_sum = reinterpret_cast<void*>(base + off);       off = up(off + M * c.Hkv * c.d_h * eb);
  w.o_loc = reinterpret_cast<float*>(base + off);      off = up(off + N * c.Hq * c.d_h * 4);
  w.bytes = off;
  return w;
}

namespace {

// The side stream RoPE runs on inside pack3d_forward: one non-blocking stream
// and two events per device, made on the device's first uncaptured call.  The
// mutex is held from the fork to the join, so calls from several host threads
// never interleave their records and waits on the shared events (their side
// work is serialised on the one side stream).
constexpr int kMaxForkDevices = 64;
struct Fork {
  cudaStream_t side = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
};
std::mutex g_fork_mutex;
Fork g_fork[kMaxForkDevices];

// Sets *out to the current device's side stream (made on first use), or to
// nullptr when cs is being captured into a graph (every launch then stays on
// cs) or the device number is out of the table's range.
cudaError_t side_stream(cudaStream_t cs, std::unique_lock<std::mutex>& lock, Fork** out) {
  *out = nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(cs, &cap);
  if (e != cudaSuccess || cap != cudaStreamCaptureStatusNone) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxForkDevices) return e;
  lock = std::unique_lock<std::mutex>(g_fork_mutex);
  Fork& f = g_fork[dev];
  if (f.side == nullptr) {
    cudaStream_t st = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (b) cudaEventDestroy(b);
      if (a) cudaEventDestroy(a);
      if (st) cudaStreamDestroy(st);
      return e;
    }
    f.side = st;
    f.start = a;
    f.done = b;
  }
  *out = &f;
  return cudaSuccess;
}

}  // namespace

cudaError_t enqueue_forward(const pack3d_config& c, const Shape& s, const ForwardWs& w, const int32_t* coords,
                            const void* q, const void* k_loc, const void* v_loc, const void* k_cmp,
                            const void* v_cmp, const float* scores, const float* gate, void* out, int32_t* err,
                            cudaStream_t cs, bool fork) {
  // RoPE reads only the coordinates and the inputs: with `fork` it runs on
  // the side stream, started after everything already on cs, while the index
  // map and the summaries run on cs; local attention waits for both.  On one
  // stream the summaries run before RoPE: both stream from HBM and are
  // independent, and the summaries write 1/16 of what they read, so RoPE
  // starts with few dirty L2 lines to evict; in the other order the summaries
  // stage would pay for writing back RoPE's output (about 10 % of its time at
  // 262k tokens).
  std::unique_lock<std::mutex> lock;
  Fork* f = nullptr;
  cudaError_t e = fork ? side_stream(cs, lock, &f) : cudaSuccess;
  if (e == cudaSuccess && f) {
    e = cudaEventRecord(f->start, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(f->side, f->start, 0);
    if (e == cudaSuccess) e = launch_rope(s, c.dtype, coords, q, w.q_rot, s.Hq, k_loc, w.k_rot, s.Hkv, f->side);
    if (e == cudaSuccess) e = cudaEventRecord(f->done, f->side);
  }
  if (e == cudaSuccess) e = launch_build_index(s, coords, w.g2p, w.members, err, cs);
  if (e == cudaSuccess) e = launch_summaries(s, c.dtype, w.members, k_cmp, v_cmp, scores, w.k_sum, w.v_sum, cs);
  if (e == cudaSuccess)
    e = f ? cudaStreamWaitEvent(cs, f->done, 0)
          : launch_rope(s, c.dtype, coords, q, w.q_rot, s.Hq, k_loc, w.k_rot, s.Hkv, cs);
  if (e == cudaSuccess)
    e = launch_local(s, c.dtype, c.flags, w.g2p, w.q_rot, w.k_rot, v_loc, w.o_loc, err, cs);
  if (e == cudaSuccess) {
    if (c.dtype == PACK3D_BF16 && !(c.flags & PACK3D_FLAG_SIMT_SUMMARY))
      e = launch_summary_attn_tc(s, w.q_rot, w.k_sum, w.v_sum, w.o_loc, gate, out, err, cs);
    else
      e = launch_summary_attn_simt(s, c.dtype, w.q_rot, w.k_sum, w.v_sum, w.o_loc, gate, out, cs);
  }
  return e;
}

}  // namespace pack3d

using namespace pack3d;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// A lattice with a zero extent holds no token: every entry point returns at
// once, before reading a pointer or launching anything.
bool empty_volume(const pack3d_config& c) { return c.Z == 0 || c.H == 0 || c.W == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int elem_bytes(int dtype) { return dtype == PACK3D_BF16 ? 2 : 4; }

pack3d_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PACK3D_OK;
  cudaGetLastError();  // clear a sticky launch-configuration error
  return PACK3D_ERR_CUDA;
}

typedef ForwardWs Workspace;

Workspace carve(const pack3d_config& c, uintptr_t base) { return carve_forward(c, base); }

// Regions of the training block after the forward workspace.
struct TrainWs {
  float* stats;   // [N,Hq,4]
  float* dqr;     // [N,Hq,64]
  float* dks;     // [M,Hkv,64], followed directly by dvs
  float* dvs;
  size_t dkv_bytes;
  float* dkl;     // [N,Hkv,64] local-branch key gradient accumulators, followed directly by dvl
  float* dvl;
  size_t dkvl_bytes;
  size_t bytes;
};

TrainWs carve_train(const pack3d_config& c, uintptr_t base) {
  const size_t N = (size_t)c.Z * c.H * c.W;
  const size_t M = N / ((size_t)c.bz * c.by * c.bx);
  const size_t A = 1024;
  TrainWs t;
  size_t off = carve(c, 0).bytes;
  t.stats = reinterpret_cast<float*>(base + off);  off = round_up(off + N * c.Hq * 16, A);
  t.dqr = reinterpret_cast<float*>(base + off);    off = round_up(off + N * c.Hq * c.d_h * 4, A);
  t.dkv_bytes = M * c.Hkv * c.d_h * 4;
  t.dks = reinterpret_cast<float*>(base + off);
  t.dvs = reinterpret_cast<float*>(base + off + t.dkv_bytes);
  off = round_up(off + 2 * t.dkv_bytes, A);
  t.dkvl_bytes = N * c.Hkv * c.d_h * 4;
  t.dkl = reinterpret_cast<float*>(base + off);
  t.dvl = reinterpret_cast<float*>(base + off + t.dkvl_bytes);
  off = round_up(off + 2 * t.dkvl_bytes, A);
  t.bytes = off;
  return t;
}

}  // namespace

extern "C" {

void pack3d_default_config(pack3d_config* cfg, int32_t Z, int32_t H, int32_t W) {
  if (!cfg) return;
  memset(cfg, 0, sizeof(*cfg));
  cfg->Z = Z; cfg->H = H; cfg->W = W;
  cfg->Hq = 8; cfg->Hkv = 2; cfg->d_h = 64;
  cfg->m_z = 11; cfg->m_y = 11; cfg->m_x = 10;
  cfg->rope_base = 10000.0;
  cfg->bz = 1; cfg->by = 4; cfg->bx = 4;
  cfg->rz = 1; cfg->ry = 3; cfg->rx = 3;
  cfg->softmax_scale = 0.125f;
  cfg->dtype = PACK3D_BF16;
  cfg->coord_scale[0] = cfg->coord_scale[1] = cfg->coord_scale[2] = 1.0;
}

pack3d_status pack3d_validate_config(const pack3d_config* c) {
  if (!c) return PACK3D_ERR_INVALID_ARG;
  if (c->reserved0 != 0 || c->reserved2 != 0 || c->wait_limit_us < 0) return PACK3D_ERR_INVALID_ARG;
  if (c->dtype != PACK3D_F32 && c->dtype != PACK3D_BF16) return PACK3D_ERR_DTYPE;
  if (c->Z < 0 || c->H < 0 || c->W < 0) return PACK3D_ERR_SHAPE;   // a zero extent is an empty volume
  const long long N = (long long)c->Z * c->H * c->W;
  if (N >= (1LL << 31) / 128) return PACK3D_ERR_SHAPE;  // keeps every element index in 32 bits
  if (c->d_h != kDh) return PACK3D_ERR_SHAPE;
  if (c->Hq <= 0 || c->Hkv <= 0 || c->Hq % c->Hkv != 0) return PACK3D_ERR_SHAPE;
  const int G = c->Hq / c->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PACK3D_ERR_SHAPE;
  if (c->m_z < 0 || c->m_y < 0 || c->m_x < 0 || 2 * (c->m_z + c->m_y + c->m_x) > c->d_h)
    return PACK3D_ERR_SHAPE;
  if (!(c->rope_base > 0.0) || !isfinite(c->rope_base)) return PACK3D_ERR_INVALID_ARG;
  if (c->bz <= 0 || c->by <= 0 || c->bx <= 0) return PACK3D_ERR_SHAPE;
  if (c->Z % c->bz || c->H % c->by || c->W % c->bx) return PACK3D_ERR_SHAPE;
  if (c->bz * c->by * c->bx > 64) return PACK3D_ERR_SHAPE;
  if (c->rz < 0 || c->ry < 0 || c->rx < 0) return PACK3D_ERR_SHAPE;
  if (!(c->softmax_scale > 0.f) || !isfinite(c->softmax_scale)) return PACK3D_ERR_INVALID_ARG;
  for (int a = 0; a < 3; ++a)
    if (!(c->coord_scale[a] > 0.0) || !isfinite(c->coord_scale[a])) return PACK3D_ERR_INVALID_ARG;
  const long long tab = (long long)c->Z * c->m_z + (long long)c->H * c->m_y + (long long)c->W * c->m_x;
  if (tab * 8 > kMaxTableBytes) return PACK3D_ERR_SHAPE;
  if (c->flags & ~(PACK3D_FLAG_SIMT_SUMMARY | PACK3D_FLAG_SIMT_LOCAL | PACK3D_FLAG_SUMMARY_CENTER |
                   PACK3D_FLAG_DIAG_STALL | PACK3D_FLAG_SUMMARY_ONE_TILE | PACK3D_FLAG_SUMMARY_TWO_TILE))
    return PACK3D_ERR_INVALID_ARG;
  if ((c->flags & PACK3D_FLAG_SUMMARY_ONE_TILE) && (c->flags & PACK3D_FLAG_SUMMARY_TWO_TILE))
    return PACK3D_ERR_INVALID_ARG;
  return PACK3D_OK;
}

size_t pack3d_workspace_bytes(const pack3d_config* cfg) {
  if (pack3d_validate_config(cfg) != PACK3D_OK) return 0;
  return carve(*cfg, 0).bytes;
}

pack3d_status pack3d_build_index(const pack3d_config* cfg, const int32_t* coords, int32_t* g2p,
                                 int32_t* members, int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!coords || !g2p || !members || !err_word) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(coords) || !aligned16(g2p) || !aligned16(members)) return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(launch_build_index(s, coords, g2p, members, err_word, (cudaStream_t)stream));
}

pack3d_status pack3d_rope(const pack3d_config* cfg, const int32_t* coords, const void* x, void* y,
                          int32_t heads, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!coords || !x || !y || heads <= 0) return PACK3D_ERR_INVALID_ARG;
  if ((long long)cfg->Z * cfg->H * cfg->W * heads >= (1LL << 31) / 16) return PACK3D_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y)) return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(launch_rope(s, cfg->dtype, coords, x, y, heads, nullptr, nullptr, 0,
                                 (cudaStream_t)stream));
}

pack3d_status pack3d_rope_qk(const pack3d_config* cfg, const int32_t* coords, const void* q, void* q_rot,
                             const void* k, void* k_rot, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!coords || !q || !q_rot || !k || !k_rot) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(q_rot) || !aligned16(k) || !aligned16(k_rot)) return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(launch_rope(s, cfg->dtype, coords, q, q_rot, s.Hq, k, k_rot, s.Hkv, (cudaStream_t)stream));
}

pack3d_status pack3d_build_summaries(const pack3d_config* cfg, const int32_t* members, const void* k_cmp,
                                     const void* v_cmp, const float* scores, void* k_sum, void* v_sum,
                                     void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!members || !k_cmp || !v_cmp || !scores || !k_sum || !v_sum) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(k_cmp) || !aligned16(v_cmp) || !aligned16(k_sum) || !aligned16(v_sum))
    return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(
      launch_summaries(s, cfg->dtype, members, k_cmp, v_cmp, scores, k_sum, v_sum, (cudaStream_t)stream));
}

pack3d_status pack3d_local_attn(const pack3d_config* cfg, const int32_t* g2p, const void* q_rot,
                                const void* k_rot, const void* v_loc, float* o_loc, int32_t* err_word,
                                void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!g2p || !q_rot || !k_rot || !v_loc || !o_loc) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(k_rot) || !aligned16(v_loc) || !aligned16(o_loc))
    return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(
      launch_local(s, cfg->dtype, cfg->flags, g2p, q_rot, k_rot, v_loc, o_loc, err_word, (cudaStream_t)stream));
}

pack3d_status pack3d_summary_attn(const pack3d_config* cfg, const void* q_rot, const void* k_sum,
                                  const void* v_sum, const float* o_loc, const float* gate, void* out,
                                  int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!q_rot || !k_sum || !v_sum || !out || (gate && !o_loc)) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(k_sum) || !aligned16(v_sum) || !aligned16(out) ||
      (o_loc && !aligned16(o_loc)))
    return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  cudaError_t e;
  if (cfg->dtype == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY))
    e = launch_summary_attn_tc(s, q_rot, k_sum, v_sum, o_loc, gate, out, err_word, (cudaStream_t)stream);
  else
    e = launch_summary_attn_simt(s, cfg->dtype, q_rot, k_sum, v_sum, o_loc, gate, out, (cudaStream_t)stream);
  return cuda_status(e);
}

pack3d_status pack3d_summary_attn_rows(const pack3d_config* cfg, int64_t tokens, int64_t summaries, const void* q_rot,
                                       const void* k_sum, const void* v_sum, const float* o_loc, const float* gate,
                                       void* out, int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (tokens < 0 || summaries < 0) return PACK3D_ERR_INVALID_ARG;
  if (tokens == 0 || summaries == 0) return PACK3D_OK;
  // The same 32-bit element-index bound as a lattice (tokens x Hq x 64 and summaries x Hkv x 64).
  if (tokens >= (1LL << 31) / 128 || summaries >= (1LL << 31) / 128) return PACK3D_ERR_SHAPE;
  if (!q_rot || !k_sum || !v_sum || !out || (gate && !o_loc)) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(k_sum) || !aligned16(v_sum) || !aligned16(out) ||
      (o_loc && !aligned16(o_loc)))
    return PACK3D_ERR_ALIGNMENT;
  Shape s = make_shape(*cfg);
  s.N = (int)tokens;
  s.M = (int)summaries;
  cudaError_t e;
  if (cfg->dtype == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY))
    e = launch_summary_attn_tc(s, q_rot, k_sum, v_sum, o_loc, gate, out, err_word, (cudaStream_t)stream);
  else
    e = launch_summary_attn_simt(s, cfg->dtype, q_rot, k_sum, v_sum, o_loc, gate, out, (cudaStream_t)stream);
  return cuda_status(e);
}

pack3d_status pack3d_exp2_fma_eval(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return PACK3D_ERR_INVALID_ARG;
  if (n == 0) return PACK3D_OK;
  if (!x || !y) return PACK3D_ERR_INVALID_ARG;
  return cuda_status(launch_exp2_fma_eval(x, y, n, (cudaStream_t)stream));
}

pack3d_status pack3d_gather_rows(const int32_t* idx, int64_t n, const void* src, void* dst, int64_t row_bytes,
                                 void* stream) {
  if (n < 0 || row_bytes <= 0 || row_bytes % 16 != 0 || row_bytes / 16 > INT32_MAX) return PACK3D_ERR_INVALID_ARG;
  if (n == 0) return PACK3D_OK;
  if (!idx || !src || !dst) return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return PACK3D_ERR_ALIGNMENT;
  return cuda_status(launch_gather_rows(idx, n, src, dst, row_bytes, (cudaStream_t)stream));
}

pack3d_status pack3d_forward(const pack3d_config* cfg, const int32_t* coords, const void* q, const void* k_loc,
                             const void* v_loc, const void* k_cmp, const void* v_cmp, const float* scores,
                             const float* gate, void* out, void* workspace, size_t workspace_bytes,
                             int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!coords || !q || !k_loc || !v_loc || !k_cmp || !v_cmp || !scores || !gate || !out || !err_word)
    return PACK3D_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace & 255u)) return PACK3D_ERR_WORKSPACE;
  Workspace w = carve(*cfg, (uintptr_t)workspace);
  if (workspace_bytes < w.bytes) return PACK3D_ERR_WORKSPACE;
  if (!aligned16(coords) || !aligned16(q) || !aligned16(k_loc) || !aligned16(v_loc) || !aligned16(k_cmp) ||
      !aligned16(v_cmp) || !aligned16(out))
    return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  return cuda_status(enqueue_forward(*cfg, s, w, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out,
                                     err_word, (cudaStream_t)stream, true));
}

size_t pack3d_train_workspace_bytes(const pack3d_config* cfg) {
  if (pack3d_validate_config(cfg) != PACK3D_OK) return 0;
  return carve_train(*cfg, 0).bytes;
}

pack3d_status pack3d_forward_backward(const pack3d_config* cfg, const int32_t* coords, const void* q,
                                      const void* k_loc, const void* v_loc, const void* k_cmp, const void* v_cmp,
                                      const float* scores, const float* gate, const void* dout, void* out,
                                      void* dq, void* dk_loc, void* dv_loc, void* dk_cmp, void* dv_cmp,
                                      float* dscores, float* dgate, void* workspace, size_t workspace_bytes,
                                      int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!coords || !q || !k_loc || !v_loc || !k_cmp || !v_cmp || !scores || !gate || !dout || !out || !dq ||
      !dk_loc || !dv_loc || !dk_cmp || !dv_cmp || !dscores || !dgate || !err_word)
    return PACK3D_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace & 255u)) return PACK3D_ERR_WORKSPACE;
  const Workspace w = carve(*cfg, (uintptr_t)workspace);
  const TrainWs t = carve_train(*cfg, (uintptr_t)workspace);
  if (workspace_bytes < t.bytes) return PACK3D_ERR_WORKSPACE;
  const void* ptrs[] = {coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, dout, out, dq,
                        dk_loc, dv_loc, dk_cmp, dv_cmp, dscores, dgate};
  for (const void* p : ptrs)
    if (!aligned16(p)) return PACK3D_ERR_ALIGNMENT;
  const Shape s = make_shape(*cfg);
  const int dt = cfg->dtype;
  const cudaStream_t cs = (cudaStream_t)stream;
  // Forward, leaving the row statistics and dgate.
  cudaError_t e = launch_build_index(s, coords, w.g2p, w.members, err_word, cs);
  if (e == cudaSuccess) e = launch_summaries(s, dt, w.members, k_cmp, v_cmp, scores, w.k_sum, w.v_sum, cs);
  if (e == cudaSuccess) e = launch_rope(s, dt, coords, q, w.q_rot, s.Hq, k_loc, w.k_rot, s.Hkv, cs);
  if (e == cudaSuccess)
    e = launch_local(s, dt, cfg->flags, w.g2p, w.q_rot, w.k_rot, v_loc, w.o_loc, err_word, cs, t.stats);
  const Train tr{t.stats, dout, dgate};
  if (e == cudaSuccess) {
    if (dt == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY))
      e = launch_summary_attn_tc(s, w.q_rot, w.k_sum, w.v_sum, w.o_loc, gate, out, err_word, cs, 0, -1, &tr);
    else
      e = launch_summary_attn_simt(s, dt, w.q_rot, w.k_sum, w.v_sum, w.o_loc, gate, out, cs, &tr);
  }
  // Backward: compressed branch, local branch, summaries (RoPE transposes fused).
  if (e == cudaSuccess) e = cudaMemsetAsync(t.dks, 0, 2 * t.dkv_bytes, cs);
  if (dt == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY)) {
    if (e == cudaSuccess)
      e = launch_summary_bwd_dq_tc(s, w.q_rot, w.k_sum, w.v_sum, dout, gate, t.stats, t.dqr, err_word, cs);
    if (e == cudaSuccess)
      e = launch_summary_bwd_dkv_tc(s, w.q_rot, w.k_sum, w.v_sum, dout, gate, t.stats, t.dks, t.dvs, err_word, cs);
  } else {
    if (e == cudaSuccess)
      e = launch_summary_bwd_dq(s, dt, w.q_rot, w.k_sum, w.v_sum, dout, gate, t.stats, t.dqr, cs);
    if (e == cudaSuccess)
      e = launch_summary_bwd_dkv(s, dt, w.q_rot, w.k_sum, w.v_sum, dout, gate, t.stats, t.dks, t.dvs, cs);
  }
  if (!(cfg->flags & PACK3D_FLAG_SIMT_LOCAL) && local_attn_tc_supported(s, dt)) {
    if (e == cudaSuccess) e = cudaMemsetAsync(t.dkl, 0, 2 * t.dkvl_bytes, cs);
    if (e == cudaSuccess)
      e = launch_local_bwd_tc(s, w.g2p, w.q_rot, w.k_rot, v_loc, dout, gate, t.stats, t.dqr, t.dkl, t.dvl,
                              err_word, cs);
    if (e == cudaSuccess) e = launch_local_bwd_finalize(s, dt, coords, t.dqr, t.dkl, t.dvl, dq, dk_loc, dv_loc, cs);
  } else {
    if (e == cudaSuccess)
      e = launch_local_bwd_dq(s, dt, w.g2p, w.q_rot, w.k_rot, v_loc, dout, gate, t.stats, t.dqr, dq, cs);
    if (e == cudaSuccess)
      e = launch_local_bwd_dkv(s, dt, w.g2p, w.q_rot, w.k_rot, v_loc, dout, gate, t.stats, dk_loc, dv_loc, cs);
  }
  if (e == cudaSuccess)
    e = launch_summaries_bwd(s, dt, coords, w.members, k_cmp, v_cmp, scores, t.dks, t.dvs, dk_cmp, dv_cmp,
                             dscores, cs);
  return cuda_status(e);
}

// ---- forward pass from host buffers -------------------------------------------

}  // extern "C"

// Streams and events of pack3d_forward_host, owned by the caller through the
// opaque handle (the library itself keeps no state between calls).
struct pack3d_pipeline {
  int device;
  cudaStream_t in, out;
  cudaEvent_t start, coords, cmp, qk, vloc, gate, done;
  cudaEvent_t chunk[PACK3D_HOST_MAX_CHUNKS];
};

namespace {

// Device staging copies of the inputs and the output, after the regions of
// the pack3d_forward workspace.
struct Staging {
  uintptr_t coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out;
  size_t bytes;
};

Staging plan_staging(const pack3d_config& c, size_t base_off) {
  const size_t N = (size_t)c.Z * c.H * c.W;
  const size_t eb = elem_bytes(c.dtype);
  const size_t A = 1024;
  Staging g;
  size_t off = round_up(base_off, A);
  g.coords = off; off = round_up(off + N * 12, A);
  g.q = off;      off = round_up(off + N * c.Hq * c.d_h * eb, A);
  g.k_loc = off;  off = round_up(off + N * c.Hkv * c.d_h * eb, A);
  g.v_loc = off;  off = round_up(off + N * c.Hkv * c.d_h * eb, A);
  g.k_cmp = off;  off = round_up(off + N * c.Hkv * c.d_h * eb, A);
  g.v_cmp = off;  off = round_up(off + N * c.Hkv * c.d_h * eb, A);
  g.scores = off; off = round_up(off + N * c.Hkv * 4, A);
  g.gate = off;   off = round_up(off + N * c.Hq * 8, A);
  g.out = off;    off = round_up(off + N * c.Hq * c.d_h * eb, A);
  g.bytes = off;
  return g;
}

}  // namespace

extern "C" {

pack3d_status pack3d_pipeline_create(pack3d_pipeline** out) {
  if (!out) return PACK3D_ERR_INVALID_ARG;
  *out = nullptr;
  pack3d_pipeline* p = new (std::nothrow) pack3d_pipeline();
  if (!p) return PACK3D_ERR_CUDA;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->out, cudaStreamNonBlocking);
  cudaEvent_t* evs[] = {&p->start, &p->coords, &p->cmp, &p->qk, &p->vloc, &p->gate, &p->done};
  for (cudaEvent_t* ev : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int c = 0; c < PACK3D_HOST_MAX_CHUNKS && e == cudaSuccess; ++c)
    e = cudaEventCreateWithFlags(&p->chunk[c], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    cudaGetLastError();
    pack3d_pipeline_destroy(p);
    return PACK3D_ERR_CUDA;
  }
  *out = p;
  return PACK3D_OK;
}

void pack3d_pipeline_destroy(pack3d_pipeline* p) {
  if (!p) return;
  cudaEvent_t evs[] = {p->start, p->coords, p->cmp, p->qk, p->vloc, p->gate, p->done};
  for (cudaEvent_t ev : evs)
    if (ev) cudaEventDestroy(ev);
  for (int c = 0; c < PACK3D_HOST_MAX_CHUNKS; ++c)
    if (p->chunk[c]) cudaEventDestroy(p->chunk[c]);
  if (p->in) cudaStreamDestroy(p->in);
  if (p->out) cudaStreamDestroy(p->out);
  delete p;
}

size_t pack3d_host_workspace_bytes(const pack3d_config* cfg) {
  if (pack3d_validate_config(cfg) != PACK3D_OK) return 0;
  return plan_staging(*cfg, carve(*cfg, 0).bytes).bytes;
}

pack3d_status pack3d_forward_host(pack3d_pipeline* pl, const pack3d_config* cfg, const int32_t* coords,
                                  const void* q, const void* k_loc, const void* v_loc, const void* k_cmp,
                                  const void* v_cmp, const float* scores, const float* gate, void* out,
                                  void* workspace, size_t workspace_bytes, int32_t* err_word, void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;
  if (!pl || !coords || !q || !k_loc || !v_loc || !k_cmp || !v_cmp || !scores || !gate || !out || !err_word)
    return PACK3D_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace & 255u)) return PACK3D_ERR_WORKSPACE;
  const Workspace w = carve(*cfg, (uintptr_t)workspace);
  const Staging g = plan_staging(*cfg, w.bytes);
  if (workspace_bytes < g.bytes) return PACK3D_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->device) {
    cudaGetLastError();
    return PACK3D_ERR_INVALID_ARG;   // the pipeline belongs to another device
  }
  const Shape s = make_shape(*cfg);
  const size_t N = (size_t)s.N, eb = elem_bytes(cfg->dtype);
  const uintptr_t base = (uintptr_t)workspace;
  auto dptr = [&](uintptr_t off) { return reinterpret_cast<void*>(base + off); };
  const cudaStream_t cs = (cudaStream_t)stream, in = pl->in, outs = pl->out;
  const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
  const size_t qb = N * s.Hq * kDh * eb, kvb = N * s.Hkv * kDh * eb;

  // The staging area may still be read by earlier work on `stream`.
  cudaError_t e = cudaEventRecord(pl->start, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(in, pl->start, 0);
  // Inputs in the order the stages need them, each group marked by an event.
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.coords), coords, N * 12, h2d, in);
  if (e == cudaSuccess) e = cudaEventRecord(pl->coords, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.k_cmp), k_cmp, kvb, h2d, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.v_cmp), v_cmp, kvb, h2d, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.scores), scores, N * s.Hkv * 4, h2d, in);
  if (e == cudaSuccess) e = cudaEventRecord(pl->cmp, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.k_loc), k_loc, kvb, h2d, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.q), q, qb, h2d, in);
  if (e == cudaSuccess) e = cudaEventRecord(pl->qk, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.v_loc), v_loc, kvb, h2d, in);
  if (e == cudaSuccess) e = cudaEventRecord(pl->vloc, in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dptr(g.gate), gate, N * s.Hq * 8, h2d, in);
  if (e == cudaSuccess) e = cudaEventRecord(pl->gate, in);

  // Each stage waits only for the copies it reads.
  const int32_t* dcoords = (const int32_t*)dptr(g.coords);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->coords, 0);
  if (e == cudaSuccess) e = launch_build_index(s, dcoords, w.g2p, w.members, err_word, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->cmp, 0);
  if (e == cudaSuccess)
    e = launch_summaries(s, cfg->dtype, w.members, dptr(g.k_cmp), dptr(g.v_cmp), (const float*)dptr(g.scores),
                         w.k_sum, w.v_sum, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->qk, 0);
  if (e == cudaSuccess)
    e = launch_rope(s, cfg->dtype, dcoords, dptr(g.q), w.q_rot, s.Hq, dptr(g.k_loc), w.k_rot, s.Hkv, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->vloc, 0);
  if (e == cudaSuccess)
    e = launch_local(s, cfg->dtype, cfg->flags, w.g2p, w.q_rot, w.k_rot, dptr(g.v_loc), w.o_loc, err_word, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->gate, 0);

  // The query x summary stage in token chunks; each chunk's rows go back to
  // the host on the second copy stream while the next chunk computes.
  const float* dgate = (const float*)dptr(g.gate);
  void* dout = dptr(g.out);
  const size_t row_bytes = (size_t)s.Hq * kDh * eb;   // one token's output
  const bool tc = cfg->dtype == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY);
  int chunks = 1;
  long quantum = (long)N;
  if (tc) {
    quantum = summary_attn_tc_token_quantum(s);
    // About 8 MiB of output per chunk, at most PACK3D_HOST_MAX_CHUNKS chunks.
    chunks = (int)min((long)PACK3D_HOST_MAX_CHUNKS, max(1L, (long)(N * row_bytes / (8u << 20))));
  }
  const long per_chunk = ((long)N / chunks + quantum - 1) / quantum * quantum;
  for (int c = 0; c < chunks && e == cudaSuccess; ++c) {
    const long t0 = c * per_chunk, t1 = min((long)N, t0 + per_chunk);
    if (t0 >= t1) break;
    if (tc)
      e = launch_summary_attn_tc(s, w.q_rot, w.k_sum, w.v_sum, w.o_loc, dgate, dout, err_word, cs, t0, t1);
    else
      e = launch_summary_attn_simt(s, cfg->dtype, w.q_rot, w.k_sum, w.v_sum, w.o_loc, dgate, dout, cs);
    if (e == cudaSuccess) e = cudaEventRecord(pl->chunk[c], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(outs, pl->chunk[c], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync((uint8_t*)out + t0 * row_bytes, (const uint8_t*)dout + t0 * row_bytes,
                          (t1 - t0) * row_bytes, cudaMemcpyDeviceToHost, outs);
  }
  // Everything joins `stream`: synchronising it covers every copy.
  if (e == cudaSuccess) e = cudaEventRecord(pl->done, outs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pl->done, 0);
  return cuda_status(e);
}

pack3d_status pack3d_check_status(int32_t* err_word, void* stream) {
  if (!err_word) return PACK3D_ERR_INVALID_ARG;
  int32_t h = 0;
  const cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&h, err_word, sizeof(h), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(err_word, 0, sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_status(e);
  if (h & PACK3D_DEVERR_TIMEOUT) return PACK3D_ERR_TIMEOUT;
  if (h & (PACK3D_DEVERR_COORD_RANGE | PACK3D_DEVERR_DUPLICATE)) return PACK3D_ERR_NOT_PERMUTATION;
  return PACK3D_OK;
}

const char* pack3d_status_string(pack3d_status s) {
  switch (s) {
    case PACK3D_OK: return "ok";
    case PACK3D_ERR_INVALID_ARG: return "invalid argument";
    case PACK3D_ERR_SHAPE: return "unsupported or inconsistent shape";
    case PACK3D_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case PACK3D_ERR_DTYPE: return "unsupported dtype";
    case PACK3D_ERR_NOT_PERMUTATION: return "coordinates are not a bijection onto the lattice";
    case PACK3D_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PACK3D_ERR_CUDA: return "CUDA runtime error";
    case PACK3D_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* pack3d_backend_info(void) {
  return "pack3d sm_100a: index map; axial RoPE (CUDA cores, 16-byte streams, shared-memory cos/sin tables); "
         "summaries (warp per block, rotation split R(c_base) R(d)); local attention (bf16 G=4: tcgen05 MMA on "
         "2x4x4 query bricks with gathered halo planes; else CUDA cores); query x summary (bf16: tcgen05 MMA, "
         "TMEM accumulators, TMA 5-stage ring, two softmax warpgroups with one MMA warp each; float: CUDA "
         "cores); host-buffer pipeline with copies overlapped on two copy streams";
}

}  // extern "C"
