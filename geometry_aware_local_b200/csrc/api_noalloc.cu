// pack3d_forward_noalloc: the whole forward pass for callers that cannot
// allocate device memory.
//
// pack3d_forward needs a caller-provided workspace (index map, membership,
// rotated Q/K, summaries, local-branch output).  Some callers cannot obtain
// one: a plugin whose host application owns every device allocation and only
// hands over input and output buffers, code on a path where cudaMalloc is
// forbidden because it may synchronise the device, or a process whose memory
// is entirely reserved by another allocator.  This entry point instead uses a
// fixed scratch array compiled into the library (a file-scope __device__
// array, kNoallocScratchBytes bytes), so it calls no cudaMalloc, cudaFree or
// other allocating routine.  Every GPU that loads the library holds the array
// until the process exits.
//
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress (with that device current) and caches it per device;
// make that first call before any stream capture.  All calls share the one
// array, so calls whose work overlaps on the GPU (for example on two streams)
// race and must be serialised by the caller.  Each region of the scratch is
// fully written by this call's kernels before it is read (the index maps are
// reset to -1 first), so nothing left by a previous call leaks into the
// result.
#include <mutex>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"
#include "pack3d.h"

namespace {

constexpr size_t kNoallocScratchBytes = PACK3D_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Same regions as pack3d_forward's workspace, carved from the static array.
struct Regions {
  size_t g2p, members, q_rot, k_rot, k_sum, v_sum, o_loc, bytes;
};

Regions plan(const pack3d_config& c) {
  const size_t N = (size_t)c.Z * c.H * c.W;
  const size_t v = (size_t)c.bz * c.by * c.bx;
  const size_t M = N / v;
  const size_t eb = c.dtype == PACK3D_BF16 ? 2 : 4;
  Regions r;
  size_t off = 0;
  r.g2p = off;     off = align_up(off + N * 4, 1024);
  r.members = off; off = align_up(off + M * v * 4, 1024);
  r.q_rot = off;   off = align_up(off + N * c.Hq * c.d_h * eb, 1024);
  r.k_rot = off;   off = align_up(off + N * c.Hkv * c.d_h * eb, 1024);
  r.k_sum = off;   off = align_up(off + M * c.Hkv * c.d_h * eb, 1024);
  r.v_sum = off;   off = align_up(off + M * c.Hkv * c.d_h * eb, 1024);
  r.o_loc = off;   off = align_up(off + N * c.Hq * c.d_h * 4, 1024);
  r.bytes = off;
  return r;
}

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_scratch_addr[dev]);
  return cudaSuccess;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool empty_volume(const pack3d_config& c) { return c.Z == 0 || c.H == 0 || c.W == 0; }

}  // namespace

using namespace pack3d;

extern "C" pack3d_status pack3d_forward_noalloc(const pack3d_config* cfg, const int32_t* coords,
                                                const void* q, const void* k_loc, const void* v_loc,
                                                const void* k_cmp, const void* v_cmp, const float* scores,
                                                const float* gate, void* out, int32_t* err_word,
                                                void* stream) {
  pack3d_status st = pack3d_validate_config(cfg);
  if (st != PACK3D_OK) return st;
  if (empty_volume(*cfg)) return PACK3D_OK;   // no token: nothing to read or launch
  if (!coords || !q || !k_loc || !v_loc || !k_cmp || !v_cmp || !scores || !gate || !out)
    return PACK3D_ERR_INVALID_ARG;
  if (!aligned16(coords) || !aligned16(q) || !aligned16(k_loc) || !aligned16(v_loc) || !aligned16(k_cmp) ||
      !aligned16(v_cmp) || !aligned16(out))
    return PACK3D_ERR_ALIGNMENT;
  const Regions r = plan(*cfg);
  if (r.bytes > kNoallocScratchBytes) return PACK3D_ERR_WORKSPACE;  // volume too large for the array
  uint8_t* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) {
    cudaGetLastError();
    return PACK3D_ERR_CUDA;
  }
  int32_t* g2p = reinterpret_cast<int32_t*>(base + r.g2p);
  int32_t* members = reinterpret_cast<int32_t*>(base + r.members);
  void* q_rot = base + r.q_rot;
  void* k_rot = base + r.k_rot;
  void* k_sum = base + r.k_sum;
  void* v_sum = base + r.v_sum;
  float* o_loc = reinterpret_cast<float*>(base + r.o_loc);

  const Shape s = make_shape(*cfg);
  const cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = launch_build_index(s, coords, g2p, members, err_word, cs);
  if (e == cudaSuccess) e = launch_rope(s, cfg->dtype, coords, q, q_rot, s.Hq, k_loc, k_rot, s.Hkv, cs);
  if (e == cudaSuccess) e = launch_summaries(s, cfg->dtype, members, k_cmp, v_cmp, scores, k_sum, v_sum, cs);
  if (e == cudaSuccess) e = launch_local(s, cfg->dtype, cfg->flags, g2p, q_rot, k_rot, v_loc, o_loc, err_word, cs);
  if (e == cudaSuccess) {
    if (cfg->dtype == PACK3D_BF16 && !(cfg->flags & PACK3D_FLAG_SIMT_SUMMARY))
      e = launch_summary_attn_tc(s, q_rot, k_sum, v_sum, o_loc, gate, out, err_word, cs);
    else
      e = launch_summary_attn_simt(s, cfg->dtype, q_rot, k_sum, v_sum, o_loc, gate, out, cs);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return PACK3D_ERR_CUDA;
  }
  return PACK3D_OK;
}
