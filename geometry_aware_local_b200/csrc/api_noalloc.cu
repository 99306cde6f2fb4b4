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
// make that first call before any stream capture.  The cached address belongs
// to the device's current context: after cudaDeviceReset the module may be
// loaded again at another address, so a process that resets a device must not
// call this entry point on it again.  All calls share the one
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
  // The same regions (and the same size check) as pack3d_forward's workspace.
  if (carve_forward(*cfg, 0).bytes > kNoallocScratchBytes) return PACK3D_ERR_WORKSPACE;  // too large
  uint8_t* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) {
    cudaGetLastError();
    return PACK3D_ERR_CUDA;
  }
  const ForwardWs w = carve_forward(*cfg, (uintptr_t)base);
  const Shape s = make_shape(*cfg);
  const cudaError_t e = enqueue_forward(*cfg, s, w, coords, q, k_loc, v_loc, k_cmp, v_cmp, scores, gate, out,
                                        err_word, (cudaStream_t)stream, false);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return PACK3D_ERR_CUDA;
  }
  return PACK3D_OK;
}
