// Internal launchers of the PACK3D kernels; the C ABI in api.cu validates
// arguments and then calls these.  Each returns the first CUDA error seen.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pack3d {

struct Shape;

cudaError_t launch_build_index(const Shape& s, const int32_t* coords, int32_t* g2p,
                               int32_t* members, int32_t* err, cudaStream_t st);

// Rotates x0 -> y0 (h0 heads) and, if x1 is not null, x1 -> y1 (h1 heads).
cudaError_t launch_rope(const Shape& s, int dtype, const int32_t* coords, const void* x0, void* y0,
                        int h0, const void* x1, void* y1, int h1, cudaStream_t st);

cudaError_t launch_summaries(const Shape& s, int dtype, const int32_t* members, const void* kc,
                             const void* vc, const float* scores, void* ks, void* vs,
                             cudaStream_t st);

cudaError_t launch_local_attn(const Shape& s, int dtype, const int32_t* g2p, const void* qr,
                              const void* kr, const void* vl, float* oloc, cudaStream_t st);

// Local attention on the best kernel for the shape: tcgen05 when supported
// and not disabled by PACK3D_FLAG_SIMT_LOCAL, else CUDA cores.
cudaError_t launch_local(const Shape& s, int dtype, int flags, const int32_t* g2p, const void* qr,
                         const void* kr, const void* vl, float* oloc, int32_t* err, cudaStream_t st);

// tcgen05 local attention (bf16, G = 4, rz = 1, ry <= 3, rx <= 3).
bool local_attn_tc_supported(const Shape& s, int dtype);
cudaError_t launch_local_attn_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, float* oloc, int32_t* err, cudaStream_t st);

// CUDA-core query x summary kernel (float, or bf16 on request).
cudaError_t launch_summary_attn_simt(const Shape& s, int dtype, const void* qr, const void* ks,
                                     const void* vs, const float* oloc, const float* gate,
                                     void* out, cudaStream_t st);

// tcgen05 query x summary kernel (bf16 only), for the tokens [tok_begin,
// tok_end) (tok_end < 0: to the end); tok_begin must be a multiple of
// summary_attn_tc_token_quantum(s), the tokens one CTA covers.
cudaError_t launch_summary_attn_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                   const float* oloc, const float* gate, void* out, int32_t* err,
                                   cudaStream_t st, long tok_begin = 0, long tok_end = -1);
long summary_attn_tc_token_quantum(const Shape& s);

}  // namespace pack3d
