// Internal launchers of the PACK3D kernels; the C ABI in api.cu validates
// arguments and then calls these.  Each returns the first CUDA error seen.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pack3d.h"

namespace pack3d {

struct Shape;

// Regions of the pack3d_forward workspace, each at a 1 KiB offset from base:
// g2p int32 [N], members int32 [M,v], q_rot, k_rot (operator dtype), k_sum,
// v_sum [M,Hkv,64], o_loc float [N,Hq,64].  `bytes` is the total size.
struct ForwardWs {
  int32_t* g2p;
  int32_t* members;
  void* q_rot;
  void* k_rot;
  void* k_sum;
  void* v_sum;
  float* o_loc;
  size_t bytes;
};
ForwardWs carve_forward(const pack3d_config& c, uintptr_t base);

// The forward pass's launches, stream-ordered on st, on a carved workspace
// (pack3d_forward and pack3d_forward_noalloc both run exactly this).  With
// `fork`, RoPE runs on a per-device side stream (made on first use) that
// starts after st's earlier work and that st waits for before local
// attention; inside a stream capture, or without `fork`, all launches stay on st.
cudaError_t enqueue_forward(const pack3d_config& c, const Shape& s, const ForwardWs& w, const int32_t* coords,
                            const void* q, const void* k_loc, const void* v_loc, const void* k_cmp,
                            const void* v_cmp, const float* scores, const float* gate, void* out, int32_t* err,
                            cudaStream_t st, bool fork);

// Extra outputs of the forward pass when it runs as the first half of the
// training block (pack3d_forward_backward): per (token, q head) row four
// floats of statistics for the backward, the gate gradient, and the output
// gradient they are formed with.  Null pointers: plain forward.
struct Train {
  float* stats;        // [N, Hq, 4]: lse2 local, lse2 compressed, delta local, delta compressed
  const void* dout;    // [N, Hq, 64] in the operator's dtype
  float* dgate;        // [N, Hq, 2]
};

cudaError_t launch_exp2_fma_eval(const float* x, float* y, long long n, cudaStream_t st);
cudaError_t launch_gather_rows(const int32_t* idx, long long n, const void* src, void* dst, long long row_bytes,
                               cudaStream_t st);
cudaError_t launch_build_index(const Shape& s, const int32_t* coords, int32_t* g2p,
                               int32_t* members, int32_t* err, cudaStream_t st);

// Rotates x0 -> y0 (h0 heads) and, if x1 is not null, x1 -> y1 (h1 heads).
cudaError_t launch_rope(const Shape& s, int dtype, const int32_t* coords, const void* x0, void* y0,
                        int h0, const void* x1, void* y1, int h1, cudaStream_t st);

cudaError_t launch_summaries(const Shape& s, int dtype, const int32_t* members, const void* kc,
                             const void* vc, const float* scores, void* ks, void* vs,
                             cudaStream_t st);

// stats (nullable): the local softmax's lse2 (log2 units of the scaled logits)
// goes to stats[4 row].
cudaError_t launch_local_attn(const Shape& s, int dtype, const int32_t* g2p, const void* qr,
                              const void* kr, const void* vl, float* oloc, cudaStream_t st,
                              float* stats = nullptr);

// Local attention on the best kernel for the shape: tcgen05 when supported
// and not disabled by PACK3D_FLAG_SIMT_LOCAL, else CUDA cores.
cudaError_t launch_local(const Shape& s, int dtype, int flags, const int32_t* g2p, const void* qr,
                         const void* kr, const void* vl, float* oloc, int32_t* err, cudaStream_t st,
                         float* stats = nullptr);

// tcgen05 local attention (bf16, G = 4, rz = 1, ry <= 3, rx <= 3).
bool local_attn_tc_supported(const Shape& s, int dtype);
cudaError_t launch_local_attn_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, float* oloc, int32_t* err, cudaStream_t st,
                                 float* stats = nullptr);

// CUDA-core query x summary kernel (float, or bf16 on request).
cudaError_t launch_summary_attn_simt(const Shape& s, int dtype, const void* qr, const void* ks,
                                     const void* vs, const float* oloc, const float* gate,
                                     void* out, cudaStream_t st, const Train* tr = nullptr);

// tcgen05 query x summary kernel (bf16 only), for the tokens [tok_begin,
// tok_end) (tok_end < 0: to the end); tok_begin must be a multiple of
// summary_attn_tc_token_quantum(s), the tokens one CTA covers.
cudaError_t launch_summary_attn_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                   const float* oloc, const float* gate, void* out, int32_t* err,
                                   cudaStream_t st, long tok_begin = 0, long tok_end = -1,
                                   const Train* tr = nullptr);
long summary_attn_tc_token_quantum(const Shape& s);

// ---- backward pass of the training block (k_backward.cu) ----
// Inputs: the forward's rotated Q / K_loc, summaries, statistics and the
// output gradient; float accumulators dqr [N,Hq,64] and dks / dvs [M,Hkv,64].

// Compressed branch, query side: dqr = scale * sum_j dS_j k~_j (overwrites dqr).
cudaError_t launch_summary_bwd_dq(const Shape& s, int dtype, const void* qr, const void* ks, const void* vs,
                                  const void* dout, const float* gate, const float* stats, float* dqr,
                                  cudaStream_t st);
// Compressed branch, summary side: dks += scale * sum_i dS_i q_i, dvs += sum_i P_i do_i
// (float atomics; dks and dvs must be zeroed first).
cudaError_t launch_summary_bwd_dkv(const Shape& s, int dtype, const void* qr, const void* ks, const void* vs,
                                   const void* dout, const float* gate, const float* stats, float* dks,
                                   float* dvs, cudaStream_t st);
// The same two steps on tcgen05 tensor cores (bf16, k_summary_bwd_tc.cu).
cudaError_t launch_summary_bwd_dq_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                     const void* dout, const float* gate, const float* stats, float* dqr,
                                     int32_t* err, cudaStream_t st);
cudaError_t launch_summary_bwd_dkv_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                      const void* dout, const float* gate, const float* stats, float* dks,
                                      float* dvs, int32_t* err, cudaStream_t st);
// Local branch, query side, plus the compressed part from dqr and the RoPE
// backward: dq = R(c)^T (scale * sum_j dS_j k_j + dqr).
cudaError_t launch_local_bwd_dq(const Shape& s, int dtype, const int32_t* g2p, const void* qr, const void* kr,
                                const void* vl, const void* dout, const float* gate, const float* stats,
                                const float* dqr, void* dq, cudaStream_t st);
// Local branch, key side, with the RoPE backward: dk_loc = R(c)^T dKlr, dv_loc.
cudaError_t launch_local_bwd_dkv(const Shape& s, int dtype, const int32_t* g2p, const void* qr, const void* kr,
                                 const void* vl, const void* dout, const float* gate, const float* stats,
                                 void* dk, void* dv, cudaStream_t st);
// Local branch on tcgen05 tensor cores (k_local_bwd_tc.cu; shapes of
// local_attn_tc_supported): dqr += scale * dQ_loc, and the rotated-frame key
// gradients added to the float accumulators dk_acc, dv_acc [N,Hkv,64]
// (zeroed first); then the finalize kernel: dq = R(c)^T dqr,
// dk_loc = R(c)^T dk_acc, dv_loc = dv_acc in the operator's dtype.
cudaError_t launch_local_bwd_tc(const Shape& s, const int32_t* g2p, const void* qr, const void* kr, const void* vl,
                                const void* dout, const float* gate, const float* stats, float* dqr, float* dk_acc,
                                float* dv_acc, int32_t* err, cudaStream_t st);
cudaError_t launch_local_bwd_finalize(const Shape& s, int dtype, const int32_t* coords, const float* dqr,
                                      const float* dka, const float* dva, void* dq, void* dk, void* dv,
                                      cudaStream_t st);
// Summaries backward: dk_cmp, dv_cmp, dscores from dks, dvs.
cudaError_t launch_summaries_bwd(const Shape& s, int dtype, const int32_t* coords, const int32_t* members,
                                 const void* kc, const void* vc, const float* scores, const float* dks,
                                 const float* dvs, void* dkc, void* dvc, float* dsc, cudaStream_t st);

}  // namespace pack3d
