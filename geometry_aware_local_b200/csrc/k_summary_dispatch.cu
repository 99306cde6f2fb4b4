// Chooses between the two builds of the query x summary kernel.
//
// With few summary tiles per query tile, the fixed cost of a CTA (tensor-
// memory allocation, the first loads, the gate epilogue) is a large share of
// its time, and one-tile CTAs two per SM hide it behind each other; with many
// summary tiles the two-tile CTA, which reads every k~ / v~ tile once for both
// query tiles, is faster.  Measured on B200 (summary attention alone, forced
// builds, one process): M = 4,096 (65k tokens) 0.784 ms one-tile vs 0.831
// two-tile; M = 16,384 (262k) 10.69 vs 10.87-10.99, but 11.13 against 10.8 in
// a long run under the power cap; M = 32,768 44.71 vs 42.51; M = 65,536 (1M)
// 180.1 vs 170.3.  So the one-tile build runs up to 48 tiles of 128 summaries.
#include "common.cuh"
#include "internal.h"

namespace pack3d {
namespace sa_two {
long token_quantum(const Shape& s);
cudaError_t launch(const Shape& s, const void* qr, const void* ks, const void* vs, const float* oloc,
                   const float* gate, void* out, int32_t* err, cudaStream_t st, long tok_begin, long tok_end,
                   const Train* tr);
}  // namespace sa_two
namespace sa_one {
long token_quantum(const Shape& s);
cudaError_t launch(const Shape& s, const void* qr, const void* ks, const void* vs, const float* oloc,
                   const float* gate, void* out, int32_t* err, cudaStream_t st, long tok_begin, long tok_end,
                   const Train* tr);
}  // namespace sa_one

namespace {
constexpr int kOneTileMaxSummaries = 6144;
// s.sa_build forces a build (PACK3D_FLAG_SUMMARY_ONE_TILE / _TWO_TILE); 0 picks by size.
bool one_tile(const Shape& s) {
  if (s.sa_build != 0) return s.sa_build == 1;
  return s.M <= kOneTileMaxSummaries;
}
}  // namespace

long summary_attn_tc_token_quantum(const Shape& s) {
  return one_tile(s) ? sa_one::token_quantum(s) : sa_two::token_quantum(s);
}

cudaError_t launch_summary_attn_tc(const Shape& s, const void* qr, const void* ks, const void* vs,
                                   const float* oloc, const float* gate, void* out, int32_t* err,
                                   cudaStream_t st, long tok_begin, long tok_end, const Train* tr) {
  return one_tile(s) ? sa_one::launch(s, qr, ks, vs, oloc, gate, out, err, st, tok_begin, tok_end, tr)
                     : sa_two::launch(s, qr, ks, vs, oloc, gate, out, err, st, tok_begin, tok_end, tr);
}

}  // namespace pack3d
