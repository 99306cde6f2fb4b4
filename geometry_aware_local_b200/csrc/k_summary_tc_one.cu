// The query x summary kernel with one 128-row query tile per CTA, two CTAs per
// SM (each with 256 tensor-memory columns and about 100 KiB of shared memory):
// an SM then runs two independent pipelines, so one CTA's set-up and
// epilogue overlap the other's main loop.  Its summaries come in tiles of 96
// so that two P buffers fit (S 96 + P 2 x 48 + O 64 columns): the
// exponentials of tile j are written while O += P v~ of tile j-1 still reads
// the other buffer (65k tokens: 0.807 -> 0.796 ms).  Same source as
// k_summary_tc.cu.
#define PACK3D_SA_GROUPS 1
#define PACK3D_SA_BN 96
#define PACK3D_SA_PBUFS 2
#define PACK3D_SA_NS sa_one
#include "k_summary_tc.cu"
