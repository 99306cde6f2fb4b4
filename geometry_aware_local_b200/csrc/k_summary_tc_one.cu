// The query x summary kernel with one 128-row query tile per CTA, two CTAs per
// SM (each with 256 tensor-memory columns and about 100 KiB of shared memory):
// an SM then runs two independent pipelines, so one CTA's set-up and
// epilogue overlap the other's main loop.  Its summaries come in tiles of 96
// so that two P buffers fit (S 96 + P 2 x 48 + O 64 columns): the
// exponentials of tile j are written while O += P v~ of tile j-1 still reads
// the other buffer (65k tokens: 0.807 -> 0.796 ms).  2 of every 16 pairs of
// exponentials run on the FMA pipe (exp2_fma), which unloads MUFU (65k:
// 0.769 -> 0.750 ms; the two-tile build at 262k is 6.8 % slower with it, so it
// keeps MUFU for all).  Same source as k_summary_tc.cu.
#define PACK3D_SA_GROUPS 1
#define PACK3D_SA_BN 96
#define PACK3D_SA_PBUFS 2
#define PACK3D_SA_POLY 2
#define PACK3D_SA_NS sa_one
#include "k_summary_tc.cu"
