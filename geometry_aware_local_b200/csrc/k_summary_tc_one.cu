// The query x summary kernel with one 128-row query tile per CTA, two CTAs per
// SM (each with 256 tensor-memory columns and about 100 KiB of shared memory):
// an SM then runs two independent pipelines, so one CTA's set-up and
// epilogue overlap the other's main loop.  Same source as k_summary_tc.cu.
#define PACK3D_SA_GROUPS 1
#define PACK3D_SA_NS sa_one
#include "k_summary_tc.cu"
