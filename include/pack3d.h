/*
 * pack3d.h - C ABI of the B200 (sm_100a) implementation of the PACK3D
 * local-global attention forward pass and its backward (the training block),
 * from "Geometry Matters in Packed 3D Attention" (method section, Key designs
 * 1-3).
 *
 * The operator maps packed 3D tokens and their lattice coordinates to packed
 * outputs, A(X, c), in five stages:
 *   1. axial grid RoPE R(c_i) on Q and K, driven by true (z,y,x) coordinates
 *      (Key design 1, equation R(c));
 *   2. exact local attention over each token's clipped lattice box, found
 *      through a grid-to-packed index map (Key design 3);
 *   3. rotate-before-compress block summaries over contiguous blocks
 *      (Key design 2, equations k~_j^R and v~_j);
 *   4. every query against all M = N / |B| summaries with its own softmax
 *      (Key design 3);
 *   5. a per-token, per-head two-way softmax gate mixing both branches
 *      (overall framework).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named in the signatures are DEVICE pointers unless stated, owned
 *   by the caller.  The library never allocates, frees or keeps a pointer
 *   after a call returns.  Buffers must be contiguous and 16-byte aligned.
 * - Layouts (packed order = the caller's token order):
 *     coords   int32 [N,3]        (z, y, x), lattice indices from 0
 *     q        T     [N,Hq,d_h]   T = float or bf16 (config.dtype)
 *     k_loc, v_loc, k_cmp, v_cmp  T [N,Hkv,d_h]
 *     scores   float [N,Hkv]      per-token block scores (one per kv head)
 *     gate     float [N,Hq,2]     channel 0 weighs local, 1 compressed
 *     out      T     [N,Hq,d_h]
 *     g2p      int32 [Z*H*W]      g2p[(z*H+y)*W+x] = packed index of site
 *     members  int32 [M,|B|]      packed index of the t-th site (raster inside
 *                                 the block) of block j (raster over blocks)
 *     k_sum, v_sum T [M,Hkv,d_h]  block summaries
 *     o_loc    float [N,Hq,d_h]   local-branch output
 *   q head h reads kv head floor(h*Hkv/Hq).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream).  Errors that the host can see (bad config, null or
 *   misaligned pointer, too-small workspace) are returned before anything is
 *   launched.  Errors only the device can see (a coordinate out of range or
 *   repeated, a bounded wait that ran out) are OR-ed into the caller's
 *   device word `err_word` as PACK3D_DEVERR_* bits; pack3d_check_status()
 *   reads them back.  Kernels never trap.
 * - No entry point holds global mutable state; calls on different streams
 *   may run concurrently as long as their buffers do not overlap.
 * - Supported shapes: d_h == 64; Hq a multiple of Hkv with Hq/Hkv a power of
 *   two <= 8; 2*(m_z+m_y+m_x) <= 64; block dims dividing the lattice, block
 *   volume <= 64; lattice extents small enough that the per-axis cos/sin
 *   tables (Z*m_z + H*m_y + W*m_x entries) fit 96 KiB of shared memory;
 *   N < 2^24 (16,777,216 tokens).
 * - Empty volumes: a lattice with Z, H or W equal to 0 (N = 0) is valid.  Every
 *   entry point then returns PACK3D_OK at once, without reading any pointer
 *   (NULL is fine) or launching anything, and the workspace sizes are those
 *   of no token.
 */
#ifndef PACK3D_H
#define PACK3D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PACK3D_OK = 0,
    PACK3D_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, bad enum   */
    PACK3D_ERR_SHAPE = 2,           /* unsupported or inconsistent shape           */
    PACK3D_ERR_ALIGNMENT = 3,       /* pointer not 16-byte aligned                 */
    PACK3D_ERR_DTYPE = 4,           /* dtype not supported by this entry point     */
    PACK3D_ERR_NOT_PERMUTATION = 5, /* coords are not a bijection onto the lattice */
    PACK3D_ERR_WORKSPACE = 6,       /* workspace missing or too small              */
    PACK3D_ERR_CUDA = 7,            /* a CUDA runtime call failed                  */
    PACK3D_ERR_TIMEOUT = 8          /* a bounded device-side wait ran out          */
} pack3d_status;

typedef enum { PACK3D_F32 = 0, PACK3D_BF16 = 1 } pack3d_dtype;

/* Bits OR-ed into the caller's device error word. */
#define PACK3D_DEVERR_COORD_RANGE 0x1  /* a coordinate outside the lattice */
#define PACK3D_DEVERR_DUPLICATE   0x2  /* two tokens share one site        */
#define PACK3D_DEVERR_TIMEOUT     0x4  /* a pipeline wait gave up          */

/* config.flags */
#define PACK3D_FLAG_SIMT_SUMMARY  0x1  /* bf16: use the CUDA-core query x summary
                                          kernel instead of the tcgen05 one   */
#define PACK3D_FLAG_SIMT_LOCAL    0x2  /* bf16: use the CUDA-core local-attention
                                          kernel instead of the tcgen05 one   */
/* The summary-centre variant ("Geometry Matters in Packed 3D Attention",
 * contribution 2 and "Future Directions" 3: the cheaper approximation that
 * rotates only at the summary centre): k~_j = R(cbar_j) sum_u a_{j,u} k_u with
 * cbar_j the block's geometric centre, block origin + ((bz-1)/2, (by-1)/2,
 * (bx-1)/2), a fractional coordinate; v~_j and every other stage unchanged.
 * Without the flag the summaries are the exact rotate-before-compress form. */
#define PACK3D_FLAG_SUMMARY_CENTER 0x4
/* Diagnostic: every tensor-core kernel withholds one step of its pipeline
 * (the query x summary kernels the load of their last summary tile, the
 * local-attention kernel the score MMA of its last key plane), so that the
 * waits that depend on it run out after wait_limit_us.  The call then reports
 * PACK3D_DEVERR_TIMEOUT in err_word (PACK3D_ERR_TIMEOUT from
 * pack3d_check_status) and its outputs are unspecified; the kernels still let
 * their issued loads and MMAs complete, free their tensor memory and return,
 * so the next call on the stream runs normally.  It exists to test that error
 * path; nothing else sets it.  No entry point that takes it runs on CUDA cores
 * only (float, PACK3D_FLAG_SIMT_*): those have no pipeline waits. */
#define PACK3D_FLAG_DIAG_STALL    0x8
/* The tensor-core query x summary kernel comes in two builds: one 128-row query
 * tile per CTA with two CTAs per SM (summaries in tiles of 96, two P buffers),
 * and two tiles per CTA with one CTA per SM (every tile of 128 summaries read
 * once for both).  By default the library picks the one-tile build up to
 * M <= 6,144 summaries and the two-tile build above; these flags force one of
 * them (setting both is an error).  Both builds form the same products in the
 * same order and group the softmax row sums differently, so their outputs
 * agree to float rounding; the flags only move the cost. */
#define PACK3D_FLAG_SUMMARY_ONE_TILE 0x10
#define PACK3D_FLAG_SUMMARY_TWO_TILE 0x20

typedef struct {
    int32_t Z, H, W;          /* lattice extents; N = Z*H*W tokens               */
    int32_t Hq, Hkv, d_h;     /* query heads, key/value heads, head dim (64)     */
    int32_t m_z, m_y, m_x;    /* rotary planes per axis (11, 11, 10 for d_h=64)  */
    int32_t reserved0;        /* must be 0                                       */
    double  rope_base;        /* omega_{a,r} = rope_base^(-r/m_a) (10000)        */
    int32_t bz, by, bx;       /* summary block dims (1, 4, 4); divide Z, H, W    */
    int32_t rz, ry, rx;       /* local window radii (1, 3, 3) = 3x7x7 box       */
    float   softmax_scale;    /* logit scale in both branches (1/sqrt(d_h))      */
    int32_t dtype;            /* pack3d_dtype of q, k, v, summaries, out         */
    int32_t flags;            /* PACK3D_FLAG_* bits                              */
    int32_t wait_limit_us;    /* limit of every bounded device-side pipeline wait,
                                 in microseconds, >= 0; 0 = the default of 2 s.
                                 A wait that runs out makes its CTA give up
                                 (PACK3D_DEVERR_TIMEOUT); a limit far below a
                                 kernel's normal step time turns healthy calls
                                 into timeouts                                  */
    double  coord_scale[3];   /* per-axis coordinate scale (z, y, x), > 0, 1 by
                                 default: the rotation angle of axis a is
                                 omega_{a,r} * coord_scale[a] * c_a, so e.g.
                                 1/(extent-1) gives normalised coordinates in
                                 [0, 1] and coord_scale[0] != 1 rescales z (the
                                 rotary-configuration sweep of the summary page,
                                 "Main Findings")                                */
    int32_t origin[3];        /* lattice origin (z, y, x) in the frame the rotation
                                 uses, 0 by default: the lattice covers sites
                                 origin + [0,Z) x [0,H) x [0,W), coords stay local
                                 (from 0), and every rotation angle is
                                 omega_{a,r} * coord_scale[a] * (origin[a] + c_a).
                                 A sub-volume (a z-slab of a larger lattice) then
                                 rotates by its sites' true coordinates, as Key
                                 design 1 requires; the local branch does not
                                 depend on it (relative positions only)           */
    int32_t reserved2;        /* must be 0                                       */
} pack3d_config;

/* Fills cfg with the pages' defaults for a Z x H x W lattice: Hq=8, Hkv=2,
 * d_h=64, m=(11,11,10), base 1e4, blocks 1x4x4, window 3x7x7, scale 1/8,
 * bf16. */
void pack3d_default_config(pack3d_config *cfg, int32_t Z, int32_t H, int32_t W);

/* Checks a config without touching the device.  Returns PACK3D_OK or the
 * reason it cannot be run. */
pack3d_status pack3d_validate_config(const pack3d_config *cfg);

/* Bytes of device workspace pack3d_forward needs (0 on an invalid config):
 * g2p, members, rotated Q and K_loc, the summaries and the float o_loc, each
 * region at a 1 KiB offset. */
size_t pack3d_workspace_bytes(const pack3d_config *cfg);

/* Stage 0 - grid-to-packed index map and block membership.
 * Cites: Key design 1 (coordinate-preserving packings are bijections onto the
 * lattice) and Key design 2 (contiguous blocks B_j).
 * In: coords [N,3].  Out: g2p [Z*H*W], members [M,|B|].  A coordinate outside
 * the lattice sets PACK3D_DEVERR_COORD_RANGE, two tokens on one site set
 * PACK3D_DEVERR_DUPLICATE (err_word required); g2p/members are then
 * unspecified. */
pack3d_status pack3d_build_index(const pack3d_config *cfg, const int32_t *coords,
                                 int32_t *g2p, int32_t *members, int32_t *err_word,
                                 void *stream);

/* Stage 1 - axial grid RoPE: y[i,h,:] = R(c_i) x[i,h,:] for `heads` heads per
 * token.  Cites: Key design 1, equation R(c): planes (2p, 2p+1), z planes
 * first, then y, then x, angle omega_{a,r} * c_a; dims past 2(m_z+m_y+m_x)
 * copied.  x, y: T [N,heads,d_h]; y may equal x (in place). */
pack3d_status pack3d_rope(const pack3d_config *cfg, const int32_t *coords, const void *x,
                          void *y, int32_t heads, void *stream);

/* Stage 1 for both rotated tensors in one launch (the form pack3d_forward
 * uses): q_rot = R(c) q with Hq heads and k_rot = R(c) k_loc with Hkv heads,
 * each exactly as pack3d_rope would compute it.  q, q_rot: T [N,Hq,d_h];
 * k, k_rot: T [N,Hkv,d_h]; each output may equal its input.  Device pointers,
 * 16-byte aligned, owned by the caller; errors as pack3d_rope. */
pack3d_status pack3d_rope_qk(const pack3d_config *cfg, const int32_t *coords, const void *q,
                             void *q_rot, const void *k, void *k_rot, void *stream);

/* Stage 3 - rotate-before-compress summaries.  For block j and kv head g:
 *   a_{j,u} = softmax over u in B_j of scores[u,g]
 *   k_sum[j,g] = sum_u a_{j,u} R(c_u) k_cmp[u,g],  v_sum[j,g] = sum_u a_{j,u} v_cmp[u,g]
 * Cites: Key design 2, equations k~_j^R and v~_j.  k_cmp is NOT rotated by the
 * caller: the rotation is applied here, before pooling.  members must come
 * from pack3d_build_index on a valid coordinate set (member t of block j sits
 * at the t-th raster site of the block). */
pack3d_status pack3d_build_summaries(const pack3d_config *cfg, const int32_t *members,
                                     const void *k_cmp, const void *v_cmp,
                                     const float *scores, void *k_sum, void *v_sum,
                                     void *stream);

/* Stage 2 - exact local attention.  For token i at (z,y,x) and q head h:
 *   o_loc[i,h] = sum_{j in N(i)} softmax_j(scale <q_rot[i,h], k_rot[j,g]>) v_loc[j,g]
 * with N(i) the tokens whose sites lie in the box |dz|<=rz, |dy|<=ry,
 * |dx|<=rx clipped at the volume (self included).  Cites: Key design 3 and
 * the summary's "local attention stays exact" contract.  q_rot, k_rot are
 * RoPE'd (stage 1); neighbours are reached through g2p, so any packing gives
 * the same result and no gathered neighbour tensor is formed.  bf16 with
 * Hq/Hkv = 4, rz = 1, ry <= 3, rx <= 3 runs on tcgen05 tensor cores (float
 * accumulation); every other shape on CUDA cores in float.  err_word
 * (nullable) receives PACK3D_DEVERR_TIMEOUT if a pipeline wait gives up. */
pack3d_status pack3d_local_attn(const pack3d_config *cfg, const int32_t *g2p,
                                const void *q_rot, const void *k_rot, const void *v_loc,
                                float *o_loc, int32_t *err_word, void *stream);

/* Stages 4+5 - every query against all M summaries, then the gate.
 *   o_cmp[i,h] = sum_j softmax_j(scale <q_rot[i,h], k_sum[j,g]>) v_sum[j,g]
 * streamed with an online softmax (no [N,M] tensor).  If gate is NULL, out =
 * o_cmp.  Otherwise (gamma0,gamma1) = softmax(gate[i,h,0], gate[i,h,1]) and
 * out = gamma0 o_loc + gamma1 o_cmp (o_loc required).  Cites: Key design 3
 * (query-summary branch) and the overall framework's tokenwise gate.
 * bf16 runs on tcgen05 tensor cores with float accumulation; float runs on
 * CUDA cores in float.  err_word (nullable) receives PACK3D_DEVERR_TIMEOUT if
 * a pipeline wait gives up. */
pack3d_status pack3d_summary_attn(const pack3d_config *cfg, const void *q_rot,
                                  const void *k_sum, const void *v_sum, const float *o_loc,
                                  const float *gate, void *out, int32_t *err_word,
                                  void *stream);

/* Stages 4+5 for an explicit number of query rows and summaries: as
 * pack3d_summary_attn, but q_rot, o_loc, gate and out hold `tokens` tokens
 * (T [tokens,Hq,d_h], float [tokens,Hq,d_h], float [tokens,Hq,2]) and k_sum,
 * v_sum hold `summaries` summaries (T [summaries,Hkv,d_h]), instead of the N and
 * M = N / |B| of the config's lattice (the config supplies the heads, the
 * scale, the dtype and the flags).  This is the form a part of a volume uses
 * when it attends to the summaries of the whole volume, e.g. one z-slab of a
 * volume split over several GPUs, against the all-gathered summaries (every
 * query still sees all M summaries, Key design 3).  tokens, summaries >= 0;
 * tokens == 0 or summaries == 0 returns PACK3D_OK at once (no summary: out is
 * not written).  Errors as pack3d_summary_attn; a count that is too large for
 * 32-bit element indices -> PACK3D_ERR_SHAPE. */
pack3d_status pack3d_summary_attn_rows(const pack3d_config *cfg, int64_t tokens, int64_t summaries,
                                       const void *q_rot, const void *k_sum, const void *v_sum,
                                       const float *o_loc, const float *gate, void *out,
                                       int32_t *err_word, void *stream);

/* Row gather for the z-slab split of one volume over several ranks (the
 * summary page and papernotes.org Key design 3: a query's local window reaches
 * r_z planes into the neighbouring slab, so each rank sends the local keys and
 * values of its boundary planes, found through its grid-to-packed map):
 *   dst row i = src row idx[i]   for 0 <= i < n,
 * rows of row_bytes bytes (a positive multiple of 16), idx[i] < 0 giving a
 * zero row.  idx (int32, n entries), src and dst are device pointers owned by
 * the caller; src and dst 16-byte aligned; every idx[i] must be a row of src
 * (not checked on the device).  n == 0 returns PACK3D_OK with nothing
 * launched.  Errors: null pointer, n < 0, or row_bytes not a positive multiple
 * of 16 or above 16 x (2^31 - 1) -> PACK3D_ERR_INVALID_ARG; misaligned src or dst ->
 * PACK3D_ERR_ALIGNMENT; a failed launch -> PACK3D_ERR_CUDA. */
pack3d_status pack3d_gather_rows(const int32_t *idx, int64_t n, const void *src, void *dst,
                                 int64_t row_bytes, void *stream);

/* Diagnostic: evaluates the FMA-pipe exponential that the one-tile build of
 * the query x summary kernel uses for 2 of every 16 pairs of its softmax
 * exponentials (Key design 3's softmax over the summaries): y[i] = 2^x[i]
 * from x = n + f, n = rint(x) put into the float's exponent, 2^f by a cubic
 * minimax fit (Remez exchange, relative error <= 7.5e-5 on [-1/2, 1/2]);
 * x is clamped at -125, so the result of a very negative x is ~2.4e-38
 * rather than 0.  x and y are device float arrays of n elements (caller
 * owned).  n == 0 -> PACK3D_OK; n < 0 or a null pointer ->
 * PACK3D_ERR_INVALID_ARG; a failed launch -> PACK3D_ERR_CUDA. */
pack3d_status pack3d_exp2_fma_eval(const float *x, float *y, int64_t n, void *stream);

/* The whole forward pass: index map, summaries, RoPE on Q and K_loc, local
 * branch, query-summary branch with the gate, all stream-ordered on `stream`:
 * the pass starts after the work already on `stream` and later work on it
 * sees every output.  Inside, RoPE runs on a library-owned side stream
 * concurrently with the index map and the summaries (one non-blocking stream
 * and two events per device, made on the device's first call and kept until
 * the process exits; calls from several host threads take turns on them).
 * While `stream` is being captured into a graph, every launch stays on it.
 * workspace: device buffer of at least pack3d_workspace_bytes(cfg) bytes,
 * 256-byte aligned; its contents on entry do not matter.  err_word: device int32
 * the caller zeroed before its first use (required). */
pack3d_status pack3d_forward(const pack3d_config *cfg, const int32_t *coords, const void *q,
                             const void *k_loc, const void *v_loc, const void *k_cmp,
                             const void *v_cmp, const float *scores, const float *gate,
                             void *out, void *workspace, size_t workspace_bytes,
                             int32_t *err_word, void *stream);

/* Size of the scratch array compiled into the library for
 * pack3d_forward_noalloc (32 MiB; held on every GPU that loads the library
 * until the process exits). */
#define PACK3D_NOALLOC_SCRATCH_BYTES (32u << 20)

/* pack3d_forward without a workspace, for callers that cannot allocate device
 * memory: a plugin whose host application owns every allocation and passes in
 * only input and output buffers, or a path where cudaMalloc is not allowed
 * because it may synchronise the device.  The paper has no counterpart; this
 * is a deployment convenience.  Same arguments, results and error behaviour as
 * pack3d_forward, except:
 *   - the scratch comes from a fixed array inside the library of
 *     PACK3D_NOALLOC_SCRATCH_BYTES bytes; a config whose workspace
 *     (pack3d_workspace_bytes) exceeds it is rejected with
 *     PACK3D_ERR_WORKSPACE before anything is launched (about 9,900 bf16
 *     tokens at Hq=8, Hkv=2);
 *   - err_word may be NULL, in which case device-detected errors are not
 *     reported;
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it: make
 *     that first call before any stream capture.  The cache belongs to the
 *     device's context: after cudaDeviceReset the library may load at another
 *     address, so do not call this entry point on a device that was reset;
 *   - every call shares the one array, so calls whose work overlaps on the
 *     GPU (e.g. on two streams) race; the caller must serialise them.
 * Nothing is allocated or freed. */
pack3d_status pack3d_forward_noalloc(const pack3d_config *cfg, const int32_t *coords,
                                     const void *q, const void *k_loc, const void *v_loc,
                                     const void *k_cmp, const void *v_cmp, const float *scores,
                                     const float *gate, void *out, int32_t *err_word,
                                     void *stream);

/* ---- forward pass from host buffers ------------------------------------------
 * Not part of the paper's method: a deployment entry point that copies the
 * inputs in, runs the forward pass and copies the output back, with the
 * copies overlapped with the stages that do not read them. */

/* Largest number of row chunks pack3d_forward_host splits the query x summary
 * stage into (each chunk's output goes back while the next one computes). */
#define PACK3D_HOST_MAX_CHUNKS 8

/* Opaque: the two copy streams and the events of pack3d_forward_host, bound to
 * the device current at creation.  Created and destroyed by the caller; one
 * pipeline must not be used by two calls at the same time. */
typedef struct pack3d_pipeline pack3d_pipeline;
pack3d_status pack3d_pipeline_create(pack3d_pipeline **pipeline);
void pack3d_pipeline_destroy(pack3d_pipeline *pipeline);

/* Bytes of device workspace pack3d_forward_host needs: the pack3d_forward
 * workspace plus device copies of every input and of the output (0 on an
 * invalid config). */
size_t pack3d_host_workspace_bytes(const pack3d_config *cfg);

/* pack3d_forward from HOST buffers: coords, q, k_loc, v_loc, k_cmp, v_cmp,
 * scores, gate and out are host pointers with the layouts of pack3d_forward
 * (page-locked memory makes the copies asynchronous; pageable memory works but
 * the copies then block the host).  The inputs are copied, in the order the
 * stages read them, on the pipeline's first copy stream; each stage runs on
 * `stream` as soon as its own inputs have arrived; the query x summary stage
 * runs in up to PACK3D_HOST_MAX_CHUNKS token chunks whose outputs are copied
 * back on the second copy stream while the next chunk computes.  All the work
 * joins `stream` before the call's work ends there: the output is in `out`
 * once `stream` is synchronised (pack3d_check_status does that).  workspace:
 * device, 256-byte aligned, at least pack3d_host_workspace_bytes(cfg) bytes,
 * not touched by other work until `stream` is synchronised.  err_word:
 * device int32, as pack3d_forward.  Errors: as pack3d_forward; a pipeline made
 * on another device -> PACK3D_ERR_INVALID_ARG. */
pack3d_status pack3d_forward_host(pack3d_pipeline *pipeline, const pack3d_config *cfg,
                                  const int32_t *coords, const void *q, const void *k_loc,
                                  const void *v_loc, const void *k_cmp, const void *v_cmp,
                                  const float *scores, const float *gate, void *out,
                                  void *workspace, size_t workspace_bytes, int32_t *err_word,
                                  void *stream);

/* ---- training block: forward and backward in one call ------------------------
 * The pages call the operator a fused forward/backward training block; this
 * call runs the forward pass and then the gradients of L = <dout, out> with
 * respect to every input, by the chain rule through the stages in reverse:
 *   gate:       dgate = gamma (dgamma - <gamma, dgamma>), dgamma_c = <dout, o_c>
 *   branches:   for each softmax row, dl_j = P_j (<do, v_j> - <do, o>) with
 *               do = gamma0 dout (local) or gamma1 dout (compressed);
 *               dq += scale sum_j dl_j k_j, dk_j += scale dl_j q, dv_j += P_j do
 *   summaries:  dk_cmp[u] = R(c_u)^T (a_u dk_sum[j]), dv_cmp[u] = a_u dv_sum[j],
 *               dscores[u] = a_u (da_u - sum_u' a_u' da_u'),
 *               da_u = <dk_sum[j], R(c_u) k_cmp[u]> + <dv_sum[j], v_cmp[u]>
 *   RoPE:       dq = R(c)^T dq_rot, dk_loc = R(c)^T dk_rot (Key design 1).
 * The forward saves per (token, q head) row the log-sum-exp of both softmaxes
 * and the deltas <do, o> (the query x summary epilogue forms them together
 * with dgate); the backward recomputes P from them.  Float accumulation
 * throughout; the summary-side gradients of the compressed branch (and, on
 * the tensor-core local path, the local key and value gradients) are summed
 * with float atomics, so their last bits may vary from run to run. */

/* Bytes of device workspace pack3d_forward_backward needs: the pack3d_forward
 * workspace, then row statistics float [N,Hq,4], the float query gradient
 * [N,Hq,d_h], float dk_sum, dv_sum [M,Hkv,d_h] and float local key / value
 * gradient accumulators [N,Hkv,d_h] (0 on an invalid config). */
size_t pack3d_train_workspace_bytes(const pack3d_config *cfg);

/* Forward pass and all input gradients.  Inputs as for pack3d_forward plus
 * dout (T [N,Hq,d_h], the gradient of the loss with respect to out).
 * Outputs (all required, device, 16-byte aligned): out (T [N,Hq,d_h]), dq
 * (T [N,Hq,d_h]), dk_loc, dv_loc, dk_cmp, dv_cmp (T [N,Hkv,d_h]), dscores
 * (float [N,Hkv]) and dgate (float [N,Hq,2]), in packed order.  workspace: at
 * least pack3d_train_workspace_bytes(cfg) bytes, 256-byte aligned.  With
 * PACK3D_FLAG_SUMMARY_CENTER the forward and the summaries' backward follow
 * the summary-centre variant (the pooled key rotated once by R(cbar_j)):
 * dk_cmp[u] = a_u R(cbar_j)^T dk_sum[j] and
 * da_u = <R(cbar_j)^T dk_sum[j], k_cmp[u]> + <dv_sum[j], v_cmp[u]>. */
pack3d_status pack3d_forward_backward(const pack3d_config *cfg, const int32_t *coords, const void *q,
                                      const void *k_loc, const void *v_loc, const void *k_cmp,
                                      const void *v_cmp, const float *scores, const float *gate,
                                      const void *dout, void *out, void *dq, void *dk_loc,
                                      void *dv_loc, void *dk_cmp, void *dv_cmp, float *dscores,
                                      float *dgate, void *workspace, size_t workspace_bytes,
                                      int32_t *err_word, void *stream);

/* Synchronises `stream`, reads the device error word, resets it to 0 and maps
 * it: COORD_RANGE/DUPLICATE -> PACK3D_ERR_NOT_PERMUTATION, TIMEOUT ->
 * PACK3D_ERR_TIMEOUT, none -> PACK3D_OK.  A failed CUDA call -> PACK3D_ERR_CUDA. */
pack3d_status pack3d_check_status(int32_t *err_word, void *stream);

/* Static text for a status code. */
const char *pack3d_status_string(pack3d_status s);

/* Static text naming the compiled architecture and kernel paths. */
const char *pack3d_backend_info(void);

#ifdef __cplusplus
}
#endif

#endif /* PACK3D_H */
