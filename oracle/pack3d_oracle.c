/*
 * PACK3D oracle: a plain, slow, float64 CPU statement of what the operator
 * computes, written from "Geometry Matters in Packed 3D Attention".
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or table with the CUDA
 * library; it reads plain float64 arrays and writes plain float64 arrays.
 *
 * Every function follows one passage of the pages:
 *   - lattice / index map ........ method "Key design 1" (coordinate-preserving
 *                                  permutations) and "Key design 2" (blocks);
 *                                  the summary's "Methodology in Plain English"
 *                                  (a packing is a bijection onto the lattice).
 *   - axial RoPE ................. "Key design 1", equation R(c).
 *   - summaries .................. "Key design 2", equations k~_j^R and v~_j.
 *   - summary-centre variant ..... the summary's "What This Paper Is About"
 *                                  (contribution 2) and "Future Directions" 3:
 *                                  the cheaper variant that rotates the pooled
 *                                  key by the block centre only.
 *   - local branch ............... "Key design 3" (neighbourhood N(i)); summary
 *                                  "local attention stays exact".
 *   - compressed branch .......... "Key design 3" / summary "every token attends
 *                                  to all M summaries".
 *   - gate ....................... "overall framework" (tokenwise learned gate).
 *   - backward pass .............. the summary's description of the operator as
 *                                  a fused forward/backward training block: the
 *                                  gradients of <dout, out> by the chain rule
 *                                  through the stages above, in reverse order.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *   omega_{a,r} = base^(-r/m_a); rotary pair p occupies dims (2p, 2p+1); pairs
 *   are ordered z, then y, then x; dims past 2(m_z+m_y+m_x) are untouched;
 *   the rotation maps (x0,x1) to (x0 cos t - x1 sin t, x0 sin t + x1 cos t);
 *   the window is an axis-aligned box of radii (rz,ry,rx) clipped at the
 *   volume boundary with the query itself included; block scores are one per
 *   token and kv head; q head h reads kv head floor(h*Hkv/Hq); gate channel 0
 *   weighs the local branch and channel 1 the compressed one; summaries are
 *   numbered in raster order over the block grid and block members in raster
 *   order inside a block.  The frequency values and pair layout are fixed by
 *   that convention only (no identity on the pages distinguishes them).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -o liborc.so pack3d_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t Z, H, W;
    int32_t Hq, Hkv, dh;
    int32_t mz, my, mx;
    double base;
    int32_t bz, by, bx;
    int32_t rz, ry, rx;
    double scale;
    double cscale[3];   /* coordinate scale per axis: angle = omega * cscale[a] * c_a */
    double origin[3];   /* lattice origin: the true coordinate of local site c is origin + c */
} orc_cfg;

/* ---- lattice and index map ------------------------------------------- */

/* Checks that coords is a bijection onto [0,Z)x[0,H)x[0,W) and builds
 * g2p[(z*H+y)*W+x] = packed index and members[j*v + t] = packed index of the
 * t-th site (raster inside the block) of block j (raster over the block grid).
 * Returns 0 on success, 1 if a coordinate is out of range, 2 on a duplicate. */
int orc_build_index(const orc_cfg *c, const int32_t *coords, int32_t *g2p, int32_t *members)
{
    long N = (long)c->Z * c->H * c->W;
    for (long s = 0; s < N; ++s) g2p[s] = -1;
    for (long i = 0; i < N; ++i) {
        int z = coords[3 * i], y = coords[3 * i + 1], x = coords[3 * i + 2];
        if (z < 0 || z >= c->Z || y < 0 || y >= c->H || x < 0 || x >= c->W) return 1;
        long s = ((long)z * c->H + y) * c->W + x;
        if (g2p[s] != -1) return 2;
        g2p[s] = (int32_t)i;
    }
    /* N distinct in-range sites for N tokens: every site is filled. */
    int nby = c->H / c->by, nbx = c->W / c->bx;
    int v = c->bz * c->by * c->bx;
    for (int z = 0; z < c->Z; ++z)
        for (int y = 0; y < c->H; ++y)
            for (int x = 0; x < c->W; ++x) {
                long j = ((long)(z / c->bz) * nby + y / c->by) * nbx + x / c->bx;
                int t = ((z % c->bz) * c->by + y % c->by) * c->bx + x % c->bx;
                members[j * v + t] = g2p[((long)z * c->H + y) * c->W + x];
            }
    return 0;
}

/* ---- axial grid RoPE, equation R(c) ------------------------------------ */

/* Angle of rotary pair p for coordinate (z,y,x) (a lattice site, or the
 * fractional centre of a block); returns 0 for untouched dims through
 * *active = 0.  R(c) is driven by the site's true coordinate (Key design 1):
 * for a lattice that is part of a larger volume, its origin plus the local
 * coordinate. */
static double pair_angle(const orc_cfg *c, int p, double z, double y, double x, int *active)
{
    int axis_pairs[3] = {c->mz, c->my, c->mx};
    double coord[3] = {z, y, x};
    int first = 0;
    for (int a = 0; a < 3; ++a) {
        if (p < first + axis_pairs[a]) {
            int r = p - first;
            double omega = pow(c->base, -(double)r / (double)axis_pairs[a]);
            *active = 1;
            return omega * (c->cscale[a] * (c->origin[a] + coord[a]));
        }
        first += axis_pairs[a];
    }
    *active = 0;
    return 0.0;
}

/* y = R(c) x for one head vector of d_h values at coordinate (cz,cy,cx). */
static void rotate_row(const orc_cfg *c, double cz, double cy, double cx, const double *xi, double *yi)
{
    for (int p = 0; p < c->dh / 2; ++p) {
        int active;
        double t = pair_angle(c, p, cz, cy, cx, &active);
        double x0 = xi[2 * p], x1 = xi[2 * p + 1];
        if (active) {
            yi[2 * p] = x0 * cos(t) - x1 * sin(t);
            yi[2 * p + 1] = x0 * sin(t) + x1 * cos(t);
        } else {
            yi[2 * p] = x0;
            yi[2 * p + 1] = x1;
        }
    }
}

/* y[i,h,:] = R(c_i) x[i,h,:] for n tokens with `heads` heads each. */
void orc_rotate(const orc_cfg *c, const int32_t *coords, const double *x, double *y,
                int heads, long n)
{
    int d = c->dh;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i)
        for (int h = 0; h < heads; ++h)
            rotate_row(c, coords[3 * i], coords[3 * i + 1], coords[3 * i + 2],
                       x + ((long)i * heads + h) * d, y + ((long)i * heads + h) * d);
}

/* ---- rotate-before-compress block summaries, equations k~_j^R, v~_j ---- */

/* For every block j and kv head g:
 *   a_{j,u} = exp(s_{u,g}) / sum_{u' in B_j} exp(s_{u',g})
 *   ksum[j,g] = sum_u a_{j,u} R(c_u) kcmp[u,g]
 *   vsum[j,g] = sum_u a_{j,u} vcmp[u,g]
 * The softmax is evaluated with its maximum subtracted (same value). */
void orc_summaries(const orc_cfg *c, const int32_t *coords, const int32_t *members,
                   const double *kcmp, const double *vcmp, const double *scores,
                   double *ksum, double *vsum)
{
    long N = (long)c->Z * c->H * c->W;
    int v = c->bz * c->by * c->bx;
    long M = N / v;
    int d = c->dh, Hkv = c->Hkv;
#pragma omp parallel for schedule(static)
    for (long j = 0; j < M; ++j) {
        double *a = (double *)malloc(sizeof(double) * v);
        double *kr = (double *)malloc(sizeof(double) * d);
        for (int g = 0; g < Hkv; ++g) {
            double smax = -INFINITY, den = 0.0;
            for (int t = 0; t < v; ++t) {
                double s = scores[(long)members[j * v + t] * Hkv + g];
                if (s > smax) smax = s;
            }
            for (int t = 0; t < v; ++t) {
                a[t] = exp(scores[(long)members[j * v + t] * Hkv + g] - smax);
                den += a[t];
            }
            for (int t = 0; t < v; ++t) a[t] /= den;
            double *ks = ksum + (j * Hkv + g) * d;
            double *vs = vsum + (j * Hkv + g) * d;
            for (int e = 0; e < d; ++e) { ks[e] = 0.0; vs[e] = 0.0; }
            for (int t = 0; t < v; ++t) {
                long u = members[j * v + t];
                rotate_row(c, coords[3 * u], coords[3 * u + 1], coords[3 * u + 2],
                           kcmp + (u * Hkv + g) * d, kr);
                for (int e = 0; e < d; ++e) {
                    ks[e] += a[t] * kr[e];
                    vs[e] += a[t] * vcmp[(u * Hkv + g) * d + e];
                }
            }
        }
        free(a);
        free(kr);
    }
}

/* ---- exact local branch ------------------------------------------------ */

/* The summary-centre variant: the same block weights a_{j,u}, the pooled
 * key left unrotated and then rotated once by the block's geometric centre,
 *   k~_j = R(cbar_j) sum_u a_{j,u} k_u,
 *   cbar_j = block origin + ((bz-1)/2, (by-1)/2, (bx-1)/2)
 * (a fractional coordinate); v~_j as in orc_summaries. */
void orc_summaries_center(const orc_cfg *c, const int32_t *members, const double *kcmp,
                          const double *vcmp, const double *scores, double *ksum, double *vsum)
{
    long N = (long)c->Z * c->H * c->W;
    int v = c->bz * c->by * c->bx;
    long M = N / v;
    int nby = c->H / c->by, nbx = c->W / c->bx;
    int d = c->dh, Hkv = c->Hkv;
#pragma omp parallel for schedule(static)
    for (long j = 0; j < M; ++j) {
        double *a = (double *)malloc(sizeof(double) * v);
        double *kp = (double *)malloc(sizeof(double) * d);
        long jx = j % nbx, jy = (j / nbx) % nby, jz = j / ((long)nbx * nby);
        double cz = jz * c->bz + 0.5 * (c->bz - 1);
        double cy = jy * c->by + 0.5 * (c->by - 1);
        double cx = jx * c->bx + 0.5 * (c->bx - 1);
        for (int g = 0; g < Hkv; ++g) {
            double smax = -INFINITY, den = 0.0;
            for (int t = 0; t < v; ++t) {
                double s = scores[(long)members[j * v + t] * Hkv + g];
                if (s > smax) smax = s;
            }
            for (int t = 0; t < v; ++t) {
                a[t] = exp(scores[(long)members[j * v + t] * Hkv + g] - smax);
                den += a[t];
            }
            for (int t = 0; t < v; ++t) a[t] /= den;
            double *vs = vsum + (j * Hkv + g) * d;
            for (int e = 0; e < d; ++e) { kp[e] = 0.0; vs[e] = 0.0; }
            for (int t = 0; t < v; ++t) {
                long u = members[j * v + t];
                for (int e = 0; e < d; ++e) {
                    kp[e] += a[t] * kcmp[(u * Hkv + g) * d + e];
                    vs[e] += a[t] * vcmp[(u * Hkv + g) * d + e];
                }
            }
            rotate_row(c, cz, cy, cx, kp, ksum + (j * Hkv + g) * d);
        }
        free(a);
        free(kp);
    }
}

/* For each sampled packed row i = rows[r] and q head h, with g = kv head of h:
 *   N(i) = tokens at lattice sites within the clipped box of radii (rz,ry,rx)
 *   l_j  = scale * <qr[r,h], klr[j,g]>,  o[r,h] = sum_j softmax(l)_j vloc[j,g].
 * qr holds the rotated queries of the sampled rows only, in sample order. */
void orc_local_attn(const orc_cfg *c, const int32_t *coords, const int32_t *g2p,
                    const double *qr, const double *klr, const double *vloc,
                    const int64_t *rows, long nrows, double *oloc)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
    long wmax = (long)(2 * c->rz + 1) * (2 * c->ry + 1) * (2 * c->rx + 1);
#pragma omp parallel for schedule(dynamic, 16)
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        int zi = coords[3 * i], yi = coords[3 * i + 1], xi = coords[3 * i + 2];
        long *nb = (long *)malloc(sizeof(long) * wmax);
        double *l = (double *)malloc(sizeof(double) * wmax);
        long cnt = 0;
        for (int z = zi - c->rz; z <= zi + c->rz; ++z)
            for (int y = yi - c->ry; y <= yi + c->ry; ++y)
                for (int x = xi - c->rx; x <= xi + c->rx; ++x) {
                    if (z < 0 || z >= c->Z || y < 0 || y >= c->H || x < 0 || x >= c->W) continue;
                    nb[cnt++] = g2p[((long)z * c->H + y) * c->W + x];
                }
        for (int h = 0; h < Hq; ++h) {
            int g = (int)(((long)h * Hkv) / Hq);
            const double *q = qr + (r * Hq + h) * d;
            double lmax = -INFINITY, den = 0.0;
            for (long k = 0; k < cnt; ++k) {
                const double *kk = klr + (nb[k] * Hkv + g) * d;
                double s = 0.0;
                for (int e = 0; e < d; ++e) s += q[e] * kk[e];
                l[k] = c->scale * s;
                if (l[k] > lmax) lmax = l[k];
            }
            double *o = oloc + (r * Hq + h) * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (long k = 0; k < cnt; ++k) {
                double p = exp(l[k] - lmax);
                den += p;
                const double *vv = vloc + (nb[k] * Hkv + g) * d;
                for (int e = 0; e < d; ++e) o[e] += p * vv[e];
            }
            for (int e = 0; e < d; ++e) o[e] /= den;
        }
        free(nb);
        free(l);
    }
}

/* ---- compressed branch: every query against all M summaries ------------ */

/* o[r,h] = sum_j softmax_j(scale <qr[r,h], ksum[j,g]>) vsum[j,g] over all M
 * summaries; qr holds the sampled rows' rotated queries in sample order. */

void orc_summary_attn(const orc_cfg *c, const double *qr, const double *ksum,
                      const double *vsum, long M, long nrows, double *ocmp)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (long r = 0; r < nrows; ++r) {
        double *l = (double *)malloc(sizeof(double) * M);
        for (int h = 0; h < Hq; ++h) {
            int g = (int)(((long)h * Hkv) / Hq);
            const double *q = qr + (r * Hq + h) * d;
            double lmax = -INFINITY, den = 0.0;
            for (long j = 0; j < M; ++j) {
                const double *kk = ksum + (j * Hkv + g) * d;
                double s = 0.0;
                for (int e = 0; e < d; ++e) s += q[e] * kk[e];
                l[j] = c->scale * s;
                if (l[j] > lmax) lmax = l[j];
            }
            double *o = ocmp + (r * Hq + h) * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (long j = 0; j < M; ++j) {
                double p = exp(l[j] - lmax);
                den += p;
                const double *vv = vsum + (j * Hkv + g) * d;
                for (int e = 0; e < d; ++e) o[e] += p * vv[e];
            }
            for (int e = 0; e < d; ++e) o[e] /= den;
        }
        free(l);
    }
}

/* ---- tokenwise softmax gate ------------------------------------------- */

/* (gamma0, gamma1) = softmax(gate[i,h,0], gate[i,h,1]);
 * out = gamma0 * oloc + gamma1 * ocmp, for the sampled rows. */
void orc_gate_mix(const orc_cfg *c, const double *gate, const int64_t *rows, long nrows,
                  const double *oloc, const double *ocmp, double *out)
{
    int d = c->dh, Hq = c->Hq;
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        for (int h = 0; h < Hq; ++h) {
            double g0 = gate[(i * Hq + h) * 2], g1 = gate[(i * Hq + h) * 2 + 1];
            double gm = g0 > g1 ? g0 : g1;
            double e0 = exp(g0 - gm), e1 = exp(g1 - gm);
            double w0 = e0 / (e0 + e1), w1 = e1 / (e0 + e1);
            for (int e = 0; e < d; ++e) {
                long k = (r * Hq + h) * d + e;
                out[k] = w0 * oloc[k] + w1 * ocmp[k];
            }
        }
    }
}

/* ======================================================================
 * Backward pass of the training block (the pages call the operator a fused
 * forward/backward block; these functions give its gradients).  With
 * L = <dout, out>, each function applies the chain rule to one forward
 * stage, in reverse order of the forward pass:
 *   gate -> both attention branches -> summaries and RoPE.
 * For a softmax over logits l_j = scale <q, k_j> with o = sum_j P_j v_j,
 *   dP_j = <do, v_j>,  dl_j = P_j (dP_j - sum_j' P_j' dP_j'),
 *   dq = scale sum_j dl_j k_j,  dk_j += scale dl_j q,  dv_j += P_j do.
 * The row quantities lse = log sum_j exp(l_j) and delta = sum_j P_j dP_j
 * (= <do, o>) are formed in a first pass over the query rows and read by
 * the second pass, which sums over queries per key; that is the same
 * arithmetic in another order.
 * ==================================================================== */

/* x = R(c)^T y: each active pair (y0, y1) becomes
 * (y0 cos t + y1 sin t, -y0 sin t + y1 cos t). */
static void rotate_row_t(const orc_cfg *c, double cz, double cy, double cx, const double *yi, double *xi)
{
    for (int p = 0; p < c->dh / 2; ++p) {
        int active;
        double t = pair_angle(c, p, cz, cy, cx, &active);
        double y0 = yi[2 * p], y1 = yi[2 * p + 1];
        if (active) {
            xi[2 * p] = y0 * cos(t) + y1 * sin(t);
            xi[2 * p + 1] = -y0 * sin(t) + y1 * cos(t);
        } else {
            xi[2 * p] = y0;
            xi[2 * p + 1] = y1;
        }
    }
}

/* x[i,h,:] = R(c_i)^T y[i,h,:]: the RoPE backward for n tokens. */
void orc_rotate_t(const orc_cfg *c, const int32_t *coords, const double *y, double *x,
                  int heads, long n)
{
    int d = c->dh;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i)
        for (int h = 0; h < heads; ++h)
            rotate_row_t(c, coords[3 * i], coords[3 * i + 1], coords[3 * i + 2],
                         y + ((long)i * heads + h) * d, x + ((long)i * heads + h) * d);
}

/* Gate backward for the sampled rows (r-th entry = token rows[r]):
 *   gamma = softmax(gate[i,h,:]),  dgamma_c = <dout, o_c>  (o_0 = oloc, o_1 = ocmp)
 *   dgate_c = gamma_c (dgamma_c - sum_c' gamma_c' dgamma_c')
 *   dol = gamma_0 dout,  doc = gamma_1 dout.
 * oloc, ocmp, dout, dol, doc hold the sampled rows in sample order. */
void orc_gate_backward(const orc_cfg *c, const double *gate, const int64_t *rows, long nrows,
                       const double *oloc, const double *ocmp, const double *dout,
                       double *dgate, double *dol, double *doc)
{
    int d = c->dh, Hq = c->Hq;
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        for (int h = 0; h < Hq; ++h) {
            double g0 = gate[(i * Hq + h) * 2], g1 = gate[(i * Hq + h) * 2 + 1];
            double gm = g0 > g1 ? g0 : g1;
            double e0 = exp(g0 - gm), e1 = exp(g1 - gm);
            double w0 = e0 / (e0 + e1), w1 = e1 / (e0 + e1);
            long k0 = (r * Hq + h) * d;
            double A = 0.0, B = 0.0;
            for (int e = 0; e < d; ++e) {
                A += dout[k0 + e] * oloc[k0 + e];
                B += dout[k0 + e] * ocmp[k0 + e];
            }
            double mean = w0 * A + w1 * B;
            dgate[(r * Hq + h) * 2] = w0 * (A - mean);
            dgate[(r * Hq + h) * 2 + 1] = w1 * (B - mean);
            for (int e = 0; e < d; ++e) {
                dol[k0 + e] = w0 * dout[k0 + e];
                doc[k0 + e] = w1 * dout[k0 + e];
            }
        }
    }
}

/* Packed indices of the tokens in the clipped box of radii (rz,ry,rx)
 * around site (zi,yi,xi); returns the count.  The box relation is symmetric:
 * j lies in the window of i exactly when i lies in the window of j. */
static long window_tokens(const orc_cfg *c, const int32_t *g2p, int zi, int yi, int xi, long *nb)
{
    long cnt = 0;
    for (int z = zi - c->rz; z <= zi + c->rz; ++z)
        for (int y = yi - c->ry; y <= yi + c->ry; ++y)
            for (int x = xi - c->rx; x <= xi + c->rx; ++x) {
                if (z < 0 || z >= c->Z || y < 0 || y >= c->H || x < 0 || x >= c->W) continue;
                nb[cnt++] = g2p[((long)z * c->H + y) * c->W + x];
            }
    return cnt;
}

/* Local branch, first pass, for the sampled rows (qr, dol, dqr in sample
 * order): dqr[r,h] = scale sum_j dl_j klr[j,g], and each row's lse and
 * delta = sum_j P_j <dol, vloc[j,g]>. */
void orc_local_attn_backward_q(const orc_cfg *c, const int32_t *coords, const int32_t *g2p,
                               const double *qr, const double *klr, const double *vloc,
                               const double *dol, const int64_t *rows, long nrows,
                               double *dqr, double *lse, double *delta)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
    long wmax = (long)(2 * c->rz + 1) * (2 * c->ry + 1) * (2 * c->rx + 1);
#pragma omp parallel for schedule(dynamic, 16)
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        long *nb = (long *)malloc(sizeof(long) * wmax);
        double *l = (double *)malloc(sizeof(double) * wmax);
        double *dp = (double *)malloc(sizeof(double) * wmax);
        long cnt = window_tokens(c, g2p, coords[3 * i], coords[3 * i + 1], coords[3 * i + 2], nb);
        for (int h = 0; h < Hq; ++h) {
            int g = (int)(((long)h * Hkv) / Hq);
            const double *q = qr + (r * Hq + h) * d;
            const double *dor = dol + (r * Hq + h) * d;
            double lmax = -INFINITY, den = 0.0, dl_mean = 0.0;
            for (long k = 0; k < cnt; ++k) {
                const double *kk = klr + (nb[k] * Hkv + g) * d;
                const double *vv = vloc + (nb[k] * Hkv + g) * d;
                double s = 0.0, t = 0.0;
                for (int e = 0; e < d; ++e) { s += q[e] * kk[e]; t += dor[e] * vv[e]; }
                l[k] = c->scale * s;
                dp[k] = t;
                if (l[k] > lmax) lmax = l[k];
            }
            for (long k = 0; k < cnt; ++k) den += exp(l[k] - lmax);
            double ls = lmax + log(den);
            for (long k = 0; k < cnt; ++k) dl_mean += exp(l[k] - ls) * dp[k];
            double *dq = dqr + (r * Hq + h) * d;
            for (int e = 0; e < d; ++e) dq[e] = 0.0;
            for (long k = 0; k < cnt; ++k) {
                double dl = exp(l[k] - ls) * (dp[k] - dl_mean);
                const double *kk = klr + (nb[k] * Hkv + g) * d;
                for (int e = 0; e < d; ++e) dq[e] += c->scale * dl * kk[e];
            }
            lse[r * Hq + h] = ls;
            delta[r * Hq + h] = dl_mean;
        }
        free(nb);
        free(l);
        free(dp);
    }
}

/* Local branch, second pass, for the listed keys: for key token j and kv
 * head g, over every query i whose window holds j (the box around j) and
 * every q head h of group g,
 *   dklr[k,g] = scale sum dl_{ih,j} qr[i,h],  dvloc[k,g] = sum P_{ih,j} dol[i,h].
 * qr, dol, lse, delta hold every token; dklr, dvloc the listed keys in order. */
void orc_local_attn_backward_kv(const orc_cfg *c, const int32_t *coords, const int32_t *g2p,
                                const double *qr, const double *klr, const double *vloc,
                                const double *dol, const double *lse, const double *delta,
                                const int64_t *keys, long nkeys, double *dklr, double *dvloc)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
    long wmax = (long)(2 * c->rz + 1) * (2 * c->ry + 1) * (2 * c->rx + 1);
#pragma omp parallel for schedule(dynamic, 16)
    for (long r = 0; r < nkeys; ++r) {
        long j = keys[r];
        long *nb = (long *)malloc(sizeof(long) * wmax);
        long cnt = window_tokens(c, g2p, coords[3 * j], coords[3 * j + 1], coords[3 * j + 2], nb);
        for (int g = 0; g < Hkv; ++g) {
            const double *kk = klr + (j * Hkv + g) * d;
            const double *vv = vloc + (j * Hkv + g) * d;
            double *dk = dklr + (r * Hkv + g) * d;
            double *dv = dvloc + (r * Hkv + g) * d;
            for (int e = 0; e < d; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
            for (long k = 0; k < cnt; ++k) {
                long i = nb[k];
                for (int h = 0; h < Hq; ++h) {
                    if ((int)(((long)h * Hkv) / Hq) != g) continue;
                    const double *q = qr + (i * Hq + h) * d;
                    const double *dor = dol + (i * Hq + h) * d;
                    double s = 0.0, t = 0.0;
                    for (int e = 0; e < d; ++e) { s += q[e] * kk[e]; t += dor[e] * vv[e]; }
                    double P = exp(c->scale * s - lse[i * Hq + h]);
                    double dl = P * (t - delta[i * Hq + h]);
                    for (int e = 0; e < d; ++e) {
                        dk[e] += c->scale * dl * q[e];
                        dv[e] += P * dor[e];
                    }
                }
            }
        }
        free(nb);
    }
}

/* Compressed branch, first pass, for nrows query rows (qr, doc in row order)
 * against all M summaries: each row's lse and delta, and, when dqr is not
 * NULL, dqr[r,h] = scale sum_j dl_j ksum[j,g]. */
void orc_summary_attn_backward_q(const orc_cfg *c, const double *qr, const double *ksum,
                                 const double *vsum, long M, long nrows, const double *doc,
                                 double *dqr, double *lse, double *delta)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (long r = 0; r < nrows; ++r) {
        double *l = (double *)malloc(sizeof(double) * M);
        double *dp = (double *)malloc(sizeof(double) * M);
        for (int h = 0; h < Hq; ++h) {
            int g = (int)(((long)h * Hkv) / Hq);
            const double *q = qr + (r * Hq + h) * d;
            const double *dor = doc + (r * Hq + h) * d;
            double lmax = -INFINITY, den = 0.0, dl_mean = 0.0;
            for (long j = 0; j < M; ++j) {
                const double *kk = ksum + (j * Hkv + g) * d;
                const double *vv = vsum + (j * Hkv + g) * d;
                double s = 0.0, t = 0.0;
                for (int e = 0; e < d; ++e) { s += q[e] * kk[e]; t += dor[e] * vv[e]; }
                l[j] = c->scale * s;
                dp[j] = t;
                if (l[j] > lmax) lmax = l[j];
            }
            for (long j = 0; j < M; ++j) den += exp(l[j] - lmax);
            double ls = lmax + log(den);
            for (long j = 0; j < M; ++j) dl_mean += exp(l[j] - ls) * dp[j];
            if (dqr) {
                double *dq = dqr + (r * Hq + h) * d;
                for (int e = 0; e < d; ++e) dq[e] = 0.0;
                for (long j = 0; j < M; ++j) {
                    double dl = exp(l[j] - ls) * (dp[j] - dl_mean);
                    const double *kk = ksum + (j * Hkv + g) * d;
                    for (int e = 0; e < d; ++e) dq[e] += c->scale * dl * kk[e];
                }
            }
            lse[r * Hq + h] = ls;
            delta[r * Hq + h] = dl_mean;
        }
        free(l);
        free(dp);
    }
}

/* Compressed branch, second pass, for the listed summaries js: over every
 * query row i (all nrows, in row order) and q head h of group g,
 *   dksum[k,g] = scale sum dl_{ih,j} qr[i,h],  dvsum[k,g] = sum P_{ih,j} doc[i,h]. */
void orc_summary_attn_backward_kv(const orc_cfg *c, const double *qr, const double *ksum,
                                  const double *vsum, long nrows, const double *doc,
                                  const double *lse, const double *delta,
                                  const int64_t *js, long nj, double *dksum, double *dvsum)
{
    int d = c->dh, Hq = c->Hq, Hkv = c->Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < nj * Hkv; ++r) {
        long jr = r / Hkv;
        int g = (int)(r % Hkv);
        long j = js[jr];
        const double *kk = ksum + (j * Hkv + g) * d;
        const double *vv = vsum + (j * Hkv + g) * d;
        double *dk = dksum + (jr * Hkv + g) * d;
        double *dv = dvsum + (jr * Hkv + g) * d;
        for (int e = 0; e < d; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
        for (long i = 0; i < nrows; ++i)
            for (int h = 0; h < Hq; ++h) {
                if ((int)(((long)h * Hkv) / Hq) != g) continue;
                const double *q = qr + (i * Hq + h) * d;
                const double *dor = doc + (i * Hq + h) * d;
                double s = 0.0, t = 0.0;
                for (int e = 0; e < d; ++e) { s += q[e] * kk[e]; t += dor[e] * vv[e]; }
                double P = exp(c->scale * s - lse[i * Hq + h]);
                double dl = P * (t - delta[i * Hq + h]);
                for (int e = 0; e < d; ++e) {
                    dk[e] += c->scale * dl * q[e];
                    dv[e] += P * dor[e];
                }
            }
    }
}

/* Summaries backward (rotate-before-compress form) for the listed blocks
 * (dksum, dvsum and the outputs in list order; member t of block jr at
 * row jr*v + t):
 *   a_u = softmax over B_j of s_{u,g},  Kcr_u = R(c_u) kcmp[u,g]
 *   dkcmp[u,g] = R(c_u)^T (a_u dksum[j,g]),  dvcmp[u,g] = a_u dvsum[j,g]
 *   da_u = <dksum[j,g], Kcr_u> + <dvsum[j,g], vcmp[u,g]>
 *   dscores[u,g] = a_u (da_u - sum_u' a_u' da_u'). */
void orc_summaries_backward(const orc_cfg *c, const int32_t *coords, const int32_t *members,
                            const double *kcmp, const double *vcmp, const double *scores,
                            const double *dksum, const double *dvsum,
                            const int64_t *blocks, long nb, double *dkcmp, double *dvcmp,
                            double *dscores)
{
    int v = c->bz * c->by * c->bx;
    int d = c->dh, Hkv = c->Hkv;
#pragma omp parallel for schedule(static)
    for (long jr = 0; jr < nb; ++jr) {
        long j = blocks[jr];
        double *a = (double *)malloc(sizeof(double) * v);
        double *da = (double *)malloc(sizeof(double) * v);
        double *kr = (double *)malloc(sizeof(double) * d);
        double *t = (double *)malloc(sizeof(double) * d);
        for (int g = 0; g < Hkv; ++g) {
            const double *dk = dksum + (jr * Hkv + g) * d;
            const double *dv = dvsum + (jr * Hkv + g) * d;
            double smax = -INFINITY, den = 0.0, mean = 0.0;
            for (int m = 0; m < v; ++m) {
                double s = scores[(long)members[j * v + m] * Hkv + g];
                if (s > smax) smax = s;
            }
            for (int m = 0; m < v; ++m) {
                a[m] = exp(scores[(long)members[j * v + m] * Hkv + g] - smax);
                den += a[m];
            }
            for (int m = 0; m < v; ++m) a[m] /= den;
            for (int m = 0; m < v; ++m) {
                long u = members[j * v + m];
                rotate_row(c, coords[3 * u], coords[3 * u + 1], coords[3 * u + 2],
                           kcmp + (u * Hkv + g) * d, kr);
                da[m] = 0.0;
                for (int e = 0; e < d; ++e)
                    da[m] += dk[e] * kr[e] + dv[e] * vcmp[(u * Hkv + g) * d + e];
                mean += a[m] * da[m];
                for (int e = 0; e < d; ++e) t[e] = a[m] * dk[e];
                long o = ((jr * v + m) * Hkv + g) * d;
                rotate_row_t(c, coords[3 * u], coords[3 * u + 1], coords[3 * u + 2], t, dkcmp + o);
                for (int e = 0; e < d; ++e) dvcmp[o + e] = a[m] * dv[e];
            }
            for (int m = 0; m < v; ++m) dscores[(jr * v + m) * Hkv + g] = a[m] * (da[m] - mean);
        }
        free(a);
        free(da);
        free(kr);
        free(t);
    }
}

/* Summary-centre variant backward, for the listed blocks (layout as
 * orc_summaries_backward): with kp_j = sum_u a_u kcmp[u,g] and
 * ksum = R(cbar_j) kp_j,
 *   dkp = R(cbar_j)^T dksum[j,g]
 *   dkcmp[u,g] = a_u dkp,  dvcmp[u,g] = a_u dvsum[j,g]
 *   da_u = <dkp, kcmp[u,g]> + <dvsum[j,g], vcmp[u,g]>
 *   dscores[u,g] = a_u (da_u - sum_u' a_u' da_u'). */
void orc_summaries_center_backward(const orc_cfg *c, const int32_t *members, const double *kcmp,
                                   const double *vcmp, const double *scores, const double *dksum,
                                   const double *dvsum, const int64_t *blocks, long nb,
                                   double *dkcmp, double *dvcmp, double *dscores)
{
    int v = c->bz * c->by * c->bx;
    int nby = c->H / c->by, nbx = c->W / c->bx;
    int d = c->dh, Hkv = c->Hkv;
#pragma omp parallel for schedule(static)
    for (long jr = 0; jr < nb; ++jr) {
        long j = blocks[jr];
        long jx = j % nbx, jy = (j / nbx) % nby, jz = j / ((long)nbx * nby);
        double cz = jz * c->bz + 0.5 * (c->bz - 1);
        double cy = jy * c->by + 0.5 * (c->by - 1);
        double cx = jx * c->bx + 0.5 * (c->bx - 1);
        double *a = (double *)malloc(sizeof(double) * v);
        double *da = (double *)malloc(sizeof(double) * v);
        double *dkp = (double *)malloc(sizeof(double) * d);
        for (int g = 0; g < Hkv; ++g) {
            const double *dv = dvsum + (jr * Hkv + g) * d;
            rotate_row_t(c, cz, cy, cx, dksum + (jr * Hkv + g) * d, dkp);
            double smax = -INFINITY, den = 0.0, mean = 0.0;
            for (int m = 0; m < v; ++m) {
                double s = scores[(long)members[j * v + m] * Hkv + g];
                if (s > smax) smax = s;
            }
            for (int m = 0; m < v; ++m) {
                a[m] = exp(scores[(long)members[j * v + m] * Hkv + g] - smax);
                den += a[m];
            }
            for (int m = 0; m < v; ++m) a[m] /= den;
            for (int m = 0; m < v; ++m) {
                long u = members[j * v + m];
                da[m] = 0.0;
                for (int e = 0; e < d; ++e)
                    da[m] += dkp[e] * kcmp[(u * Hkv + g) * d + e] + dv[e] * vcmp[(u * Hkv + g) * d + e];
                mean += a[m] * da[m];
                long o = ((jr * v + m) * Hkv + g) * d;
                for (int e = 0; e < d; ++e) {
                    dkcmp[o + e] = a[m] * dkp[e];
                    dvcmp[o + e] = a[m] * dv[e];
                }
            }
            for (int m = 0; m < v; ++m) dscores[(jr * v + m) * Hkv + g] = a[m] * (da[m] - mean);
        }
        free(a);
        free(da);
        free(dkp);
    }
}
