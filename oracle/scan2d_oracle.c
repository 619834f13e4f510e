/*
 * scan2d_oracle.c -- plain, slow, fp64 reference of the 2D selective-scan forward and of
 * its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load this code.  The product path (the CUDA library) shares
 * no code with it and never calls it.
 *
 * Sources (web pages on 2DMamba, arXiv 2412.00678):
 *   [J]  "2DMamba 精读：从小白到博士，彻底拆解 2DMamba" (juejin.cn)
 *          4.4  "2DMamba 的核心：二维 selective scan"   -- 1D recurrence h_t = A_t h_{t-1} + B_t x_t
 *          4.5  "2DMamba 如何扩展到二维？" (1) 横向扫描 -- horizontal recurrence
 *                                         (2) 纵向扫描 -- vertical recurrence, output y = C h
 *          5.3  "数学层面的关键理解"                    -- unrolled (Manhattan) form
 *   [PN] papernotes.org notes on the CVPR 2025 paper, "关键设计" (2D selective SSM
 *          architecture; the 3x3 example; the hardware-aware operator)
 *
 * What is computed, for every (b, d) map and every state n (readings of the pages that
 * are not printed there are marked READING):
 *   Abar[i,j]  = exp(delta[i,j] * A[d,n])                       READING: zero-order exp,
 *   Bbar[i,j]  = delta[i,j] * B[n,i,j]                           simplified Euler Bbar
 *   hh[i,j]    = Abar[i,j]*hh[i,j-1] + Bbar[i,j]*x[i,j]          [J 4.5(1)], hh[i,-1] = 0
 *   h[i,j]     = Abar[i,j]*h[i-1,j]  + hh[i,j]                   [J 4.5(2)], h[-1,j]  = 0
 *   y[i,j]    += C[n,i,j]*h[i,j]                                 [J 4.5(2)] output
 * and finally y[i,j] += Dskip[d]*x[i,j] once (READING: the skip term is not on the pages).
 * The same Abar is used in both scans and the vertical scan adds no second Bbar
 * ([J 4.5(2)] writes Abar_{i,j} and h^hor_{i,j} only).
 *
 * Scan order ([PN 消融实验要点]: horizontal-then-vertical and vertical-then-horizontal are
 * both studied; READING: the same two recurrences in the other order).  With bit 4 of the
 * mask set, each (b, d, n) map is scanned vertical-first:
 *   vv[i,j]    = Abar[i,j]*vv[i-1,j] + Bbar[i,j]*x[i,j]          vv[-1,j] = 0
 *   h[i,j]     = Abar[i,j]*h[i,j-1]  + vv[i,j]                   h[i,-1]  = 0
 *   y[i,j]    += C[n,i,j]*h[i,j]
 *
 * Orientations (READING of "reverse scans" in [PN 局限与展望] and "四象限" in [J 7.4]):
 * an orientation flips the map in H and/or W, runs the scan above from its own corner
 * with its own B_k, C_k (stored in the original, unflipped coordinates), and its output is
 * added at the original positions.  Bit 0 = top-left (no flip), bit 1 = top-right (flip
 * W), bit 2 = bottom-left (flip H), bit 3 = bottom-right (both).  delta and A are shared.
 *
 * Layouts (all dense, row-major, W fastest):
 *   x, delta : (batch, channels, H, W)      fp32 or bf16 bits
 *   A        : (channels, N)                fp32
 *   B, C     : (batch, K, N, H, W)          fp32 or bf16 bits, K = number of orientations
 *   Dskip    : (channels)                   fp32, NULL means 0
 *   y        : (batch, channels, H, W)      fp64 (output of this file)
 * Every stored input value is converted exactly to double before use.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_VERSION 3

/* bf16 bits -> double, exact (a bf16 value is the top 16 bits of an IEEE fp32 value). */
static double bf16_to_double(uint16_t v)
{
    uint32_t u = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Element e of a buffer holding fp32 (is_bf16 == 0) or bf16 bits (is_bf16 != 0). */
static double load(const void *buf, size_t e, int is_bf16)
{
    if (is_bf16)
        return bf16_to_double(((const uint16_t *)buf)[e]);
    return (double)((const float *)buf)[e];
}

typedef struct {
    const void *x, *delta, *B, *C;
    const float *A, *Dskip;
    int batch, channels, H, W, N, K, is_bf16;
    int vfirst;                                     /* bit 4 of the mask: vertical first */
} problem;

/* Orientation number (0..3) of the k-th set bit of the mask, or -1. */
static int orientation_of(unsigned mask, int k)
{
    int seen = 0;
    for (int o = 0; o < 4; ++o) {
        if (mask & (1u << o)) {
            if (seen == k)
                return o;
            ++seen;
        }
    }
    return -1;
}

/*
 * One orientation of one (b, d) map, scanned over the sub-rectangle of scan-order rows
 * 0..rows-1 and scan-order columns 0..cols-1.  Scan-order (ii, jj) maps to the original
 * position (flipH ? H-1-ii : ii, flipW ? W-1-jj : jj).  The result C.h is added into
 * yacc (an H*W array in original coordinates).  hcol is scratch of length >= cols.
 */
static void scan_one_orientation(const problem *p, int b, int d, int k, int orient,
                                 int rows, int cols, double *yacc, double *hcol)
{
    const int vfirst = p->vfirst;
    const int H = p->H, W = p->W, N = p->N, K = p->K;
    const int flipW = orient & 1, flipH = (orient >> 1) & 1;
    const size_t map = ((size_t)b * p->channels + d) * (size_t)H * W;
    for (int n = 0; n < N; ++n) {
        const double An = (double)p->A[(size_t)d * N + n];
        const size_t bc = (((size_t)b * K + k) * N + n) * (size_t)H * W;
        for (int jj = 0; jj < cols; ++jj)
            hcol[jj] = 0.0;                                /* h[-1, j] = 0 */
        for (int ii = 0; ii < rows; ++ii) {
            const int i = flipH ? H - 1 - ii : ii;
            double hh = 0.0;                               /* hh[i, -1] = 0 */
            for (int jj = 0; jj < cols; ++jj) {
                const int j = flipW ? W - 1 - jj : jj;
                const size_t pos = (size_t)i * W + j;
                const double dl = load(p->delta, map + pos, p->is_bf16);
                const double xv = load(p->x, map + pos, p->is_bf16);
                const double Bv = load(p->B, bc + pos, p->is_bf16);
                const double Cv = load(p->C, bc + pos, p->is_bf16);
                const double abar = exp(dl * An);          /* Abar = exp(delta*A)   */
                if (!vfirst) {
                    hh = abar * hh + (dl * Bv) * xv;       /* horizontal, [J 4.5(1)] */
                    hcol[jj] = abar * hcol[jj] + hh;       /* vertical,   [J 4.5(2)] */
                    yacc[pos] += Cv * hcol[jj];            /* y = C h,    [J 4.5(2)] */
                } else {
                    hcol[jj] = abar * hcol[jj] + (dl * Bv) * xv;   /* vertical first  */
                    hh = abar * hh + hcol[jj];             /* then horizontal       */
                    yacc[pos] += Cv * hh;                  /* y = C h               */
                }
            }
        }
    }
}

static int check(const problem *p, unsigned mask)
{
    if (!p->x || !p->delta || !p->A || !p->B || !p->C)
        return -1;
    if (p->batch < 1 || p->channels < 1 || p->H < 1 || p->W < 1 || p->N < 1)
        return -2;
    if ((mask & 0xFu) == 0 || (mask & ~0x1Fu))
        return -4;
    return 0;
}

static void init_problem(problem *p, const void *x, const void *delta, const float *A,
                         const void *B, const void *C, const float *Dskip, int batch,
                         int channels, int H, int W, int N, int is_bf16, unsigned mask)
{
    p->x = x; p->delta = delta; p->A = A; p->B = B; p->C = C; p->Dskip = Dskip;
    p->batch = batch; p->channels = channels; p->H = H; p->W = W; p->N = N;
    p->is_bf16 = is_bf16;
    p->vfirst = (mask >> 4) & 1u;
    p->K = 0;
    for (int o = 0; o < 4; ++o)
        p->K += (mask >> o) & 1u;
}

/* y for the maps listed in maps[2*m] = b, maps[2*m+1] = d; y_out is (nmaps, H, W). */
int scan2d_oracle_maps(const void *x, const void *delta, const float *A, const void *B,
                       const void *C, const float *Dskip, double *y_out, int batch,
                       int channels, int H, int W, int N, int is_bf16, unsigned orient_mask,
                       const int *maps, int nmaps)
{
    problem p;
    init_problem(&p, x, delta, A, B, C, Dskip, batch, channels, H, W, N, is_bf16, orient_mask);
    int rc = check(&p, orient_mask);
    if (rc)
        return rc;
    if (!y_out || (nmaps > 0 && !maps))
        return -1;
    double *hcol = (double *)malloc(sizeof(double) * (size_t)W);
    if (!hcol)
        return -8;
    const size_t HW = (size_t)H * W;
    for (int m = 0; m < nmaps; ++m) {
        const int b = maps[2 * m], d = maps[2 * m + 1];
        if (b < 0 || b >= batch || d < 0 || d >= channels) {
            free(hcol);
            return -2;
        }
        double *ym = y_out + (size_t)m * HW;
        const size_t map = ((size_t)b * channels + d) * HW;
        const double Dd = Dskip ? (double)Dskip[d] : 0.0;
        for (size_t pos = 0; pos < HW; ++pos)
            ym[pos] = 0.0;
        for (int k = 0; k < p.K; ++k)
            scan_one_orientation(&p, b, d, k, orientation_of(orient_mask, k), H, W, ym, hcol);
        for (size_t pos = 0; pos < HW; ++pos)                     /* + Dskip * x, once */
            ym[pos] += Dd * load(x, map + pos, is_bf16);
    }
    free(hcol);
    return 0;
}

/* y for every map; y_out is (batch, channels, H, W). */
int scan2d_oracle_fwd(const void *x, const void *delta, const float *A, const void *B,
                      const void *C, const float *Dskip, double *y_out, int batch,
                      int channels, int H, int W, int N, int is_bf16, unsigned orient_mask)
{
    if (batch < 1 || channels < 1)
        return -2;
    int *maps = (int *)malloc(sizeof(int) * 2 * (size_t)batch * channels);
    if (!maps)
        return -8;
    for (int b = 0, m = 0; b < batch; ++b)
        for (int d = 0; d < channels; ++d, ++m) {
            maps[2 * m] = b;
            maps[2 * m + 1] = d;
        }
    int rc = scan2d_oracle_maps(x, delta, A, B, C, Dskip, y_out, batch, channels, H, W, N,
                                is_bf16, orient_mask, maps, batch * channels);
    free(maps);
    return rc;
}

/*
 * y at single positions.  points[4*q .. 4*q+3] = (b, d, i, j).  Only the rectangle between
 * each orientation's starting corner and (i, j) can reach (i, j), so the scan runs over
 * that rectangle alone: the same recurrences, cut short.
 */
int scan2d_oracle_points(const void *x, const void *delta, const float *A, const void *B,
                         const void *C, const float *Dskip, double *y_out, int batch,
                         int channels, int H, int W, int N, int is_bf16, unsigned orient_mask,
                         const int *points, int npoints)
{
    problem p;
    init_problem(&p, x, delta, A, B, C, Dskip, batch, channels, H, W, N, is_bf16, orient_mask);
    int rc = check(&p, orient_mask);
    if (rc)
        return rc;
    if (!y_out || (npoints > 0 && !points))
        return -1;
    double *hcol = (double *)malloc(sizeof(double) * (size_t)W);
    double *yacc = (double *)malloc(sizeof(double) * (size_t)H * W);
    if (!hcol || !yacc) {
        free(hcol);
        free(yacc);
        return -8;
    }
    for (int q = 0; q < npoints; ++q) {
        const int b = points[4 * q], d = points[4 * q + 1];
        const int i = points[4 * q + 2], j = points[4 * q + 3];
        if (b < 0 || b >= batch || d < 0 || d >= channels || i < 0 || i >= H || j < 0 || j >= W) {
            free(hcol);
            free(yacc);
            return -2;
        }
        const size_t pos = (size_t)i * W + j;
        double total = 0.0;
        for (int k = 0; k < p.K; ++k) {
            const int o = orientation_of(orient_mask, k);
            const int flipW = o & 1, flipH = (o >> 1) & 1;
            const int rows = flipH ? H - i : i + 1;
            const int cols = flipW ? W - j : j + 1;
            yacc[pos] = 0.0;
            /* positions other than (i, j) inside the rectangle also get written; only
               (i, j) is read, so they are cleared lazily by writing the whole rectangle. */
            for (int ii = 0; ii < rows; ++ii) {
                const int ri = flipH ? H - 1 - ii : ii;
                for (int jj = 0; jj < cols; ++jj)
                    yacc[(size_t)ri * W + (flipW ? W - 1 - jj : jj)] = 0.0;
            }
            scan_one_orientation(&p, b, d, k, o, rows, cols, yacc, hcol);
            total += yacc[pos];
        }
        const size_t map = ((size_t)b * channels + d) * (size_t)H * W;
        total += (Dskip ? (double)Dskip[d] : 0.0) * load(x, map + pos, is_bf16);
        y_out[q] = total;
    }
    free(hcol);
    free(yacc);
    return 0;
}

/*
 * Gradients of the forward above (the pages give no backward pass; these are the plain
 * chain-rule adjoints of the two recurrences, READING: the training gradient of y).
 *
 * For a cotangent dy (fp64, (batch, channels, H, W)) they are the derivatives of
 *   L = sum_{b,d,i,j} dy[b,d,i,j] * y[b,d,i,j]
 * with respect to x, delta (same layout as x), A (channels, N), B and C
 * ((batch, K, N, H, W), summed over the channels that share them) and Dskip (channels).
 *
 * Writing s1 for the first scan's state and s2 for the second's (s1 = hh, s2 = h in the
 * horizontal-first order; s1 = vv, s2 = h vertical-first), the adjoint of s2 runs the
 * second scan backwards and the adjoint of s1 runs the first scan backwards:
 *   g2[p] = C[p]*dy[p] + Abar[p+e2]*g2[p+e2]     (e2 = the second scan's step)
 *   g1[p] = g2[p]      + Abar[p+e1]*g1[p+e1]     (e1 = the first scan's step)
 *   dL/dAbar[p] = g2[p]*s2[p-e2] + g1[p]*s1[p-e1],   dL/du[p] = g1[p],  u = delta*B*x
 * and then, with Abar = exp(delta*A):
 *   dx     += g1*delta*B                dB += g1*delta*x
 *   ddelta += dAbar*Abar*A + g1*B*x      dC += dy*s2
 *   dA     += dAbar*Abar*delta           dDskip += dy*x,  dx += Dskip*dy (once).
 *
 * majorant != 0 replaces every stored value by its magnitude and the factor A by |A|
 * (Abar itself keeps exp(delta*A)).  Every term of every sum is then non-negative, so
 * each output is the sum of the magnitudes of the terms that make up the true gradient:
 * the scale against which the rounding error of any evaluation order is bounded.
 */
static double mag(double v, int majorant) { return majorant ? fabs(v) : v; }

static void bwd_one_orientation(const problem *p, const double *dy, int b, int d, int k,
                                int orient, int majorant, double *a, double *u, double *s1,
                                double *s2, double *g1, double *g2, double *dx, double *ddelta,
                                double *dA, double *dB, double *dC)
{
    const int H = p->H, W = p->W, N = p->N, K = p->K;
    const int flipW = orient & 1, flipH = (orient >> 1) & 1;
    const size_t HW = (size_t)H * W;
    const size_t map = ((size_t)b * p->channels + d) * HW;
/* scan-order (ii, jj) -> index into the per-map work arrays */
#define AT(ii, jj) ((size_t)(ii) * W + (size_t)(jj))
    for (int n = 0; n < N; ++n) {
        const double An = (double)p->A[(size_t)d * N + n];
        const double Af = majorant ? fabs(An) : An;
        const size_t bc = (((size_t)b * K + k) * N + n) * HW;
        /* forward states, kept whole */
        for (int ii = 0; ii < H; ++ii)
            for (int jj = 0; jj < W; ++jj) {
                const int i = flipH ? H - 1 - ii : ii;     /* original position */
                const int j = flipW ? W - 1 - jj : jj;
                const size_t pos = (size_t)i * W + j, t = AT(ii, jj);
                const double dl = mag(load(p->delta, map + pos, p->is_bf16), majorant);
                const double xv = mag(load(p->x, map + pos, p->is_bf16), majorant);
                const double Bv = mag(load(p->B, bc + pos, p->is_bf16), majorant);
                a[t] = exp(dl * An);
                u[t] = (dl * Bv) * xv;
                if (!p->vfirst) {
                    s1[t] = a[t] * (jj > 0 ? s1[AT(ii, jj - 1)] : 0.0) + u[t];
                    s2[t] = a[t] * (ii > 0 ? s2[AT(ii - 1, jj)] : 0.0) + s1[t];
                } else {
                    s1[t] = a[t] * (ii > 0 ? s1[AT(ii - 1, jj)] : 0.0) + u[t];
                    s2[t] = a[t] * (jj > 0 ? s2[AT(ii, jj - 1)] : 0.0) + s1[t];
                }
            }
        /* adjoints, from the far corner back */
        for (int ii = H - 1; ii >= 0; --ii)
            for (int jj = W - 1; jj >= 0; --jj) {
                const int i = flipH ? H - 1 - ii : ii;     /* original position */
                const int j = flipW ? W - 1 - jj : jj;
                const size_t pos = (size_t)i * W + j, t = AT(ii, jj);
                const double gy = mag(dy[map + pos], majorant);
                const double Cv = mag(load(p->C, bc + pos, p->is_bf16), majorant);
                const int has_r = jj + 1 < W, has_d = ii + 1 < H;
                if (!p->vfirst) {
                    g2[t] = Cv * gy + (has_d ? a[AT(ii + 1, jj)] * g2[AT(ii + 1, jj)] : 0.0);
                    g1[t] = g2[t] + (has_r ? a[AT(ii, jj + 1)] * g1[AT(ii, jj + 1)] : 0.0);
                } else {
                    g2[t] = Cv * gy + (has_r ? a[AT(ii, jj + 1)] * g2[AT(ii, jj + 1)] : 0.0);
                    g1[t] = g2[t] + (has_d ? a[AT(ii + 1, jj)] * g1[AT(ii + 1, jj)] : 0.0);
                }
            }
        /* what each position contributes */
        double dA_n = 0.0;
        for (int ii = 0; ii < H; ++ii)
            for (int jj = 0; jj < W; ++jj) {
                const int i = flipH ? H - 1 - ii : ii;     /* original position */
                const int j = flipW ? W - 1 - jj : jj;
                const size_t pos = (size_t)i * W + j, t = AT(ii, jj);
                const double dl = mag(load(p->delta, map + pos, p->is_bf16), majorant);
                const double xv = mag(load(p->x, map + pos, p->is_bf16), majorant);
                const double Bv = mag(load(p->B, bc + pos, p->is_bf16), majorant);
                const double gy = mag(dy[map + pos], majorant);
                double s2_prev, s1_prev;                  /* s2[p - e2], s1[p - e1] */
                if (!p->vfirst) {
                    s2_prev = ii > 0 ? s2[AT(ii - 1, jj)] : 0.0;
                    s1_prev = jj > 0 ? s1[AT(ii, jj - 1)] : 0.0;
                } else {
                    s2_prev = jj > 0 ? s2[AT(ii, jj - 1)] : 0.0;
                    s1_prev = ii > 0 ? s1[AT(ii - 1, jj)] : 0.0;
                }
                const double dabar = g2[t] * s2_prev + g1[t] * s1_prev;
                dx[map + pos] += g1[t] * dl * Bv;
                ddelta[map + pos] += dabar * a[t] * Af + g1[t] * Bv * xv;
                dA_n += dabar * a[t] * dl;
                dB[bc + pos] += g1[t] * dl * xv;
                dC[bc + pos] += gy * s2[t];
            }
        dA[(size_t)d * N + n] += dA_n;
    }
#undef AT
}

int scan2d_oracle_bwd(const void *x, const void *delta, const float *A, const void *B,
                      const void *C, const float *Dskip, const double *dy, double *dx,
                      double *ddelta, double *dA, double *dB, double *dC, double *dDskip,
                      int batch, int channels, int H, int W, int N, int is_bf16,
                      unsigned orient_mask, int majorant)
{
    problem p;
    init_problem(&p, x, delta, A, B, C, Dskip, batch, channels, H, W, N, is_bf16, orient_mask);
    int rc = check(&p, orient_mask);
    if (rc)
        return rc;
    if (!dy || !dx || !ddelta || !dA || !dB || !dC || !dDskip)
        return -1;
    const size_t HW = (size_t)H * W;
    const size_t nx = (size_t)batch * channels * HW, nbc = (size_t)batch * p.K * N * HW;
    double *work = (double *)malloc(sizeof(double) * 6 * HW);
    if (!work)
        return -8;
    memset(dx, 0, sizeof(double) * nx);
    memset(ddelta, 0, sizeof(double) * nx);
    memset(dA, 0, sizeof(double) * (size_t)channels * N);
    memset(dB, 0, sizeof(double) * nbc);
    memset(dC, 0, sizeof(double) * nbc);
    memset(dDskip, 0, sizeof(double) * (size_t)channels);
    for (int b = 0; b < batch; ++b)
        for (int d = 0; d < channels; ++d) {
            for (int k = 0; k < p.K; ++k)
                bwd_one_orientation(&p, dy, b, d, k, orientation_of(orient_mask, k), majorant,
                                    work, work + HW, work + 2 * HW, work + 3 * HW, work + 4 * HW,
                                    work + 5 * HW, dx, ddelta, dA, dB, dC);
            /* the skip term y += Dskip*x, added once */
            const size_t map = ((size_t)b * channels + d) * HW;
            const double Dd = Dskip ? mag((double)Dskip[d], majorant) : 0.0;
            for (size_t pos = 0; pos < HW; ++pos) {
                const double gy = mag(dy[map + pos], majorant);
                dx[map + pos] += Dd * gy;
                dDskip[d] += gy * mag(load(x, map + pos, is_bf16), majorant);
            }
        }
    free(work);
    return 0;
}

int scan2d_oracle_version(void) { return ORACLE_VERSION; }
