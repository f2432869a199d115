/*
 * na2d_oracle.c -- plain, slow, fp64 reference for 2D Neighborhood Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header or table with the
 * CUDA library.
 *
 * What it computes (Neighborhood Attention Transformer, Sec. 3.1, Eqs. (2)-(4),
 * restated in the Qiita write-up "NAT: sliding-window attention", section
 * "Neighborhood Attention (NA)"):
 *
 *   for every query pixel (i, j) of an H x W map, per batch b and head h,
 *     A_n  = q(i,j) . key(r_n, t_n) + B(i,j ; r_n,t_n)                  Eq. (2)
 *     V_n  = value(r_n, t_n)                                             Eq. (3)
 *     out  = sum_n softmax(A / sqrt(d))_n * V_n                          Eq. (4)
 *   over the ks x ks neighbourhood {(r_n, t_n)} of (i, j).
 *
 * Readings taken where the pages leave a step open:
 *   - the neighbourhood is the ks x ks window whose start is
 *     clamp(i - floor(ks/2), 0, H - ks) on rows (same on columns): every
 *     pixel keeps the same span and corner pixels see a window that is not
 *     centred on them (Sec. 1 and App. C "repeated windows at edge pixels";
 *     the NA border drawing of the Qiita page);
 *   - the bias B is read from a per-head (2ks-1) x (2ks-1) table at
 *     [key_row - query_row + ks - 1][key_col - query_col + ks - 1];
 *     a NULL table means zero bias (App. B.1 ablates the bias away);
 *   - 1/sqrt(d) multiplies the bias as well as the dot product, exactly as
 *     Eq. (4) divides the whole of A by sqrt(d); d is the per-head size;
 *   - window entries are ordered row-major over the window: n = a*ks + c.
 *
 * Layouts (all contiguous, innermost last):
 *   q, k, v, out : [B][heads][H][W][d]
 *   rpb          : [heads][2ks-1][2ks-1]
 *   attn         : [B][heads][H][W][ks*ks]
 *
 * All arithmetic is fp64.  Inputs that come from 16-bit tensors are
 * converted exactly before they get here.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Start of the ks-wide window of position i on an axis of length L
 * (Sec. 3.1 "nearest neighbours", App. C, Qiita NA border figure). */
long na2d_oracle_window_start(long i, long L, long ks)
{
    long s = i - ks / 2;
    if (s < 0) s = 0;
    if (s > L - ks) s = L - ks;
    return s;
}

static size_t idx5(long b, long h, long i, long j, long heads, long H, long W, long last)
{
    return ((((size_t)b * heads + h) * H + i) * W + j) * (size_t)last;
}

static double bias_at(const double *rpb, long h, long ks, long dr, long dc)
{
    long span = 2 * ks - 1;
    if (!rpb) return 0.0;
    return rpb[((size_t)h * span + (dr + ks - 1)) * span + (dc + ks - 1)];
}

/* Eq. (2) for one query: A[n] = q . key_n + B, unscaled. */
static void logits_one(const double *q, const double *k, const double *rpb,
                       long b, long h, long i, long j,
                       long heads, long H, long W, long d, long ks, double *A)
{
    const double *qv = q + idx5(b, h, i, j, heads, H, W, d);
    long si = na2d_oracle_window_start(i, H, ks);
    long sj = na2d_oracle_window_start(j, W, ks);
    for (long a = 0; a < ks; a++) {
        for (long c = 0; c < ks; c++) {
            long r = si + a, t = sj + c;
            const double *kv = k + idx5(b, h, r, t, heads, H, W, d);
            double dot = 0.0;
            for (long x = 0; x < d; x++) dot += qv[x] * kv[x];
            A[a * ks + c] = dot + bias_at(rpb, h, ks, r - i, t - j);
        }
    }
}

/* softmax(scale * A) over n entries, in place, with the maximum subtracted. */
static void softmax_row(double *A, long n, double scale)
{
    double m = -INFINITY, sum = 0.0;
    for (long t = 0; t < n; t++) if (scale * A[t] > m) m = scale * A[t];
    for (long t = 0; t < n; t++) { A[t] = exp(scale * A[t] - m); sum += A[t]; }
    for (long t = 0; t < n; t++) A[t] /= sum;
}

/* Eqs. (3)-(4) for one query: out = sum_n P[n] * value_n. */
static void weighted_sum_one(const double *P, const double *v,
                             long b, long h, long i, long j,
                             long heads, long H, long W, long d, long ks, double *o)
{
    long si = na2d_oracle_window_start(i, H, ks);
    long sj = na2d_oracle_window_start(j, W, ks);
    for (long x = 0; x < d; x++) o[x] = 0.0;
    for (long a = 0; a < ks; a++) {
        for (long c = 0; c < ks; c++) {
            const double *vv = v + idx5(b, h, si + a, sj + c, heads, H, W, d);
            double p = P[a * ks + c];
            for (long x = 0; x < d; x++) o[x] += p * vv[x];
        }
    }
}

static int threads_for(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* The "QK + B" step alone (Eq. 2): attn = unscaled logits. */
void na2d_oracle_qk_rpb(const double *q, const double *k, const double *rpb, double *attn,
                        long B, long heads, long H, long W, long d, long ks, int nthreads)
{
    long rows = B * heads * H;
#pragma omp parallel for schedule(dynamic) num_threads(threads_for(nthreads))
    for (long row = 0; row < rows; row++) {
        long i = row % H, bh = row / H, h = bh % heads, b = bh / heads;
        for (long j = 0; j < W; j++)
            logits_one(q, k, rpb, b, h, i, j, heads, H, W, d, ks,
                       attn + idx5(b, h, i, j, heads, H, W, ks * ks));
    }
}

/* softmax(scale * attn) over each row of ks*ks entries, in place (Eq. 4). */
void na2d_oracle_softmax(double *attn, long nrows, long ks, double scale, int nthreads)
{
#pragma omp parallel for schedule(static) num_threads(threads_for(nthreads))
    for (long r = 0; r < nrows; r++) softmax_row(attn + (size_t)r * ks * ks, ks * ks, scale);
}

/* The "AV" step alone (Eqs. 3-4): out = attn applied to the window's values. */
void na2d_oracle_av(const double *attn, const double *v, double *out,
                    long B, long heads, long H, long W, long d, long ks, int nthreads)
{
    long rows = B * heads * H;
#pragma omp parallel for schedule(dynamic) num_threads(threads_for(nthreads))
    for (long row = 0; row < rows; row++) {
        long i = row % H, bh = row / H, h = bh % heads, b = bh / heads;
        for (long j = 0; j < W; j++)
            weighted_sum_one(attn + idx5(b, h, i, j, heads, H, W, ks * ks), v,
                             b, h, i, j, heads, H, W, d, ks,
                             out + idx5(b, h, i, j, heads, H, W, d));
    }
}

/* Full NA_k (Eq. 4) for the rows row_begin <= (b*heads + h)*H + i < row_end
 * (all W columns of each row); pass 0 and B*heads*H for the whole map. */
void na2d_oracle_forward_rows(const double *q, const double *k, const double *v,
                              const double *rpb, double *out,
                              long B, long heads, long H, long W, long d, long ks,
                              long row_begin, long row_end, int nthreads)
{
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel num_threads(threads_for(nthreads))
    {
        double *A = (double *)malloc(sizeof(double) * (size_t)ks * ks);
#pragma omp for schedule(dynamic)
        for (long row = row_begin; row < row_end; row++) {
            long i = row % H, bh = row / H, h = bh % heads, b = bh / heads;
            for (long j = 0; j < W; j++) {
                logits_one(q, k, rpb, b, h, i, j, heads, H, W, d, ks, A);
                softmax_row(A, ks * ks, scale);
                weighted_sum_one(A, v, b, h, i, j, heads, H, W, d, ks,
                                 out + idx5(b, h, i, j, heads, H, W, d));
            }
        }
        free(A);
    }
}

void na2d_oracle_forward(const double *q, const double *k, const double *v,
                         const double *rpb, double *out,
                         long B, long heads, long H, long W, long d, long ks, int nthreads)
{
    na2d_oracle_forward_rows(q, k, v, rpb, out, B, heads, H, W, d, ks, 0, B * heads * H, nthreads);
}

/* Full NA_k for a list of n query points pts[4*t .. 4*t+3] = (b, h, i, j);
 * out is [n][d] and, when attn is not NULL, the softmax weights go to
 * attn [n][ks*ks] and the unscaled logits to logits [n][ks*ks] (either may be NULL). */
void na2d_oracle_forward_points(const double *q, const double *k, const double *v,
                                const double *rpb, const int64_t *pts, long n,
                                double *out, double *logits, double *attn,
                                long B, long heads, long H, long W, long d, long ks, int nthreads)
{
    double scale = 1.0 / sqrt((double)d);
    (void)B;
#pragma omp parallel num_threads(threads_for(nthreads))
    {
        double *A = (double *)malloc(sizeof(double) * (size_t)ks * ks);
#pragma omp for schedule(dynamic)
        for (long t = 0; t < n; t++) {
            long b = (long)pts[4 * t], h = (long)pts[4 * t + 1];
            long i = (long)pts[4 * t + 2], j = (long)pts[4 * t + 3];
            logits_one(q, k, rpb, b, h, i, j, heads, H, W, d, ks, A);
            if (logits)
                for (long m = 0; m < ks * ks; m++) logits[(size_t)t * ks * ks + m] = A[m];
            softmax_row(A, ks * ks, scale);
            if (attn)
                for (long m = 0; m < ks * ks; m++) attn[(size_t)t * ks * ks + m] = A[m];
            weighted_sum_one(A, v, b, h, i, j, heads, H, W, d, ks, out + (size_t)t * d);
        }
        free(A);
    }
}

/*
 * Gradients of NA_k: the backward pass of Eqs. (2)-(4).  NATTEN computes
 * "QK+B" and "AV" and the gradients of their backward passes (Qiita write-up,
 * section "NATTEN"); the NAT paper, Sec. 3.2, makes the operator a PyTorch
 * autograd function.  For a scalar loss L with dout = dL/d(out), the chain
 * rule through out = sum_n P_n v_n, P = softmax(z), z = A / sqrt(d),
 * A_n = q . k_n + B_n gives, per query (i, j) and window entry n:
 *
 *   dP_n   = dout . v_n
 *   dz_n   = P_n (dP_n - sum_m P_m dP_m)          (softmax Jacobian)
 *   dA_n   = dz_n / sqrt(d)
 *   dq(i,j)       += sum_n dA_n k_n
 *   dk(r_n, t_n)  += dA_n q(i,j)
 *   dv(r_n, t_n)  += P_n dout(i,j)
 *   drpb[h][r_n - i + ks - 1][t_n - j + ks - 1] += dA_n
 *
 * dout, dq, dk, dv are [B][heads][H][W][d]; drpb is [heads][2ks-1][2ks-1]
 * and may be NULL (no bias gradient).  The (b, h) maps run in parallel; each
 * map accumulates its own bias gradient, and those are summed over b in
 * order at the end.
 */
void na2d_oracle_backward(const double *q, const double *k, const double *v, const double *rpb,
                          const double *dout, double *dq, double *dk, double *dv, double *drpb,
                          long B, long heads, long H, long W, long d, long ks, int nthreads)
{
    long span = 2 * ks - 1, nn = ks * ks, maps = B * heads;
    size_t total = (size_t)maps * H * W * d;
    double scale = 1.0 / sqrt((double)d);
    double *dB = (double *)calloc((size_t)maps * span * span, sizeof(double));
    for (size_t t = 0; t < total; t++) dq[t] = dk[t] = dv[t] = 0.0;
#pragma omp parallel num_threads(threads_for(nthreads))
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)nn);
        double *dP = (double *)malloc(sizeof(double) * (size_t)nn);
#pragma omp for schedule(dynamic)
        for (long bh = 0; bh < maps; bh++) {
            long b = bh / heads, h = bh % heads;
            for (long i = 0; i < H; i++) {
                for (long j = 0; j < W; j++) {
                    long si = na2d_oracle_window_start(i, H, ks);
                    long sj = na2d_oracle_window_start(j, W, ks);
                    size_t qi = idx5(b, h, i, j, heads, H, W, d);
                    logits_one(q, k, rpb, b, h, i, j, heads, H, W, d, ks, P);
                    softmax_row(P, nn, scale);
                    double pdp = 0.0;
                    for (long a = 0; a < ks; a++) {
                        for (long c = 0; c < ks; c++) {
                            long n = a * ks + c;
                            size_t ki = idx5(b, h, si + a, sj + c, heads, H, W, d);
                            double s = 0.0;
                            for (long x = 0; x < d; x++) s += dout[qi + x] * v[ki + x];
                            dP[n] = s;
                            pdp += P[n] * s;
                        }
                    }
                    for (long a = 0; a < ks; a++) {
                        for (long c = 0; c < ks; c++) {
                            long n = a * ks + c;
                            size_t ki = idx5(b, h, si + a, sj + c, heads, H, W, d);
                            double dA = P[n] * (dP[n] - pdp) * scale;
                            for (long x = 0; x < d; x++) {
                                dq[qi + x] += dA * k[ki + x];
                                dk[ki + x] += dA * q[qi + x];
                                dv[ki + x] += P[n] * dout[qi + x];
                            }
                            dB[((size_t)bh * span + (si + a - i + ks - 1)) * span + (sj + c - j + ks - 1)] += dA;
                        }
                    }
                }
            }
        }
        free(P);
        free(dP);
    }
    if (drpb) {
        for (long h = 0; h < heads; h++)
            for (long e = 0; e < span * span; e++) {
                double s = 0.0;
                for (long b = 0; b < B; b++) s += dB[((size_t)(b * heads + h)) * span * span + e];
                drpb[(size_t)h * span * span + e] = s;
            }
    }
    free(dB);
}

/*
 * SASA (stand-alone self-attention): the centred k x k window of every
 * query, with the positions outside the map taken as zero padding.  The NAT
 * paper, Sec. 3.2, calls SASA a special case of NA on a zero-padded input;
 * the Qiita write-up's SASA/NA drawing shows the difference at the borders
 * (SASA's window stays centred and reaches into the padding, NA's is
 * shifted inward).  Per query (i, j), window entry (a, c) is the position
 * (i - ks/2 + a, j - ks/2 + c); there the key and value are the map's when
 * the position is inside the map and zero otherwise, and the bias is the
 * table's entry for that displacement (a - ks/2, c - ks/2) in both cases:
 *
 *   A_n = q . key_n + B[h][a][c],  out = sum_n softmax(A / sqrt(d))_n value_n.
 */
void na2d_oracle_sasa_forward(const double *q, const double *k, const double *v, const double *rpb,
                              double *out, long B, long heads, long H, long W, long d, long ks,
                              int nthreads)
{
    long rows = B * heads * H, span = 2 * ks - 1, nn = ks * ks, half = ks / 2;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel num_threads(threads_for(nthreads))
    {
        double *A = (double *)malloc(sizeof(double) * (size_t)nn);
#pragma omp for schedule(dynamic)
        for (long row = 0; row < rows; row++) {
            long i = row % H, bh = row / H, h = bh % heads, b = bh / heads;
            for (long j = 0; j < W; j++) {
                const double *qv = q + idx5(b, h, i, j, heads, H, W, d);
                for (long a = 0; a < ks; a++) {
                    for (long c = 0; c < ks; c++) {
                        long r = i - half + a, t = j - half + c;
                        double dot = 0.0;
                        if (r >= 0 && r < H && t >= 0 && t < W) {
                            const double *kv = k + idx5(b, h, r, t, heads, H, W, d);
                            for (long x = 0; x < d; x++) dot += qv[x] * kv[x];
                        }
                        double bias = rpb ? rpb[((size_t)h * span + (a - half + ks - 1)) * span + (c - half + ks - 1)]
                                          : 0.0;
                        A[a * ks + c] = dot + bias;
                    }
                }
                softmax_row(A, nn, scale);
                double *o = out + idx5(b, h, i, j, heads, H, W, d);
                for (long x = 0; x < d; x++) o[x] = 0.0;
                for (long a = 0; a < ks; a++) {
                    for (long c = 0; c < ks; c++) {
                        long r = i - half + a, t = j - half + c;
                        if (r < 0 || r >= H || t < 0 || t >= W) continue;  /* zero value */
                        const double *vv = v + idx5(b, h, r, t, heads, H, W, d);
                        for (long x = 0; x < d; x++) o[x] += A[a * ks + c] * vv[x];
                    }
                }
            }
        }
        free(A);
    }
}

/*
 * Neighborhood attention over 1, 2 or 3 axes with dilation.  The NATTEN
 * library supports "1D to 3D" NA (Qiita write-up, section "NATTEN"; NAT
 * Sec. 3.2: 1D and 2D data), and the DiNAT abstract names a dilated NA; the
 * pages give no formula for dilation.  Reading: a dilation dl on an axis of
 * length L splits it into dl interleaved sub-grids (positions = r mod dl),
 * and a query attends within its own sub-grid with NA's clamped window of
 * ka positions:
 *
 *   r = i mod dl,  i' = i div dl,  L' = ceil((L - r) / dl),
 *   start' = clamp(i' - ka/2, 0, L' - ka),  keys at r + (start' + t) dl,
 *   bias index (start' + t) - i' + ka - 1 on that axis.
 *
 * 1D and 2D are the cases with unit extents and kernel sizes on the leading
 * axes; with dl = 1 every axis is plain NA.  Layouts:
 * q, k, v, out [B][heads][L0][L1][L2][d]; rpb [heads][2k0-1][2k1-1][2k2-1]
 * or NULL.  Every sub-grid must hold a window: floor(La / dla) >= ka.
 */
static long axis_start(long i, long L, long ka, long dl, long *r, long *ip)
{
    long rr = i % dl, ii = i / dl, Lp = (L - rr + dl - 1) / dl;
    long s = ii - ka / 2;
    if (s < 0) s = 0;
    if (s > Lp - ka) s = Lp - ka;
    *r = rr;
    *ip = ii;
    return s;
}

void na2d_oracle_nd_forward(const double *q, const double *k, const double *v, const double *rpb, double *out,
                            long B, long heads, long L0, long L1, long L2, long d,
                            long k0, long k1, long k2, long dl0, long dl1, long dl2, int nthreads)
{
    long rows = B * heads * L0 * L1, nn = k0 * k1 * k2;
    long s0 = 2 * k0 - 1, s1 = 2 * k1 - 1, s2 = 2 * k2 - 1;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel num_threads(threads_for(nthreads))
    {
        double *A = (double *)malloc(sizeof(double) * (size_t)nn);
        long *pos = (long *)malloc(sizeof(long) * (size_t)nn);
#pragma omp for schedule(dynamic)
        for (long row = 0; row < rows; row++) {
            long i1 = row % L1, t0 = row / L1, i0 = t0 % L0, bh = t0 / L0, h = bh % heads;
            for (long i2 = 0; i2 < L2; i2++) {
                long r0, r1, r2, p0, p1, p2;
                long st0 = axis_start(i0, L0, k0, dl0, &r0, &p0);
                long st1 = axis_start(i1, L1, k1, dl1, &r1, &p1);
                long st2 = axis_start(i2, L2, k2, dl2, &r2, &p2);
                size_t map = (size_t)bh * L0 * L1 * L2;
                const double *qv = q + (map + ((size_t)i0 * L1 + i1) * L2 + i2) * d;
                long n = 0;
                for (long a = 0; a < k0; a++)
                    for (long b = 0; b < k1; b++)
                        for (long c = 0; c < k2; c++, n++) {
                            long j0 = r0 + (st0 + a) * dl0, j1 = r1 + (st1 + b) * dl1, j2 = r2 + (st2 + c) * dl2;
                            long kp = (long)(map + ((size_t)j0 * L1 + j1) * L2 + j2);
                            const double *kv = k + (size_t)kp * d;
                            double dot = 0.0;
                            for (long x = 0; x < d; x++) dot += qv[x] * kv[x];
                            if (rpb)
                                dot += rpb[(((size_t)h * s0 + (st0 + a - p0 + k0 - 1)) * s1 +
                                            (st1 + b - p1 + k1 - 1)) * s2 + (st2 + c - p2 + k2 - 1)];
                            A[n] = dot;
                            pos[n] = kp;
                        }
                softmax_row(A, nn, scale);
                double *o = out + (map + ((size_t)i0 * L1 + i1) * L2 + i2) * d;
                for (long x = 0; x < d; x++) o[x] = 0.0;
                for (long m = 0; m < nn; m++) {
                    const double *vv = v + (size_t)pos[m] * d;
                    for (long x = 0; x < d; x++) o[x] += A[m] * vv[x];
                }
            }
        }
        free(A);
        free(pos);
    }
}

int na2d_oracle_max_threads(void)
{
    return threads_for(0);
}
