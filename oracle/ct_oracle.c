/*
 * ct_oracle.c -- fp64 CPU oracle for ONNX ConvTranspose.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  The CUDA product path
 * never links, loads or calls it, and it shares no code with that path.
 *
 * What it computes (ai.onnx.ConvTranspose README, "Description" and the
 * "Inputs"/"Attributes" tables; ClikaRT::ops::conv_transpose, the layout
 * paragraph): the transpose of a convolution.  Written out as a scatter, for
 * every batch n, group g, in-channel c of group g, out-channel ml of group g,
 * input position i and kernel tap k:
 *
 *     o_a = i_a * stride_a - pad_begin_a + k_a * dilation_a      (each axis a)
 *     if 0 <= o_a < out_a on every axis:
 *         Y[n, g*M/G + ml, o] += X[n, c, i] * W[c, ml, k]
 *
 * followed by Y[n, m, :] += B[m] when a bias is given.  Alongside Y it
 * accumulates A[n, m, o] = sum |X * W| over the same terms, which scales the
 * acceptance tolerance.
 *
 * Layouts are channels-first and dense row-major: X[N, C, D1..Dr],
 * W[C, M/G, k1..kr], Y[N, M, out1..outr].  All values are fp64.  Resolution
 * of pads and output sizes is the caller's job (oracle/resolver.py).
 *
 * The loop is a plain scatter with no blocking or reordering; OpenMP splits
 * it over independent (n, m) output planes, each owned by one thread.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Pad a rank-r geometry to three axes: missing leading axes have size 1,
 * kernel 1, stride 1, dilation 1, pad 0 and out 1, which leaves the scatter
 * unchanged. */
static void widen3(int rank, const int64_t *src, int64_t fill, int64_t dst[3])
{
    for (int a = 0; a < 3; ++a) dst[a] = fill;
    for (int a = 0; a < rank; ++a) dst[3 - rank + a] = src[a];
}

int ct_oracle_conv_transpose(int rank, int64_t N, int64_t C, int64_t M, int64_t G,
                             const int64_t *in_, const int64_t *k_, const int64_t *s_,
                             const int64_t *d_, const int64_t *pb_, const int64_t *out_,
                             const double *x, const double *w, const double *bias,
                             double *y, double *absy)
{
    if (rank < 1 || rank > 3 || G <= 0 || C % G != 0 || M % G != 0) return 1;
    int64_t in[3], k[3], s[3], d[3], pb[3], out[3];
    widen3(rank, in_, 1, in);
    widen3(rank, k_, 1, k);
    widen3(rank, s_, 1, s);
    widen3(rank, d_, 1, d);
    widen3(rank, pb_, 0, pb);
    widen3(rank, out_, 1, out);

    const int64_t Cg = C / G, Mg = M / G;
    const int64_t in_sz = in[0] * in[1] * in[2];
    const int64_t k_sz = k[0] * k[1] * k[2];
    const int64_t out_sz = out[0] * out[1] * out[2];

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            const int64_t g = m / Mg, ml = m % Mg;
            double *yp = y + (n * M + m) * out_sz;
            double *ap = absy + (n * M + m) * out_sz;
            memset(yp, 0, (size_t)out_sz * sizeof(double));
            memset(ap, 0, (size_t)out_sz * sizeof(double));
            for (int64_t cl = 0; cl < Cg; ++cl) {
                const int64_t c = g * Cg + cl;
                const double *xp = x + (n * C + c) * in_sz;
                const double *wp = w + (c * Mg + ml) * k_sz;
                for (int64_t i0 = 0; i0 < in[0]; ++i0)
                for (int64_t i1 = 0; i1 < in[1]; ++i1)
                for (int64_t i2 = 0; i2 < in[2]; ++i2) {
                    const double xv = xp[(i0 * in[1] + i1) * in[2] + i2];
                    for (int64_t k0 = 0; k0 < k[0]; ++k0) {
                        const int64_t o0 = i0 * s[0] - pb[0] + k0 * d[0];
                        if (o0 < 0 || o0 >= out[0]) continue;
                        for (int64_t k1 = 0; k1 < k[1]; ++k1) {
                            const int64_t o1 = i1 * s[1] - pb[1] + k1 * d[1];
                            if (o1 < 0 || o1 >= out[1]) continue;
                            for (int64_t k2 = 0; k2 < k[2]; ++k2) {
                                const int64_t o2 = i2 * s[2] - pb[2] + k2 * d[2];
                                if (o2 < 0 || o2 >= out[2]) continue;
                                const double p = xv * wp[(k0 * k[1] + k1) * k[2] + k2];
                                const int64_t o = (o0 * out[1] + o1) * out[2] + o2;
                                yp[o] += p;
                                ap[o] += fabs(p);
                            }
                        }
                    }
                }
            }
            if (bias) {
                for (int64_t o = 0; o < out_sz; ++o) yp[o] += bias[m];
            }
        }
    }
    return 0;
}

/*
 * The same definition evaluated at selected output points, for outputs too
 * large to scatter in full.  A point (n, m, o) receives exactly the terms of
 * the scatter above whose landing position is o: those (c, i, k) with
 * i_a * stride_a - pad_begin_a + k_a * dilation_a == o_a on every axis.  For
 * each tap k that means i_a = (o_a + pad_begin_a - k_a * dilation_a) / stride_a
 * when the division is exact and 0 <= i_a < in_a.
 *
 * pts holds npts rows of (2 + rank) int64: n, m, o_1..o_r.
 */
int ct_oracle_points(int rank, int64_t N, int64_t C, int64_t M, int64_t G,
                     const int64_t *in_, const int64_t *k_, const int64_t *s_,
                     const int64_t *d_, const int64_t *pb_, const int64_t *out_,
                     const double *x, const double *w, const double *bias,
                     const int64_t *pts, int64_t npts, double *yv, double *av)
{
    if (rank < 1 || rank > 3 || G <= 0 || C % G != 0 || M % G != 0) return 1;
    int64_t in[3], k[3], s[3], d[3], pb[3], out[3];
    widen3(rank, in_, 1, in);
    widen3(rank, k_, 1, k);
    widen3(rank, s_, 1, s);
    widen3(rank, d_, 1, d);
    widen3(rank, pb_, 0, pb);
    widen3(rank, out_, 1, out);
    const int64_t Cg = C / G, Mg = M / G;
    const int64_t in_sz = in[0] * in[1] * in[2];
    const int64_t k_sz = k[0] * k[1] * k[2];

    for (int64_t p = 0; p < npts; ++p) {
        const int64_t *pt = pts + p * (2 + rank);
        const int64_t n = pt[0], m = pt[1];
        int64_t o[3] = {0, 0, 0};
        for (int a = 0; a < rank; ++a) o[3 - rank + a] = pt[2 + a];
        if (n < 0 || n >= N || m < 0 || m >= M) return 2;
        for (int a = 0; a < 3; ++a)
            if (o[a] < 0 || o[a] >= out[a]) return 2;
        const int64_t g = m / Mg, ml = m % Mg;
        double acc = 0.0, aacc = 0.0;
        for (int64_t cl = 0; cl < Cg; ++cl) {
            const int64_t c = g * Cg + cl;
            const double *xp = x + (n * C + c) * in_sz;
            const double *wp = w + (c * Mg + ml) * k_sz;
            for (int64_t k0 = 0; k0 < k[0]; ++k0) {
                const int64_t t0 = o[0] + pb[0] - k0 * d[0];
                if (t0 % s[0] != 0) continue;
                const int64_t i0 = t0 / s[0];
                if (i0 < 0 || i0 >= in[0]) continue;
                for (int64_t k1 = 0; k1 < k[1]; ++k1) {
                    const int64_t t1 = o[1] + pb[1] - k1 * d[1];
                    if (t1 % s[1] != 0) continue;
                    const int64_t i1 = t1 / s[1];
                    if (i1 < 0 || i1 >= in[1]) continue;
                    for (int64_t k2 = 0; k2 < k[2]; ++k2) {
                        const int64_t t2 = o[2] + pb[2] - k2 * d[2];
                        if (t2 % s[2] != 0) continue;
                        const int64_t i2 = t2 / s[2];
                        if (i2 < 0 || i2 >= in[2]) continue;
                        const double v = xp[(i0 * in[1] + i1) * in[2] + i2] *
                                         wp[(k0 * k[1] + k1) * k[2] + k2];
                        acc += v;
                        aacc += fabs(v);
                    }
                }
            }
        }
        if (bias) acc += bias[m];
        yv[p] = acc;
        av[p] = aacc;
    }
    return 0;
}
