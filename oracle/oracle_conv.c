/*
 * oracle_conv.c -- plain CPU reference for NHWC/NDHWC convolution forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the GPU library is
 * checked against.  Only the test suite, the package smoke check and the
 * bench's CPU-baseline leg load it.  It shares no source, header, table or
 * helper with the CUDA library, and the library never calls it.
 *
 * What it computes (the plain definition of the operation the three MLX pull
 * requests "Bound winograd conv2d working set by tiling the batch",
 * "Use the explicit gemm for wide convs on neural accelerators" and
 * "Decompose small kernel-depth 3D convs into 2D convs" all check their GPU
 * kernels against with a "CPU reference" / "CPU convolution"):
 *
 *   out[n,oh,ow,o] = sum_{kh<KH} sum_{kw<KW} sum_{c<C}
 *                      in[n, oh*sh - ph + kh*dh, ow*sw - pw + kw*dw, c] * w[o,kh,kw,c]
 *
 * with in NHWC, w OHWI, out NHWC, terms whose input index falls outside the
 * image counted as zero (symmetric zero padding), no kernel flip
 * (cross-correlation), groups = 1, and
 *   OH = floor((H + 2*ph - dh*(KH-1) - 1) / sh) + 1   (same for OW).
 * The 3D form adds a depth axis the same way (id = od*sd - pd + kd*dd) over
 * NDHWC inputs and O,KD,KH,KW,I weights; the depth-tap decomposition page
 * ("Decompose small kernel-depth 3D convs into 2D convs", section Change)
 * describes the frames as [OD,H,W,C] and the weight slices as [O,KH,KW,C].
 *
 * Every input element is converted exactly to double (fp32 by value, fp16 and
 * bf16 by decoding their bit patterns here) and every sum is accumulated in
 * double, in the order of the definition: kh, then kw, then c (the depth
 * version: kd, kh, kw, c).  No final rounding.  No -ffast-math.
 *
 * Two modes: the full output tensor, or a list of output pixels
 * ((n,oh,ow) or (n,od,oh,ow)), each with all O channels.  OpenMP over pixels.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double decode_f16(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 10) & 0x1f;
    int f = b & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* zero or subnormal: f * 2^-24 */
    else if (e == 31)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32: widen by a 16-bit shift. */
static double decode_bf16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return (double)x;
}

static double decode_one(int dtype, const void *base, size_t i)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[i];
    if (dtype == ORACLE_F16)
        return decode_f16(((const uint16_t *)base)[i]);
    return decode_bf16(((const uint16_t *)base)[i]);
}

int oracle_decode(int dtype, const void *src, double *dst, long long count)
{
    if (dtype < ORACLE_F32 || dtype > ORACLE_BF16 || count < 0)
        return 1;
    for (long long i = 0; i < count; ++i)
        dst[i] = decode_one(dtype, src, (size_t)i);
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static long long out_extent(long long in, int k, int s, int p, int d)
{
    return (in + 2LL * p - (long long)d * (k - 1) - 1) / s + 1;
}

/*
 * 3D convolution; the 2D entry point is the same sum with D = KD = 1.
 * pixels: NULL for the full tensor (out is [N][OD][OH][OW][O]), else npix
 * quadruples (n, od, oh, ow) and out is [npix][O].
 * Returns 0 on success, 1 for invalid arguments, 2 if memory ran out.
 */
int oracle_conv3d(const void *in, const void *w, int dtype,
                  int N, int D, int H, int W, int C, int O,
                  int KD, int KH, int KW,
                  int sd, int sh, int sw, int pd, int ph, int pw,
                  int dd, int dh, int dw,
                  const int *pixels, long long npix, double *out, int threads)
{
    if (dtype < ORACLE_F32 || dtype > ORACLE_BF16)
        return 1;
    if (N < 0 || D <= 0 || H <= 0 || W <= 0 || C <= 0 || O <= 0 || KD <= 0 || KH <= 0 || KW <= 0)
        return 1;
    if (sd <= 0 || sh <= 0 || sw <= 0 || dd <= 0 || dh <= 0 || dw <= 0 || pd < 0 || ph < 0 || pw < 0)
        return 1;
    long long OD = out_extent(D, KD, sd, pd, dd);
    long long OH = out_extent(H, KH, sh, ph, dh);
    long long OW = out_extent(W, KW, sw, pw, dw);
    if (OD <= 0 || OH <= 0 || OW <= 0)
        return 1;

    const long long K = (long long)KD * KH * KW * C;       /* one weight row */
    double *wd = (double *)malloc(sizeof(double) * (size_t)(K * O));
    if (!wd)
        return 2;
    oracle_decode(dtype, w, wd, K * O);

    long long P = pixels ? npix : (long long)N * OD * OH * OW;
    int failed = 0;

#ifdef _OPENMP
    int nt = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel num_threads(nt) reduction(| : failed)
#endif
    {
        double *win = (double *)malloc(sizeof(double) * (size_t)K);
        if (!win) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
            for (long long p = 0; p < P; ++p) {
                long long n, od, oh, ow;
                if (pixels) {
                    n = pixels[4 * p + 0];
                    od = pixels[4 * p + 1];
                    oh = pixels[4 * p + 2];
                    ow = pixels[4 * p + 3];
                } else {
                    long long r = p;
                    ow = r % OW; r /= OW;
                    oh = r % OH; r /= OH;
                    od = r % OD; r /= OD;
                    n = r;
                }
                if (n < 0 || n >= N || od < 0 || od >= OD || oh < 0 || oh >= OH || ow < 0 || ow >= OW) {
                    for (int o = 0; o < O; ++o)
                        out[p * O + o] = NAN;
                    continue;
                }
                /* The input values the sum touches, in (kd, kh, kw, c) order;
                 * a term whose input index is outside the volume is zero. */
                long long k = 0;
                for (int kd = 0; kd < KD; ++kd) {
                    long long id = od * sd - pd + (long long)kd * dd;
                    for (int kh = 0; kh < KH; ++kh) {
                        long long ih = oh * sh - ph + (long long)kh * dh;
                        for (int kw = 0; kw < KW; ++kw) {
                            long long iw = ow * sw - pw + (long long)kw * dw;
                            int inside = id >= 0 && id < D && ih >= 0 && ih < H && iw >= 0 && iw < W;
                            size_t base = inside ? (size_t)((((n * D + id) * H + ih) * W + iw) * C) : 0;
                            for (int c = 0; c < C; ++c)
                                win[k++] = inside ? decode_one(dtype, in, base + c) : 0.0;
                        }
                    }
                }
                for (int o = 0; o < O; ++o) {
                    const double *wo = wd + (size_t)o * K;
                    double acc = 0.0;
                    for (long long j = 0; j < K; ++j)
                        acc += win[j] * wo[j];
                    out[p * O + o] = acc;
                }
            }
            free(win);
        }
    }
    free(wd);
    return failed ? 2 : 0;
}

/* 2D convolution: pixels are triples (n, oh, ow); full output is [N][OH][OW][O]. */
int oracle_conv2d(const void *in, const void *w, int dtype,
                  int N, int H, int W, int C, int O, int KH, int KW,
                  int sh, int sw, int ph, int pw, int dh, int dw,
                  const int *pixels, long long npix, double *out, int threads)
{
    int *quad = NULL;
    if (pixels) {
        quad = (int *)malloc(sizeof(int) * (size_t)(4 * (npix > 0 ? npix : 1)));
        if (!quad)
            return 2;
        for (long long p = 0; p < npix; ++p) {
            quad[4 * p + 0] = pixels[3 * p + 0];
            quad[4 * p + 1] = 0;
            quad[4 * p + 2] = pixels[3 * p + 1];
            quad[4 * p + 3] = pixels[3 * p + 2];
        }
    }
    int rc = oracle_conv3d(in, w, dtype, N, 1, H, W, C, O, 1, KH, KW,
                           1, sh, sw, 0, ph, pw, 1, dh, dw, quad, npix, out, threads);
    free(quad);
    return rc;
}
