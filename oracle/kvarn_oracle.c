/*
 * kvarn_oracle.c -- plain, slow, fp64 CPU oracle for the KVarN hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or constant generator with the CUDA path.
 *
 * Sources (web pages about the paper "KVarN: Variance-Normalized KV-Cache
 * Quantization Mitigates Error Accumulation in Reasoning Tasks"):
 *   [abs]  codewithpapers.app paper record, abstract: a Hadamard rotation, then
 *          a variance normalisation with two scales, one along the token axis
 *          and one along the channel axis, of K and of V, then 2-bit codes.
 *   [how]  rndamp.com article, section "How It Works", item 1 (Hadamard
 *          transform in the channel dimension, O(N log N) online) and item 2
 *          (iterative algorithm balancing the rows and columns so that the
 *          variance is approximately uniform before quantisation).
 *   [num]  rndamp.com article, section "Numbers": two scales per value, the
 *          second one fused into the dequantisation kernel.
 * Parameters the pages leave open are fixed by the build specification:
 * 128-token blocks, 4 sweeps, 2-bit asymmetric round-to-nearest with a
 * per-group scale and min over 32 channels, fp16 scales, bf16 residual tail.
 *
 * Every routine is the plain definition, written for a reader to check by
 * eye: the rotation is the explicit O(n^2) matrix-vector product with the
 * Sylvester Hadamard matrix (the FWHT is only a fast way to compute it), the
 * variances are two-pass population variances, attention is an explicit
 * softmax.  Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread -lm.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

/* ------------------------------------------------------------------ */
/* Rotation [how, item 1; abs]                                         */
/* ------------------------------------------------------------------ */

/* Sylvester-ordered Hadamard entry H_n[i][j] = (-1)^popcount(i & j). */
static int kvo_hsign(int i, int j)
{
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* Unnormalised Sylvester Hadamard matrix of order n, row-major n x n. */
void kvo_hadamard_matrix(int n, double *H)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            H[i * n + j] = (double)kvo_hsign(i, j);
}

/*
 * Rotate one D-channel vector: y = blockdiag(H_hb, ..., H_hb) x / sqrt(hb).
 * hb is the Hadamard block (hb == D for a full rotation, hb == 32 gives the
 * three-block rotation used at D = 96); hb == 0 means no rotation.
 * The normalised H_hb / sqrt(hb) is symmetric and orthogonal, so the same
 * routine also undoes the rotation.
 */
void kvo_rotate(const double *x, int D, int hb, double *y)
{
    if (hb == 0) {
        memcpy(y, x, sizeof(double) * (size_t)D);
        return;
    }
    const double norm = 1.0 / sqrt((double)hb);
    for (int b = 0; b < D; b += hb) {
        for (int i = 0; i < hb; ++i) {
            double acc = 0.0;
            for (int j = 0; j < hb; ++j)
                acc += (double)kvo_hsign(i, j) * x[b + j];
            y[b + i] = acc * norm;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Dual-axis variance normalisation [how, item 2; abs]                 */
/* ------------------------------------------------------------------ */

/*
 * A variance at most this fraction of the mean square counts as zero: the
 * values agree to about 2^-20 of their size, below what the scales can
 * resolve (a difference that small only arises from rounding, and whether
 * it survives depends on the working precision, not on the data).
 */
#define KVO_ZERO_VAR_REL 0x1p-40

/*
 * Population standard deviation of n values, or 0 when their variance is
 * zero (KVO_ZERO_VAR_REL).  The variance does not change when every value
 * is shifted by the same amount, so it is taken of z_i - z_0 (two passes:
 * mean, then the mean square deviation).  The shift makes a constant
 * sequence give exactly zero, whatever rounding the mean of equal values
 * would carry.
 */
static double kvo_std_or_zero(const double *z, int n)
{
    const double z0 = z[0];
    double mean = 0.0;
    for (int i = 0; i < n; ++i) mean += z[i] - z0;
    mean /= (double)n;
    double var = 0.0;
    for (int i = 0; i < n; ++i) {
        const double e = (z[i] - z0) - mean;
        var += e * e;
    }
    var /= (double)n;
    const double mz = z0 + mean;             /* mean of the values */
    return var > KVO_ZERO_VAR_REL * (var + mz * mz) ? sqrt(var) : 0.0;
}

/*
 * X is the rotated block, T tokens (rows) x D channels (columns).
 * Start from c = 1.  Each sweep first sets every row scale
 *     r_t = std_d( X[t][d] / c[d] ),
 * then every column scale
 *     c_d = std_t( X[t][d] / r[t] ),
 * then moves the common factor of the channel scales into the token scales:
 *     g = geometric mean of c,  c_d <- c_d / g,  r_t <- r_t * g.
 * Only the products r_t c_d enter Y = X / (r c), and they are unchanged by
 * the last step; without it a block whose tokens share a large common part
 * lets r grow and c shrink by the same factor every sweep, far outside the
 * binary16 range the scales are stored in.
 * A row or column whose variance is zero carries no scale information: it
 * takes scale 1 and stays out of the gauge step (g is the geometric mean of
 * the other channel scales, 1 if there are none; such rows are not
 * multiplied by g).
 * After the last sweep every column of X / (r c) with nonzero variance has
 * variance exactly 1, the row variances are close to uniform and the channel
 * scales have geometric mean 1.  sweeps == 0 leaves r = c = 1.
 */
void kvo_normalize(const double *X, int T, int D, int sweeps, double *r, double *c)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(T > D ? T : D));
    for (int d = 0; d < D; ++d) c[d] = 1.0;
    for (int t = 0; t < T; ++t) r[t] = 1.0;
    for (int k = 0; k < sweeps; ++k) {
        for (int t = 0; t < T; ++t) {
            for (int d = 0; d < D; ++d) z[d] = X[(size_t)t * D + d] / c[d];
            r[t] = kvo_std_or_zero(z, D);          /* 0 marks a zero-variance row */
        }
        for (int d = 0; d < D; ++d) {
            for (int t = 0; t < T; ++t) z[t] = X[(size_t)t * D + d] / (r[t] > 0.0 ? r[t] : 1.0);
            c[d] = kvo_std_or_zero(z, T);          /* 0 marks a zero-variance column */
        }
        double lsum = 0.0;
        int n = 0;
        for (int d = 0; d < D; ++d)
            if (c[d] > 0.0) { lsum += log(c[d]); ++n; }
        const double g = n > 0 ? exp(lsum / (double)n) : 1.0;
        for (int d = 0; d < D; ++d) c[d] = c[d] > 0.0 ? c[d] / g : 1.0;
        for (int t = 0; t < T; ++t) r[t] = r[t] > 0.0 ? r[t] * g : 1.0;
    }
    free(z);
}

/* ------------------------------------------------------------------ */
/* Block quantiser: rotate, normalise, 2-bit asymmetric RTN            */
/* ------------------------------------------------------------------ */

/*
 * Quantise one block X (T x D, token-major) of K or V.
 *   Xrot  (T x D)   rotated block                         (may be NULL)
 *   r (T), c (D)    normalisation scales (unrounded fp64)
 *   s, m (T x D/G)  per-(token, group) step and minimum, G contiguous channels
 *   v (T x D)       pre-rounding level (Y - m) / s        (may be NULL)
 *   codes (T x D)   2-bit codes 0..3, one per byte (unpacked)
 * Y = Xrot / (r_t c_d) with the unrounded scales; within each group
 * m = min Y, s = (max Y - m) / 3, code = clamp(rint((Y - m) / s), 0, 3), and
 * a group with s == 0 gets code 0 everywhere.  The returned r includes the
 * token gauge described below.
 */
void kvo_quantize_block(const double *X, int T, int D, int hb, int sweeps, int G,
                        double *Xrot, double *r, double *c, double *s, double *m,
                        double *v, uint8_t *codes)
{
    double *xr = (double *)malloc(sizeof(double) * (size_t)T * D);
    for (int t = 0; t < T; ++t)
        kvo_rotate(X + (size_t)t * D, D, hb, xr + (size_t)t * D);
    kvo_normalize(xr, T, D, sweeps, r, c);

    const int ng = D / G;
    double *y = (double *)malloc(sizeof(double) * (size_t)G);
    for (int t = 0; t < T; ++t) {
        /* Token gauge: r_t times (s, m) of the token is what dequantises, so a
         * power of two can move between them exactly.  When the token's
         * largest |Y| reaches 2^14, 2^k (k = floor(log2 max|Y|) - 13) moves
         * into r_t, which brings max|Y| into [2^13, 2^14) and keeps s and m
         * inside binary16; Y / 2^k is exact and the codes do not change. */
        double ymax = 0.0;
        for (int d = 0; d < D; ++d) {
            const double a = fabs(xr[(size_t)t * D + d] / (r[t] * c[d]));
            if (a > ymax) ymax = a;
        }
        double tg = 1.0;
        if (ymax >= 16384.0) {
            int e2;
            (void)frexp(ymax, &e2);                 /* ymax = f * 2^e2, f in [0.5, 1) */
            tg = ldexp(1.0, (e2 - 1) - 13);
        }
        for (int g = 0; g < ng; ++g) {
            double lo = INFINITY, hi = -INFINITY;
            for (int i = 0; i < G; ++i) {
                const int d = g * G + i;
                y[i] = xr[(size_t)t * D + d] / (r[t] * c[d]) / tg;
                if (y[i] < lo) lo = y[i];
                if (y[i] > hi) hi = y[i];
            }
            const double step = (hi - lo) / 3.0;
            s[(size_t)t * ng + g] = step;
            m[(size_t)t * ng + g] = lo;
            for (int i = 0; i < G; ++i) {
                const size_t e = (size_t)t * D + (size_t)g * G + i;
                double lvl = 0.0;
                int q = 0;
                if (step > 0.0) {
                    lvl = (y[i] - lo) / step;
                    double rq = rint(lvl);
                    if (rq < 0.0) rq = 0.0;
                    if (rq > 3.0) rq = 3.0;
                    q = (int)rq;
                }
                if (v) v[e] = lvl;
                codes[e] = (uint8_t)q;
            }
        }
        r[t] *= tg;
    }
    if (Xrot) memcpy(Xrot, xr, sizeof(double) * (size_t)T * D);
    free(y);
    free(xr);
}

/* ------------------------------------------------------------------ */
/* IEEE-754 binary16, written from the format's definition             */
/* ------------------------------------------------------------------ */

/* Round a double to the nearest binary16 (ties to even); return its bits. */
uint16_t kvo_f16_bits(double x)
{
    if (isnan(x)) return 0x7E00;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    /* largest finite binary16 is 65504; halfway to the next power is 65520 */
    if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: value = q * 2^-24, q an integer in [0, 1024] */
        double q = rint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q); /* q == 1024 is the smallest normal */
    }
    int e2;
    (void)frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                 /* a = 1.mmm * 2^E */
    double frac = rint((ldexp(a, -E) - 1.0) * 1024.0);
    if (frac >= 1024.0) { frac = 0.0; E += 1; }
    if (E + 15 >= 31) return (uint16_t)(sign | 0x7C00);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)frac);
}

/* Exact value of a binary16 bit pattern. */
double kvo_f16_value(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int E = (h >> 10) & 0x1F;
    const int F = h & 0x3FF;
    double v;
    if (E == 0) v = ldexp((double)F, -24);
    else if (E == 31) v = F ? NAN : INFINITY;
    else v = ldexp(1.0 + (double)F / 1024.0, E - 15);
    return sign ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Packed block record (the cache layout the library writes)           */
/* ------------------------------------------------------------------ */

/*
 * One record per (sequence, kv head, block) and per tensor (K or V):
 *   codes    T*D/4 bytes of 2-bit codes
 *   s        T*(D/G) binary16 steps, token-major  s[t*(D/G) + g]
 *   m        T*(D/G) binary16 minima, token-major m[t*(D/G) + g]
 *   r        T binary16 token scales
 *   c        D binary16 channel scales
 * and zero padding up to a multiple of 128 bytes.
 *
 * Where the codes sit (layout):
 *   0 natural  byte t*D/4 + d/4, bits 2*(d%4)   (any T; oracle-only tests)
 *   1 K order  (T = 128) word w of lane l of 16-token unit u, bit 16*half+2*pos:
 *              u = t/16, l = 4*(t%8) + (d%8)/2, half = d%2, q = d/8, n = (t%16)/8,
 *              F = D/64; q < 8F: w = n*F + q/8, pos = q%8; else w = 2F, pos = q-8F+4n;
 *              word at byte ((u*32 + l)*(D/32) + w)*4
 *   2 V order  (T = 128) j = d/8, l = 4*(d%8) + (t%8)/2, half = t%2, a = (t%32)/8,
 *              w = a/2, pos = 4*(a%2) + t/32; word at byte ((j*32 + l)*2 + w)*4,
 *              bit 16*half+2*pos
 * The library writes K blocks in layout 1 and V blocks in layout 2.
 */
size_t kvo_record_bytes(int T, int D, int G)
{
    size_t b = (size_t)T * D / 4 + (size_t)T * (D / G) * 4 + 2 * (size_t)T + 2 * (size_t)D;
    return (b + 127) / 128 * 128;
}

/* Byte offset and bit (within that byte) of the code of (token t, channel d). */
static void kvo_code_site(int T, int D, int layout, int t, int d, size_t *byte, int *bit)
{
    if (layout == 0) {
        *byte = (size_t)t * D / 4 + d / 4;
        *bit = 2 * (d % 4);
        return;
    }
    size_t word;
    int wbit;
    if (layout == 1) {
        const int u = t / 16, l = 4 * (t % 8) + (d % 8) / 2, half = d % 2, q = d / 8, n = (t % 16) / 8;
        const int F = D / 64;
        int w, pos;
        if (q < 8 * F) { w = n * F + q / 8; pos = q % 8; }
        else { w = 2 * F; pos = q - 8 * F + 4 * n; }
        word = ((size_t)(u * 32 + l) * (D / 32) + w) * 4;
        wbit = 16 * half + 2 * pos;
    } else {
        const int j = d / 8, l = 4 * (d % 8) + (t % 8) / 2, half = t % 2, a = (t % 32) / 8;
        const int w = a / 2, pos = 4 * (a % 2) + t / 32;
        word = ((size_t)(j * 32 + l) * 2 + w) * 4;
        wbit = 16 * half + 2 * pos;
    }
    (void)T;
    *byte = word + wbit / 8;
    *bit = wbit % 8;
}

void kvo_pack_record(int T, int D, int G, int layout, const uint8_t *codes, const double *r,
                     const double *c, const double *s, const double *m, uint8_t *rec)
{
    const int ng = D / G;
    memset(rec, 0, kvo_record_bytes(T, D, G));
    uint8_t *pc = rec;
    uint8_t *ps = pc + (size_t)T * D / 4;
    uint8_t *pm = ps + (size_t)T * ng * 2;
    uint8_t *pr = pm + (size_t)T * ng * 2;
    uint8_t *pcs = pr + 2 * (size_t)T;
    for (int t = 0; t < T; ++t)
        for (int d = 0; d < D; ++d) {
            size_t byte;
            int bit;
            kvo_code_site(T, D, layout, t, d, &byte, &bit);
            pc[byte] |= (uint8_t)((codes[(size_t)t * D + d] & 3) << bit);
        }
    for (size_t i = 0; i < (size_t)T * ng; ++i) {
        uint16_t hs = kvo_f16_bits(s[i]), hm = kvo_f16_bits(m[i]);
        ps[2 * i] = (uint8_t)(hs & 0xFF); ps[2 * i + 1] = (uint8_t)(hs >> 8);
        pm[2 * i] = (uint8_t)(hm & 0xFF); pm[2 * i + 1] = (uint8_t)(hm >> 8);
    }
    for (int t = 0; t < T; ++t) {
        uint16_t h = kvo_f16_bits(r[t]);
        pr[2 * t] = (uint8_t)(h & 0xFF); pr[2 * t + 1] = (uint8_t)(h >> 8);
    }
    for (int d = 0; d < D; ++d) {
        uint16_t h = kvo_f16_bits(c[d]);
        pcs[2 * d] = (uint8_t)(h & 0xFF); pcs[2 * d + 1] = (uint8_t)(h >> 8);
    }
}

static double kvo_load_f16(const uint8_t *p)
{
    return kvo_f16_value((uint16_t)(p[0] | (p[1] << 8)));
}

/*
 * Read a record back: codes (T x D, one per byte) and the stored scales,
 * widened exactly from binary16.
 */
void kvo_unpack_record(int T, int D, int G, int layout, const uint8_t *rec, uint8_t *codes,
                       double *r, double *c, double *s, double *m)
{
    const int ng = D / G;
    const uint8_t *pc = rec;
    const uint8_t *ps = pc + (size_t)T * D / 4;
    const uint8_t *pm = ps + (size_t)T * ng * 2;
    const uint8_t *pr = pm + (size_t)T * ng * 2;
    const uint8_t *pcs = pr + 2 * (size_t)T;
    for (int t = 0; t < T; ++t)
        for (int d = 0; d < D; ++d) {
            size_t byte;
            int bit;
            kvo_code_site(T, D, layout, t, d, &byte, &bit);
            codes[(size_t)t * D + d] = (uint8_t)((pc[byte] >> bit) & 3);
        }
    for (size_t i = 0; i < (size_t)T * ng; ++i) {
        s[i] = kvo_load_f16(ps + 2 * i);
        m[i] = kvo_load_f16(pm + 2 * i);
    }
    for (int t = 0; t < T; ++t) r[t] = kvo_load_f16(pr + 2 * t);
    for (int d = 0; d < D; ++d) c[d] = kvo_load_f16(pcs + 2 * d);
}

/*
 * Dequantise a record [num, second scale fused]:
 *   Xhat_rot[t][d] = r_t * c_d * (s_{t,g} * code + m_{t,g})
 * and, unless rotated != 0, rotate back to the original channel basis.
 */
void kvo_dequantize_record(const uint8_t *rec, int T, int D, int G, int layout, int hb, int rotated,
                           double *Xhat)
{
    const int ng = D / G;
    uint8_t *codes = (uint8_t *)malloc((size_t)T * D);
    double *r = (double *)malloc(sizeof(double) * (size_t)T);
    double *c = (double *)malloc(sizeof(double) * (size_t)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)T * ng);
    double *m = (double *)malloc(sizeof(double) * (size_t)T * ng);
    double *row = (double *)malloc(sizeof(double) * (size_t)D);
    kvo_unpack_record(T, D, G, layout, rec, codes, r, c, s, m);
    for (int t = 0; t < T; ++t) {
        for (int d = 0; d < D; ++d) {
            const int g = d / G;
            row[d] = r[t] * c[d] * (s[(size_t)t * ng + g] * (double)codes[(size_t)t * D + d]
                                    + m[(size_t)t * ng + g]);
        }
        if (rotated) memcpy(Xhat + (size_t)t * D, row, sizeof(double) * (size_t)D);
        else kvo_rotate(row, D, hb, Xhat + (size_t)t * D);
    }
    free(row); free(m); free(s); free(c); free(r); free(codes);
}

/* ------------------------------------------------------------------ */
/* Decode attention over a dequantised cache [abs; num]                */
/* ------------------------------------------------------------------ */

/*
 * Single-token decode attention, explicit softmax:
 *   q    Hq x D
 *   K, V Hkv x L x D   (already dequantised, original basis)
 *   out  Hq x D,  out_h = sum_t softmax_t(scale * q_h . k_t) v_t
 * Query head h reads kv head h / (Hq / Hkv).  L == 0 gives zeros.
 */
void kvo_attention(const double *q, int Hq, int Hkv, int D, int L,
                   const double *K, const double *V, double scale, double *out)
{
    const int grp = Hq / Hkv;
    double *sc = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int h = 0; h < Hq; ++h) {
        const int kh = h / grp;
        const double *Kh = K + (size_t)kh * L * D;
        const double *Vh = V + (size_t)kh * L * D;
        double *o = out + (size_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (L == 0) continue;
        double mx = -INFINITY;
        for (int t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += q[(size_t)h * D + d] * Kh[(size_t)t * D + d];
            sc[t] = acc * scale;
            if (sc[t] > mx) mx = sc[t];
        }
        double den = 0.0;
        for (int t = 0; t < L; ++t) { sc[t] = exp(sc[t] - mx); den += sc[t]; }
        for (int t = 0; t < L; ++t)
            for (int d = 0; d < D; ++d) o[d] += sc[t] * Vh[(size_t)t * D + d];
        for (int d = 0; d < D; ++d) o[d] /= den;
    }
    free(sc);
}

/* ------------------------------------------------------------------ */
/* Many blocks, threaded over independent blocks (CPU baseline)        */
/* ------------------------------------------------------------------ */

/* Widen one input element: dtype 0 = fp32, 1 = bf16 (upper half of fp32). */
static double kvo_load_input(const void *x, int dtype, size_t i)
{
    if (dtype == 0) return (double)((const float *)x)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)x)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *x; int dtype; int64_t nunits; int T, D, hb, sweeps, G, layout;
    uint8_t *records; int nthreads, tid;
} kvo_job;

static void *kvo_worker(void *arg)
{
    kvo_job *j = (kvo_job *)arg;
    const size_t n = (size_t)j->T * j->D, ng = (size_t)j->D / j->G;
    const size_t rb = kvo_record_bytes(j->T, j->D, j->G);
    double *X = (double *)malloc(sizeof(double) * n);
    double *r = (double *)malloc(sizeof(double) * (size_t)j->T);
    double *c = (double *)malloc(sizeof(double) * (size_t)j->D);
    double *s = (double *)malloc(sizeof(double) * (size_t)j->T * ng);
    double *m = (double *)malloc(sizeof(double) * (size_t)j->T * ng);
    uint8_t *codes = (uint8_t *)malloc(n);
    for (int64_t u = j->tid; u < j->nunits; u += j->nthreads) {
        for (size_t i = 0; i < n; ++i) X[i] = kvo_load_input(j->x, j->dtype, (size_t)u * n + i);
        kvo_quantize_block(X, j->T, j->D, j->hb, j->sweeps, j->G, NULL, r, c, s, m, NULL, codes);
        kvo_pack_record(j->T, j->D, j->G, j->layout, codes, r, c, s, m, j->records + (size_t)u * rb);
    }
    free(codes); free(m); free(s); free(c); free(r); free(X);
    return NULL;
}

/*
 * Quantise nunits consecutive T x D input blocks (fp32 or bf16) into packed
 * records with code layout `layout`, on nthreads POSIX threads.  Returns the number of threads used.
 */
int kvo_quantize_many(const void *x, int dtype, int64_t nunits, int T, int D, int hb,
                      int sweeps, int G, int layout, uint8_t *records, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    kvo_job jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (kvo_job){x, dtype, nunits, T, D, hb, sweeps, G, layout, records, nthreads, i};
        pthread_create(&th[i], NULL, kvo_worker, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    return nthreads;
}
