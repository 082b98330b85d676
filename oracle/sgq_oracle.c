/*
 * sgq_oracle.c -- the CPU oracle for the activation-sparse int4 GEMV.
 *
 * TEST INFRASTRUCTURE ONLY: a plain, slow, obviously correct fp64 restatement
 * of the hot path, used to check the CUDA library and to time a CPU baseline.
 * It shares no code with the CUDA library and the library never calls it.
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 *
 * Sources, by page and section:
 *   [P1] "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract.
 *   [P5] "SVD Contextual Sparsity Predictors for Fast LLM Inference", Abstract.
 *
 * Every floating-point step is a single IEEE double operation (no contraction),
 * so results do not depend on the compiler.
 */
#include "sgq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <stddef.h>
#include <stdint.h>

/* ------------------------------------------------------------------------- */
/* Number formats.                                                           */
/* ------------------------------------------------------------------------- */

/* Round a >= 0 (finite) to the nearest number that has p significant bits and
 * an exponent no lower than emin (values below 2^emin share the quantum of the
 * lowest normal binade, i.e. they become subnormals). Ties go to even. */
static double round_to_grid(double a, int p, int emin)
{
    if (a == 0.0)
        return 0.0;
    int e;
    frexp(a, &e);            /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < emin)
        E = emin;
    double quantum = ldexp(1.0, E - (p - 1));
    return nearbyint(a / quantum) * quantum; /* a / quantum is exact */
}

/* Encode a value that is already on the grid of a format with p significant
 * bits, minimum normal exponent emin and exponent bias 'bias'. */
static uint32_t encode_on_grid(double a, int p, int emin, int bias)
{
    if (a == 0.0)
        return 0;
    if (a < ldexp(1.0, emin))          /* subnormal: a = m * 2^(emin-p+1) */
        return (uint32_t)(a / ldexp(1.0, emin - (p - 1)));
    int e;
    double f = frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) */
    uint32_t m = (uint32_t)(f * ldexp(1.0, p)) - (1u << (p - 1));
    return ((uint32_t)(e - 1 + bias) << (p - 1)) | m;
}

double oracle_half_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 15 - 10);
    return sign ? -v : v;
}

uint16_t oracle_double_to_half(double v)
{
    if (isnan(v))
        return 0x7e00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a))
        return sign | 0x7c00;
    a = round_to_grid(a, 11, -14);
    if (a >= 65536.0)                             /* rounded past the largest finite */
        return sign | 0x7c00;
    return sign | (uint16_t)encode_on_grid(a, 11, -14, 15);
}

double oracle_bf16_to_double(uint16_t b)
{
    int sign = b >> 15;
    int e = (b >> 7) & 0xff;
    int m = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);                /* subnormal */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 127 - 7);
    return sign ? -v : v;
}

uint16_t oracle_double_to_bf16(double v)
{
    if (isnan(v))
        return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a))
        return sign | 0x7f80;
    a = round_to_grid(a, 8, -126);
    if (a >= ldexp(1.0, 128))
        return sign | 0x7f80;
    return sign | (uint16_t)encode_on_grid(a, 8, -126, 127);
}

/* ------------------------------------------------------------------------- */
/* Group-wise asymmetric int4 quantization ([P1] Abstract: group-wise low-bit  */
/* quantization is the dominant way to fit the weights).                     */
/* Readings (the page fixes none of these): 4 bits, asymmetric, one group =   */
/* g consecutive input channels of one output row; the range always contains */
/* 0; scale s = fp16(range / 15); zero z = rint(-lo / s) clamped to [0, 15],  */
/* stored as an integer-valued fp16; code q = clamp(rint(w / s) + z, 0, 15);  */
/* rint rounds half to even; a group whose scale is 0 gets s = 1, z = 0.      */
/* ------------------------------------------------------------------------- */

/* Clamp to [0, 15]; a zero (including -0, from -lo when lo = +0) becomes +0,
 * since the zero point and the codes are unsigned integers. */
static double clamp15(double v)
{
    if (v <= 0.0)
        return 0.0;
    if (v > 15.0)
        return 15.0;
    return v;
}

int oracle_quantize(const uint16_t *W, int N, int K, int g,
                    uint8_t *q, uint16_t *s, uint16_t *z)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0)
        return -2;
    int G = K / g;
    for (int n = 0; n < N; ++n) {
        for (int grp = 0; grp < G; ++grp) {
            const uint16_t *wrow = W + (size_t)n * K + (size_t)grp * g;
            double lo = 0.0, hi = 0.0;
            for (int j = 0; j < g; ++j) {
                double w = oracle_half_to_double(wrow[j]);
                if (!isfinite(w))
                    return -1;
                if (w < lo)
                    lo = w;
                if (w > hi)
                    hi = w;
            }
            uint16_t s_bits = oracle_double_to_half((hi - lo) / 15.0);
            double sv = oracle_half_to_double(s_bits);
            double zv;
            if (sv == 0.0) {
                s_bits = 0x3c00; /* 1.0 */
                sv = 1.0;
                zv = 0.0;
            } else {
                zv = clamp15(nearbyint(-lo / sv));
            }
            s[(size_t)n * G + grp] = s_bits;
            z[(size_t)n * G + grp] = oracle_double_to_half(zv);
            for (int j = 0; j < g; ++j) {
                double w = oracle_half_to_double(wrow[j]);
                double c = clamp15(nearbyint(w / sv) + zv);
                q[(size_t)n * K + (size_t)grp * g + j] = (uint8_t)c;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Packed layout, version 1 (the library's own format; the page names a      */
/* sparsity-aware layout for memory locality but does not give it).          */
/* Channel-major: row k of qweight holds the codes of input channel k for    */
/* all N outputs, so skipping channel k skips one run of N/2 bytes.          */
/*   qweight[k][b] = q[2b][k] | q[2b+1][k] << 4                              */
/*   sz[grp][n][0] = s[n][grp],  sz[grp][n][1] = z[n][grp]                   */
/* ------------------------------------------------------------------------- */

int oracle_pack_layout(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                       int N, int K, int g, uint8_t *qweight, uint16_t *sz)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || N % 2 != 0)
        return -2;
    int G = K / g;
    for (int k = 0; k < K; ++k)
        for (int b = 0; b < N / 2; ++b) {
            uint8_t lo = q[(size_t)(2 * b) * K + k];
            uint8_t hi = q[(size_t)(2 * b + 1) * K + k];
            qweight[(size_t)k * (N / 2) + b] = (uint8_t)(lo | (hi << 4));
        }
    for (int grp = 0; grp < G; ++grp)
        for (int n = 0; n < N; ++n) {
            sz[((size_t)grp * N + n) * 2 + 0] = s[(size_t)n * G + grp];
            sz[((size_t)grp * N + n) * 2 + 1] = z[(size_t)n * G + grp];
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Static 2:4 weight sparsity composed with activation sparsity ([P3]        */
/* "SparseDecoding: Decoding-Aware Pruning for Accurate and Efficient LLM     */
/* Inference", Abstract: an N:M sparse matrix-vector product with bitmask    */
/* indexing). Reading: the 2:4 blocks run along the outputs of each channel  */
/* row and the g channels of a quantization group share the choice; in each */
/* (group, block of 4 outputs) the 2 outputs with the largest sum of w^2     */
/* over the group are kept, equal sums keeping the lower output. A block     */
/* holding NaN/Inf keeps outputs 0 and 1 with zero codes (s = 1, z = 0).     */
/* ------------------------------------------------------------------------- */

int oracle_nm_keep(const uint16_t *W, int N, int K, int g, uint8_t *keep, uint8_t *bad)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || N % 4 != 0)
        return -2;
    int G = K / g;
    for (int grp = 0; grp < G; ++grp)
        for (int j = 0; j < N / 4; ++j) {
            double e[4];
            int nonfinite = 0;
            for (int i = 0; i < 4; ++i) {
                double acc = 0.0;
                for (int r = 0; r < g; ++r) {
                    double w = oracle_half_to_double(W[(size_t)(4 * j + i) * K + (size_t)grp * g + r]);
                    if (!isfinite(w))
                        nonfinite = 1;
                    acc += w * w;
                }
                e[i] = acc;
            }
            uint8_t nib = 0x3;
            if (!nonfinite) {
                int first = -1, second = -1;
                for (int i = 0; i < 4; ++i) {
                    if (first < 0 || e[i] > e[first]) {
                        second = first;
                        first = i;
                    } else if (second < 0 || e[i] > e[second]) {
                        second = i;
                    }
                }
                nib = (uint8_t)((1u << first) | (1u << second));
            }
            keep[(size_t)grp * (N / 4) + j] = nib;
            bad[(size_t)grp * (N / 4) + j] = (uint8_t)nonfinite;
        }
    return 0;
}

int oracle_pack_layout_nm(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                          const uint8_t *keep, const uint8_t *bad, int N, int K, int g,
                          uint8_t *qweight, uint8_t *keep_packed, uint16_t *sz)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || N % 8 != 0)
        return -2;
    int G = K / g;
    for (int grp = 0; grp < G; ++grp) {
        for (int j = 0; j < N / 4; ++j) {
            uint8_t nib = keep[(size_t)grp * (N / 4) + j];
            int isbad = bad[(size_t)grp * (N / 4) + j];
            int out[2], h = 0;
            for (int i = 0; i < 4 && h < 2; ++i)
                if (nib & (1u << i))
                    out[h++] = 4 * j + i;
            if (h != 2)
                return -2;
            for (h = 0; h < 2; ++h) {
                size_t slot = (size_t)grp * (N / 2) + 2 * j + h;
                sz[slot * 2 + 0] = isbad ? (uint16_t)0x3c00 : s[(size_t)out[h] * G + grp];
                sz[slot * 2 + 1] = isbad ? (uint16_t)0 : z[(size_t)out[h] * G + grp];
            }
            for (int r = 0; r < g; ++r) {
                int k = grp * g + r;
                uint8_t c0 = isbad ? 0 : q[(size_t)out[0] * K + k];
                uint8_t c1 = isbad ? 0 : q[(size_t)out[1] * K + k];
                qweight[(size_t)k * (N / 4) + j] = (uint8_t)(c0 | (c1 << 4));
            }
        }
        for (int jj = 0; jj < N / 8; ++jj)
            keep_packed[(size_t)grp * (N / 8) + jj] =
                (uint8_t)(keep[(size_t)grp * (N / 4) + 2 * jj] |
                          (keep[(size_t)grp * (N / 4) + 2 * jj + 1] << 4));
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Active set ([P1] Abstract: dynamic sparsity, runtime gathering of the     */
/* sparse indices; [P5] Abstract: ReGLU neurons that are zero are skipped).  */
/* Readings: channel k is active when |x[k]| > t (strict), so t = 0 keeps    */
/* exactly the nonzero channels; NaN is never active; indices ascend; for a  */
/* batch the active set is the union over rows.                              */
/* ------------------------------------------------------------------------- */

int oracle_select(const uint16_t *x, int B, int K, const float *t,
                  int32_t *idx, int32_t *count)
{
    if (B <= 0 || K <= 0)
        return -2;
    int32_t c = 0;
    for (int k = 0; k < K; ++k) {
        int active = 0;
        for (int b = 0; b < B; ++b) {
            double a = fabs(oracle_bf16_to_double(x[(size_t)b * K + k]));
            if (a > (double)t[b])
                active = 1;
        }
        if (active)
            idx[c++] = k;
    }
    *count = c;
    return 0;
}

/* The same active set as a bitmask: bit k % 32 of word k / 32 set exactly for
 * k in S (the bitmask indexing of "SparseDecoding: Decoding-Aware Pruning for
 * Accurate and Efficient LLM Inference", Abstract). */
int oracle_select_mask(const uint16_t *x, int B, int K, const float *t,
                       uint32_t *mask, int32_t *count)
{
    if (B <= 0 || K <= 0)
        return -2;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    if (!idx)
        return -3;
    int32_t c = 0;
    int rc = oracle_select(x, B, K, t, idx, &c);
    if (rc == 0) {
        for (int w = 0; w < (K + 31) / 32; ++w)
            mask[w] = 0u;
        for (int32_t i = 0; i < c; ++i)
            mask[idx[i] / 32] |= 1u << (idx[i] % 32);
        *count = c;
    }
    free(idx);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* The sparse GEMV: y = W_deq[:, S] x[S] with W_deq[n][k] = s (q - z) of the  */
/* group of k ([P1] Abstract: a GEMV over the quantized weights restricted   */
/* to the active channels). Every row of a batch uses the same active set.   */
/* ------------------------------------------------------------------------- */

/* Output n of batch row b over the listed channels, in list order. */
static void gemv_output(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                        int N, int K, int g, const uint16_t *x, int b, int n,
                        const int32_t *idx, int count,
                        double *y, double *sumabs, uint16_t *y_bf16)
{
    int G = K / g;
    double acc = 0.0, acc_abs = 0.0;
    for (int i = 0; i < count; ++i) {
        int k = idx[i];
        int grp = k / g;
        double sv = oracle_half_to_double(s[(size_t)n * G + grp]);
        double zv = oracle_half_to_double(z[(size_t)n * G + grp]);
        double w = sv * ((double)q[(size_t)n * K + k] - zv);
        double p = w * oracle_bf16_to_double(x[(size_t)b * K + k]);
        acc += p;
        acc_abs += fabs(p);
    }
    size_t o = (size_t)b * N + n;
    if (y)
        y[o] = acc;
    if (sumabs)
        sumabs[o] = acc_abs;
    if (y_bf16)
        y_bf16[o] = oracle_double_to_bf16(acc);
}

static int gemv_args_ok(int N, int K, int g, int B, const int32_t *idx, int count)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || B <= 0 || count < 0 || count > K)
        return -2;
    for (int i = 0; i < count; ++i)
        if (idx[i] < 0 || idx[i] >= K)
            return -3;
    return 0;
}

int oracle_gemv(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                int N, int K, int g, const uint16_t *x, int B,
                const int32_t *idx, int count,
                double *y, double *sumabs, uint16_t *y_bf16)
{
    int rc = gemv_args_ok(N, K, g, B, idx, count);
    if (rc)
        return rc;
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n)
            gemv_output(q, s, z, N, K, g, x, b, n, idx, count, y, sumabs, y_bf16);
    return 0;
}

/* The same GEMV with the outputs shared out over `threads` OpenMP threads.
 * Each output is still one sum in list order by one thread, so the results
 * are bit-identical to oracle_gemv; only the wall time changes. */
int oracle_gemv_threads(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                        int N, int K, int g, const uint16_t *x, int B,
                        const int32_t *idx, int count,
                        double *y, double *sumabs, uint16_t *y_bf16, int threads)
{
    int rc = gemv_args_ok(N, K, g, B, idx, count);
    if (rc)
        return rc;
    if (threads < 1)
        return -2;
    long long total = (long long)B * N;
#pragma omp parallel for num_threads(threads) schedule(static)
    for (long long o = 0; o < total; ++o)
        gemv_output(q, s, z, N, K, g, x, (int)(o / N), (int)(o % N), idx, count, y, sumabs,
                    y_bf16);
    return 0;
}

int oracle_gemv_dense(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                      int N, int K, int g, const uint16_t *x, int B,
                      double *y, double *sumabs, uint16_t *y_bf16)
{
    if (N <= 0 || K <= 0 || g <= 0 || K % g != 0 || B <= 0)
        return -2;
    int G = K / g;
    for (int b = 0; b < B; ++b) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, acc_abs = 0.0;
            for (int k = 0; k < K; ++k) {
                int grp = k / g;
                double sv = oracle_half_to_double(s[(size_t)n * G + grp]);
                double zv = oracle_half_to_double(z[(size_t)n * G + grp]);
                double w = sv * ((double)q[(size_t)n * K + k] - zv);
                double p = w * oracle_bf16_to_double(x[(size_t)b * K + k]);
                acc += p;
                acc_abs += fabs(p);
            }
            size_t o = (size_t)b * N + n;
            if (y)
                y[o] = acc;
            if (sumabs)
                sumabs[o] = acc_abs;
            if (y_bf16)
                y_bf16[o] = oracle_double_to_bf16(acc);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Gated activation between the up/gate and down projections of an FFN       */
/* ([P5] Abstract: ReGLU FFNs, whose ReLU zeros are the skipped neurons).    */
/* h = act(gate) * up; SiLU(v) = v / (1 + e^-v); ReLU(v) = v if v > 0 else 0. */
/* ------------------------------------------------------------------------- */

/* act(g) of the gated FFN: SiLU g / (1 + e^-g) or ReLU max(g, 0) ([P5]
 * Abstract for ReLU gating; SiLU is the Llama / Qwen gate). */
static double oracle_act(double gv, int act)
{
    if (act == 0)
        return gv / (1.0 + exp(-gv));
    return (gv > 0.0) ? gv : 0.0;
}

int oracle_glu(const uint16_t *gate, const uint16_t *up, int64_t n, int act,
               double *h, uint16_t *h_bf16)
{
    if (n < 0 || (act != 0 && act != 1))
        return -2;
    for (int64_t i = 0; i < n; ++i) {
        double gv = oracle_bf16_to_double(gate[i]);
        double uv = oracle_bf16_to_double(up[i]);
        double hv = oracle_act(gv, act) * uv;
        if (h)
            h[i] = hv;
        if (h_bf16)
            h_bf16[i] = oracle_double_to_bf16(hv);
    }
    return 0;
}

int oracle_act_mul(const double *gate, const double *up, int64_t n, int act,
                   double *h, uint16_t *h_bf16)
{
    if (n < 0 || (act != 0 && act != 1))
        return -2;
    for (int64_t i = 0; i < n; ++i) {
        double hv = oracle_act(gate[i], act) * up[i];
        if (h)
            h[i] = hv;
        if (h_bf16)
            h_bf16[i] = oracle_double_to_bf16(hv);
    }
    return 0;
}
