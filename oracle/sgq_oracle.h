/*
 * sgq_oracle.h -- the CPU oracle for the activation-sparse int4 GEMV.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, fp64 restatement of what
 * the hot path computes. Only the test suite, the smoke check and the CPU
 * baseline leg of bench.py may load it. The product library (libsgq) shares
 * no code with it and never calls it.
 *
 * Sources, by page and section:
 *   [P1] "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract:
 *        group-wise low-bit weight quantization; dynamic activation sparsity
 *        (only part of the network contributes for a given input); a GEMV that
 *        works on the quantized layout; runtime gathering of sparse indices.
 *   [P5] "SVD Contextual Sparsity Predictors for Fast LLM Inference", Abstract:
 *        ReGLU feed-forward blocks whose inactive (zero) neurons are skipped by
 *        conditional computation.
 *
 * Readings taken where the pages are silent are listed beside each function.
 * All buffers are host memory owned by the caller.
 */
#ifndef SGQ_ORACLE_H
#define SGQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE binary16 and bfloat16 <-> double. Decoding is exact; encoding rounds to
 * nearest, ties to even, straight from double (one rounding). */
double   oracle_half_to_double(uint16_t h);
uint16_t oracle_double_to_half(double v);
double   oracle_bf16_to_double(uint16_t b);
uint16_t oracle_double_to_bf16(double v);

/* Group-wise asymmetric 4-bit quantization of W (fp16, [N][K] row-major).
 * Outputs: q [N][K] codes 0..15, s and z [N][K/g] as fp16 bit patterns.
 * Returns 0, -1 if W holds a NaN or infinity, -2 on a bad shape. */
int oracle_quantize(const uint16_t *W, int N, int K, int g,
                    uint8_t *q, uint16_t *s, uint16_t *z);

/* Lays the codes out in the channel-major packed format (layout version 1):
 * qweight [K][N/2] bytes, sz [K/g][N][2] fp16 (scale, zero). */
int oracle_pack_layout(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                       int N, int K, int g, uint8_t *qweight, uint16_t *sz);

/* 2:4 weight sparsity along the outputs, shared by the g channels of a group:
 * keep [K/g][N/4] nibbles (bit i = output 4j + i kept; the 2 largest sums of
 * w^2 over the group, ties to the lower output), bad [K/g][N/4] = 1 where the
 * block holds NaN/Inf (then keep = 0x3). */
int oracle_nm_keep(const uint16_t *W, int N, int K, int g, uint8_t *keep, uint8_t *bad);

/* The 2:4 packed layout from the codes of oracle_quantize and the keep choice:
 * qweight [K][N/4] (byte j = slot 2j | slot 2j+1 << 4, slots = kept outputs of
 * block j ascending), keep_packed [K/g][N/8] (block 2jj | block 2jj+1 << 4),
 * sz [K/g][N/2][2] fp16 (scale, zero) per slot; bad blocks get zero codes
 * with s = 1, z = 0. */
int oracle_pack_layout_nm(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                          const uint8_t *keep, const uint8_t *bad, int N, int K, int g,
                          uint8_t *qweight, uint8_t *keep_packed, uint16_t *sz);

/* Active set of a bf16 activation batch x [B][K] against thresholds t[B]:
 * idx <- ascending unique k with |x[b][k]| > t[b] for some b; *count <- size. */
int oracle_select(const uint16_t *x, int B, int K, const float *t,
                  int32_t *idx, int32_t *count);

/* The same set as a bitmask: mask [(K + 31) / 32] words, bit k % 32 of word
 * k / 32 set exactly when k is in S; *count <- |S|. */
int oracle_select_mask(const uint16_t *x, int B, int K, const float *t,
                       uint32_t *mask, int32_t *count);

/* y[b][n] = sum over the listed k of W_deq[n][k] * x[b][k], in fp64, ascending
 * k. Also returns sumabs[b][n] = sum of |W_deq[n][k] * x[b][k]| over the same
 * k, and y rounded to bf16. Any of y, sumabs, y_bf16 may be NULL. */
int oracle_gemv(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                int N, int K, int g, const uint16_t *x, int B,
                const int32_t *idx, int count,
                double *y, double *sumabs, uint16_t *y_bf16);

/* oracle_gemv with the B * N outputs shared out over `threads` OpenMP
 * threads; every output keeps its sum order, so the results are identical. */
int oracle_gemv_threads(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                        int N, int K, int g, const uint16_t *x, int B,
                        const int32_t *idx, int count,
                        double *y, double *sumabs, uint16_t *y_bf16, int threads);

/* Same with every k of 0..K-1 (the dense quantized GEMV). */
int oracle_gemv_dense(const uint8_t *q, const uint16_t *s, const uint16_t *z,
                      int N, int K, int g, const uint16_t *x, int B,
                      double *y, double *sumabs, uint16_t *y_bf16);

/* Gated activation h = act(gate) * up over n elements (bf16 in).
 * act 0 = SiLU, 1 = ReLU. h in fp64 and rounded to bf16 (either may be NULL). */
int oracle_glu(const uint16_t *gate, const uint16_t *up, int64_t n, int act,
               double *h, uint16_t *h_bf16);

/* The same on fp64 gate and up (the unrounded sums of the gate and up
 * projections of one FFN): h = act(gate) * up in fp64, and rounded to bf16. */
int oracle_act_mul(const double *gate, const double *up, int64_t n, int act,
                   double *h, uint16_t *h_bf16);

#ifdef __cplusplus
}
#endif
#endif
