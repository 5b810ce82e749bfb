/*
 * attn_selftest.h -- diagnostic entry point of libattn (not part of the attention
 * API).  It runs the tensor-core building blocks of the forward kernel on one
 * 128-row tile so a test can check each against a plain matrix product:
 *   TMA load of three bf16 [128, d] row-major tiles A, B, V (128-byte swizzle),
 *   S = A B^T with tcgen05.mma from shared memory (K-major A and B), fp32 in TMEM;
 *   P = bf16(S) written back into TMEM;
 *   O = P V with tcgen05.mma, A = P from TMEM, B = V from shared memory (MN-major).
 * a, b, v: DEVICE bf16 [128, d] (16-byte aligned); s_out: DEVICE fp32 [128, 128];
 * o_out: DEVICE fp32 [128, d]; d in {64, 128}.  Asynchronous on `stream`.
 *
 * attn_selftest_umma_e4m3 is the same check for the 8-bit path of attn_fwd_e4m3:
 * a, b, v are DEVICE E4M3 [128, 128] (one byte per element), S = A B^T with
 * tcgen05.mma kind::f8f6f4, P = e4m3(S) (round to nearest even, saturating) in
 * TMEM, O = P V; s_out fp32 [128, 128], o_out fp32 [128, 128].
 *
 * attn_selftest_exp2 evaluates the forward kernel's FMA-pipe exponential 2^x
 * (polynomial with exponent-field scaling; "FlashAttention V4 deep-dive", section
 * 3.2, software exponential on the FMA units) on n DEVICE floats x: y_poly from the
 * packed two-lane form the kernel runs, y_scalar from the scalar form, y_ref from
 * CUDA's exp2f, each a DEVICE fp32 [n].  Asynchronous on `stream`.
 */
#ifndef LIBATTN_ATTN_SELFTEST_H
#define LIBATTN_ATTN_SELFTEST_H
#include "attn.h"
#ifdef __cplusplus
extern "C" {
#endif
ATTN_API attn_status_t attn_selftest_umma(const void* a, const void* b, const void* v, float* s_out,
                                 float* o_out, int d, attn_stream_t stream);
ATTN_API attn_status_t attn_selftest_umma_e4m3(const void* a, const void* b, const void* v,
                                               float* s_out, float* o_out, attn_stream_t stream);
ATTN_API attn_status_t attn_selftest_exp2(const float* x, float* y_poly, float* y_scalar, float* y_ref,
                                          int n, attn_stream_t stream);
#ifdef __cplusplus
}
#endif
#endif
