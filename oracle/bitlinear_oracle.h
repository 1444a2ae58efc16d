/*
 * CPU oracle for the BitLinear W1.58·A8 matmul (BitNet b1.58).
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and
 * the benchmark's CPU-baseline / reference arm may load this library.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Plain, slow, obviously correct: every function follows one definition of
 * the pages and is cited beside it.  Page names used in the citations:
 *   [BitNet 三值权重实战]  "1.58-bit 大模型极限量化实战：从 BitNet 三值权重到
 *                          单颗 CPU 跑起 100B 模型" (chenxutan.com/d/5049.html)
 *   [1.58 位大模型]        nxmr.cn/news/148658 (a flattened single-paragraph page)
 *   [硬件协同优化]         2kiu.com/news/4928193
 *
 * Floating point: IEEE binary32 with round-to-nearest-even, compiled with
 * -ffp-contract=off -fno-fast-math (no fused multiply-add, no reassociation).
 */
#ifndef BITLINEAR_ORACLE_H
#define BITLINEAR_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };

/* Exact Σ|W| as per-exponent integer bins: bins[E] = Σ of the 24-bit
 * significands of the elements whose binary32 biased exponent is E.  The exact
 * sum is Σ_E bins[E]·2^(max(E,1)-150).  Returns 0, or -1 on a non-finite input. */
int orc_abs_exponent_bins(const void* W, int dtype, int64_t count, int64_t bins[256]);

/* Ternary codes ŵ = clip(round(W/α), -1, 1) (round half to even). */
int orc_ternarize(const void* W, int dtype, int64_t count, float alpha, int8_t* codes);

/* Bytes per packed row: 16·ceil(K/64). */
int64_t orc_packed_row_bytes(int64_t K);

/* 2-bit packing of codes [N][K] into packed [N][orc_packed_row_bytes(K)]. */
void orc_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed);

/* Per-token absmax int8 quantisation: beta[M], xq[M][K]. */
int orc_quantize_act(const void* x, int dtype, int64_t M, int64_t K, int8_t* xq, float* beta);

/* acc[M][N] = Σ_k xq[m][k]·ŵ[n][k] by add / subtract / skip.  Returns 0, or -1
 * if an accumulator leaves the int32 range. */
int orc_ternary_matmul(const int8_t* xq, const int8_t* codes, int64_t M, int64_t N, int64_t K,
                       int32_t* acc, int threads);

/* y[M][N] = fp32(acc)·fp32(α·β_m/127) (+ bias[n]). */
void orc_dequant(const int32_t* acc, const float* beta, float alpha, const float* bias,
                 int64_t M, int64_t N, float* y);

/* Whole forward (act quant + product + dequant) on unpacked codes. */
int orc_forward(const void* x, int dtype, int64_t M, int64_t K, const int8_t* codes, float alpha,
                const float* bias, int64_t N, int8_t* xq, float* beta, int32_t* acc, float* y,
                int threads);

/* Block-diagonal Hadamard rotation of each row (blocks of `block`, a power of
 * two dividing K) by the binary32 butterfly network, outputs times `scale`. */
int orc_hadamard(const void* x, int dtype, int64_t M, int64_t K, int64_t block, float scale, float* out);

/* One α per group of `group` consecutive elements of each row of W [N][K]:
 * alpha[N][ceil(K/group)], exact mean rounded to binary64 then binary32. */
int orc_absmean_groups(const void* W, int dtype, int64_t N, int64_t K, int64_t group, float* alpha);

/* Ternary codes with one α per group. */
int orc_ternarize_groups(const void* W, int dtype, int64_t N, int64_t K, int64_t group, const float* alpha,
                         int8_t* codes);

/* Product and dequantisation with one α per group (see the source). */
int orc_forward_groups(const int8_t* xq, const float* beta, int64_t M, int64_t K, const int8_t* codes,
                       const float* alpha, int64_t group, const float* bias, int64_t N, float* y, int threads);

/* Per-token absmax 4-bit quantisation, packed two per byte: xq4[M][ceil(K/2)]. */
int orc_quantize_act_a4(const void* x, int dtype, int64_t M, int64_t K, uint8_t* xq4, float* beta);

/* Unpacks 4-bit activations into int8 [M][K]. */
void orc_unpack_a4(const uint8_t* xq4, int64_t M, int64_t K, int8_t* xq);

/* y = fp32(acc)·fp32(α·β_m/7) (+ bias[n]). */
void orc_dequant_a4(const int32_t* acc, const float* beta, float alpha, const float* bias, int64_t M, int64_t N,
                    float* y);

/* Straight-through backward of the BitLinear layer (see the source):
 * gx[M][K] = α·(g·Ŵ), gw[N][K] = mask ⊙ (gᵀ·x̃·β/127). */
int orc_ste_grad_x(const float* g, int64_t M, int64_t N, const int8_t* codes, int64_t K, float alpha, float* gx,
                   int threads);
int orc_ste_grad_w(const float* g, int64_t M, int64_t N, const int8_t* xq, const float* beta, int64_t K,
                   const void* W, int dtype, float alpha, float* gw, int threads);

#ifdef __cplusplus
}
#endif
#endif
