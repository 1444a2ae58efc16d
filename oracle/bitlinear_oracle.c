/*
 * CPU oracle for the BitLinear W1.58·A8 matmul.  TEST INFRASTRUCTURE: see the
 * header for who may use it.  Every function is the definition written out,
 * in the order the pages state it; nothing is blocked, fused or reordered.
 */
#include "bitlinear_oracle.h"

#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bfloat16 is the top half of a binary32: widening is exact. */
static float orc_load(const void* p, int dtype, int64_t i) {
    uint32_t bits;
    float f;
    if (dtype == ORC_BF16) {
        bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    } else {
        memcpy(&bits, (const float*)p + i, 4);
    }
    memcpy(&f, &bits, 4);
    return f;
}

/* [BitNet 三值权重实战] §2.3: α = mean(|W|) over the whole tensor (per-tensor
 * absmean; the layer's code in §4.1 calls weight.abs().mean()).  The sum is
 * kept exact here: each |w| = significand·2^(E-150), so adding significands
 * per exponent E in 64-bit integers loses nothing.  The caller turns the bins
 * into α = RN32(RN64(Σ|W| / count)). */
int orc_abs_exponent_bins(const void* W, int dtype, int64_t count, int64_t bins[256]) {
    for (int e = 0; e < 256; ++e) bins[e] = 0;
    for (int64_t i = 0; i < count; ++i) {
        float w = orc_load(W, dtype, i);
        uint32_t bits;
        memcpy(&bits, &w, 4);
        bits &= 0x7FFFFFFFu;                 /* |w| */
        uint32_t e = bits >> 23;
        uint32_t sig = bits & 0x7FFFFFu;
        if (e == 255) return -1;             /* inf or NaN: no mean */
        if (e != 0) sig |= 0x800000u;        /* implicit leading one */
        bins[e] += (int64_t)sig;
    }
    return 0;
}

/* [BitNet 三值权重实战] §2.3 and §4.1: Ŵ = clip(round(W/α), -1, 1); the code
 * uses torch.round, which rounds half to even (rintf under the default
 * rounding mode).  W/α is one binary32 division.  α = 0 happens only when the
 * mean underflows; then W/α is ±inf (clipped to ±1) or 0/0 = NaN, and a NaN
 * quotient is read as the zero weight. */
int orc_ternarize(const void* W, int dtype, int64_t count, float alpha, int8_t* codes) {
    for (int64_t i = 0; i < count; ++i) {
        float q = orc_load(W, dtype, i) / alpha;
        if (q != q) {
            codes[i] = 0;
            continue;
        }
        float r = rintf(q);
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        codes[i] = (int8_t)r;
    }
    return 0;
}

/* Storage: 2 physical bits per weight, 00/01/10 for -1/0/+1
 * ([BitNet 三值权重实战] §5.3), rows contiguous along the input features
 * (weight[out][in], §4.2; channel-contiguous packing, [硬件协同优化] §4.3).
 * Within a row, weights are taken 16 at a time into one little-endian 32-bit
 * word: weight 16g + 4s + b goes to byte b of word g, bits 2s..2s+1.  Rows are
 * padded to a multiple of 64 weights (16 bytes) with the zero code 01. */
int64_t orc_packed_row_bytes(int64_t K) { return 16 * ((K + 63) / 64); }

void orc_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed) {
    const int64_t rb = orc_packed_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        uint8_t* row = packed + n * rb;
        for (int64_t j = 0; j < rb; ++j) row[j] = 0;
        for (int64_t k = 0; k < rb * 4; ++k) {
            int code = (k < K) ? (int)codes[n * K + k] + 1 : 1;
            int64_t g = k / 16;          /* word */
            int i = (int)(k % 16);       /* position in the word: i = 4s + b */
            int s = i / 4, b = i % 4;
            row[4 * g + b] |= (uint8_t)(code << (2 * s));
        }
    }
}

/* [BitNet 三值权重实战] §2.4 and §4.1, one row of x (one token) at a time:
 * β = max|x| + 1e-8 (the code's epsilon, added in binary32), then
 * x̃ = clip(round(x·127/β), -127, 127), evaluated left to right as the code
 * writes it: (x·127) then /β, each rounded to binary32; round half to even.
 * Per token follows [1.58 位大模型] §3.2 (value ranges differ between tokens). */
int orc_quantize_act(const void* x, int dtype, int64_t M, int64_t K, int8_t* xq, float* beta) {
    for (int64_t m = 0; m < M; ++m) {
        float mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(orc_load(x, dtype, m * K + k));
            if (a > mx) mx = a;
        }
        float b = mx + 1e-8f;
        beta[m] = b;
        for (int64_t k = 0; k < K; ++k) {
            float t = orc_load(x, dtype, m * K + k) * 127.0f;
            t = t / b;
            float r = rintf(t);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            xq[m * K + k] = (int8_t)r;
        }
    }
    return 0;
}

/* [1.58 位大模型] §3.3: Y[m][n] = Σ_{k: W=1} X[m][k] - Σ_{k: W=-1} X[m][k];
 * a zero weight is skipped.  Integer addition is exact, so order is free. */
int orc_ternary_matmul(const int8_t* xq, const int8_t* codes, int64_t M, int64_t N, int64_t K,
                       int32_t* acc, int threads) {
    int bad = 0;
    (void)threads;
#ifdef _OPENMP
    int nt = threads > 0 ? threads : 1;
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt) reduction(| : bad)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* xr = xq + m * K;
            const int8_t* wr = codes + n * K;
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (wr[k] == 1) s += xr[k];
                else if (wr[k] == -1) s -= xr[k];
            }
            if (s > INT32_MAX || s < INT32_MIN) bad = 1;
            acc[m * N + n] = (int32_t)s;
        }
    }
    return bad ? -1 : 0;
}

/* [BitNet 三值权重实战] §2.4–§2.5 and §4.2: y = (x̃·Ŵᵀ)·(α·β/127) + bias.
 * The code forms alpha*beta/127.0 from Python floats (binary64, left to
 * right) and scales a float32 tensor by it, which rounds the scalar to
 * binary32 and multiplies once in binary32; the bias add is binary32. */
void orc_dequant(const int32_t* acc, const float* beta, float alpha, const float* bias,
                 int64_t M, int64_t N, float* y) {
    for (int64_t m = 0; m < M; ++m) {
        double sd = (double)alpha * (double)beta[m];
        sd = sd / 127.0;
        float s = (float)sd;
        for (int64_t n = 0; n < N; ++n) {
            float v = (float)acc[m * N + n];
            v = v * s;
            if (bias) v = v + bias[n];
            y[m * N + n] = v;
        }
    }
}

/* [BitNet 三值权重实战] §3.2, inference path: quantise x, integer product,
 * dequantise and add bias (the weight codes are cached from §2.3). */
int orc_forward(const void* x, int dtype, int64_t M, int64_t K, const int8_t* codes, float alpha,
                const float* bias, int64_t N, int8_t* xq, float* beta, int32_t* acc, float* y,
                int threads) {
    orc_quantize_act(x, dtype, M, K, xq, beta);
    int rc = orc_ternary_matmul(xq, codes, M, N, K, acc, threads);
    orc_dequant(acc, beta, alpha, bias, M, N, y);
    return rc;
}
