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

/* ------------------------------------------------------------------------
 * Rotation before the absmax quantisation ([BitNet 三值权重实战] §6.2: an
 * orthogonal (Hadamard) rotation of the activations spreads an outlier's
 * energy over all dimensions before absmax quantisation).
 *
 * out[m][·] = x[m][·]·H, H block-diagonal with Sylvester Hadamard blocks of
 * order `block` (a power of two dividing K): inside a block,
 * out[j] = Σ_i x[i]·(-1)^popcount(i & j).  Evaluated by the fast
 * Walsh–Hadamard butterfly network in binary32 with the stages in a fixed
 * order, h = 1, 2, 4, …, block/2: each butterfly replaces the pair at
 * positions (i, i + h), i & h == 0, by (a + b, a - b).  Every output is then
 * multiplied by `scale` (1 for activations; 1/block, a power of two, for the
 * weights, so that (x·H)·(W·H/block)ᵀ = x·Wᵀ in exact arithmetic). */
int orc_hadamard(const void* x, int dtype, int64_t M, int64_t K, int64_t block, float scale, float* out) {
    if (block < 1 || (block & (block - 1)) != 0 || K % block != 0) return -1;
    for (int64_t m = 0; m < M; ++m) {
        float* v = out + m * K;
        for (int64_t k = 0; k < K; ++k) v[k] = orc_load(x, dtype, m * K + k);
        for (int64_t s = 0; s < K; s += block) {
            float* b = v + s;
            for (int64_t h = 1; h < block; h <<= 1) {
                for (int64_t i = 0; i < block; ++i) {
                    if (i & h) continue;
                    float p = b[i], q = b[i + h];
                    b[i] = p + q;
                    b[i + h] = p - q;
                }
            }
        }
        if (scale != 1.0f)
            for (int64_t k = 0; k < K; ++k) v[k] = v[k] * scale;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Scale granularity finer than the tensor: per output row ([1.58 位大模型]
 * §3.1, §4.2: alpha = mean(|w|, axis=-1)) and per block of consecutive input
 * features within a row ([硬件协同优化] §2.3, §4.2: one scale per 128
 * elements, scale[C_out][C_in/128]).  Both are groups of `group` consecutive
 * elements of a row (group >= K: one group per row); the last group of a row
 * may be shorter.  Each α is the exact mean rounded once to binary64 and once
 * to binary32, as for the tensor. */

/* RN64(S / count) where S·2^149 = limbs (little-endian 32-bit digits). */
static double orc_exact_mean(const uint64_t* limbs_in, int nlimbs, uint64_t count) {
    enum { EXTRA = 4 };                /* 128 more bits below the sum for the quotient */
    uint32_t num[32], q[32];
    int n = nlimbs + EXTRA;
    for (int j = 0; j < EXTRA; ++j) num[j] = 0;
    for (int j = 0; j < nlimbs; ++j) num[EXTRA + j] = (uint32_t)limbs_in[j];
    /* long division by count, most significant digit first */
    unsigned __int128 rem = 0;
    for (int j = n - 1; j >= 0; --j) {
        unsigned __int128 cur = (rem << 32) | num[j];
        q[j] = (uint32_t)(cur / count);
        rem = cur % count;
    }
    int top = -1;
    for (int j = n - 1; j >= 0 && top < 0; --j)
        for (int b = 31; b >= 0; --b)
            if ((q[j] >> b) & 1u) {
                top = 32 * j + b;
                break;
            }
    if (top < 0) return 0.0;
    /* quotient Q = S·2^(149+128)/count; keep 53 bits below and including the top */
    uint64_t mant = 0;
    for (int b = 0; b < 53; ++b) {
        int pos = top - 52 + b;
        if (pos >= 0 && ((q[pos >> 5] >> (pos & 31)) & 1u)) mant |= 1ull << b;
    }
    int round_pos = top - 53;
    int round_bit = round_pos >= 0 && ((q[round_pos >> 5] >> (round_pos & 31)) & 1u);
    int sticky = rem != 0;
    for (int pos = 0; pos < round_pos && !sticky; ++pos)
        if ((q[pos >> 5] >> (pos & 31)) & 1u) sticky = 1;
    int e = top - 52 - 149 - 128;
    if (round_bit && (sticky || (mant & 1ull))) {
        ++mant;
        if (mant == (1ull << 53)) {
            mant >>= 1;
            ++e;
        }
    }
    return ldexp((double)mant, e);
}

int orc_absmean_groups(const void* W, int dtype, int64_t N, int64_t K, int64_t group, float* alpha) {
    if (group < 1) return -1;
    const int64_t G = (K + group - 1) / group;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t k0 = g * group, k1 = k0 + group < K ? k0 + group : K;
            uint64_t limbs[10] = {0};
            for (int64_t k = k0; k < k1; ++k) {
                float w = orc_load(W, dtype, n * K + k);
                uint32_t bits;
                memcpy(&bits, &w, 4);
                bits &= 0x7FFFFFFFu;
                uint32_t e = bits >> 23, sig = bits & 0x7FFFFFu;
                if (e == 255) return -1;
                if (e != 0) sig = sig | 0x800000u;
                /* |w|·2^149 = sig·2^(max(e,1)-1) */
                uint32_t p = (e != 0 ? e : 1u) - 1u;
                uint64_t v = (uint64_t)sig << (p & 31u);
                limbs[p >> 5] += v & 0xFFFFFFFFull;
                limbs[(p >> 5) + 1] += v >> 32;
            }
            for (int j = 0; j + 1 < 10; ++j) {
                limbs[j + 1] += limbs[j] >> 32;
                limbs[j] &= 0xFFFFFFFFull;
            }
            alpha[n * G + g] = (float)orc_exact_mean(limbs, 10, (uint64_t)(k1 - k0));
        }
    }
    return 0;
}

/* Codes with one α per group: ŵ = clip(round(W/α_g), -1, 1), as orc_ternarize. */
int orc_ternarize_groups(const void* W, int dtype, int64_t N, int64_t K, int64_t group, const float* alpha,
                         int8_t* codes) {
    const int64_t G = (K + group - 1) / group;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float qg = orc_load(W, dtype, n * K + k) / alpha[n * G + k / group];
            if (qg != qg) {
                codes[n * K + k] = 0;
                continue;
            }
            float rg = rintf(qg);
            if (rg > 1.0f) rg = 1.0f;
            if (rg < -1.0f) rg = -1.0f;
            codes[n * K + k] = (int8_t)rg;
        }
    return 0;
}

/* Product and dequantisation with one α per group: for each group b the
 * integer sum acc_b = Σ_{k in b} x̃·ŵ (add / subtract / skip), then
 * S = Σ_b α_b·acc_b in binary64, groups in order (each product is exact);
 * y = RN32( RN32(S)·s_m ) (+ bias[n]) with s_m = RN32(RN64(β_m / 127)): the
 * per-token dequantisation of the activations, then the weights' scale, as
 * [1.58 位大模型] §4.3 scales the product by alpha afterwards. */
int orc_forward_groups(const int8_t* xq, const float* beta, int64_t M, int64_t K, const int8_t* codes,
                       const float* alpha, int64_t group, const float* bias, int64_t N, float* y, int threads) {
    const int64_t G = (K + group - 1) / group;
    (void)threads;
#ifdef _OPENMP
    int nt = threads > 0 ? threads : 1;
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double sd = (double)beta[m] / 127.0;
            float s = (float)sd;
            double S = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t k0 = g * group, k1 = k0 + group < K ? k0 + group : K;
                int64_t a = 0;
                for (int64_t k = k0; k < k1; ++k) {
                    int8_t w = codes[n * K + k];
                    if (w == 1) a += xq[m * K + k];
                    else if (w == -1) a -= xq[m * K + k];
                }
                S += (double)alpha[n * G + g] * (double)a;
            }
            float v = (float)S;
            v = v * s;
            if (bias) v = v + bias[n];
            y[m * N + n] = v;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * 4-bit activations ([BitNet CPU 实测] §2.1: later variants quantise the
 * activations to 4 bits; §6.2).  The absmax rule of [BitNet 三值权重实战] §2.4
 * with the 4-bit signed range: β = max|x| + 1e-8, x̃ = clip(round((x·7)/β),
 * -7, 7).  Stored two per byte: element k in byte k/2, the low nibble for even
 * k, two's complement; the high nibble of the last byte of an odd-K row is 0.
 * The dequantisation scale is RN32(RN64(α·β/7)). */
int orc_quantize_act_a4(const void* x, int dtype, int64_t M, int64_t K, uint8_t* xq4, float* beta) {
    const int64_t rb = (K + 1) / 2;
    for (int64_t m = 0; m < M; ++m) {
        float mx = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(orc_load(x, dtype, m * K + k));
            if (a > mx) mx = a;
        }
        float b4 = mx + 1e-8f;
        beta[m] = b4;
        for (int64_t j = 0; j < rb; ++j) xq4[m * rb + j] = 0;
        for (int64_t k = 0; k < K; ++k) {
            float t = orc_load(x, dtype, m * K + k) * 7.0f;
            t = t / b4;
            float r4 = rintf(t);
            if (r4 > 7.0f) r4 = 7.0f;
            if (r4 < -7.0f) r4 = -7.0f;
            uint8_t nib = (uint8_t)((int)r4 & 0xF);
            xq4[m * rb + k / 2] |= (uint8_t)(nib << (4 * (k % 2)));
        }
    }
    return 0;
}

/* Unpacks 4-bit activations [M][ceil(K/2)] into int8 [M][K]. */
void orc_unpack_a4(const uint8_t* xq4, int64_t M, int64_t K, int8_t* xq) {
    const int64_t rb = (K + 1) / 2;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            int nib = (xq4[m * rb + k / 2] >> (4 * (k % 2))) & 0xF;
            xq[m * K + k] = (int8_t)(nib >= 8 ? nib - 16 : nib);
        }
}

/* y = fp32(acc)·fp32(α·β_m/7) (+ bias[n]), as orc_dequant with 7 for 127. */
void orc_dequant_a4(const int32_t* acc, const float* beta, float alpha, const float* bias, int64_t M, int64_t N,
                    float* y) {
    for (int64_t m = 0; m < M; ++m) {
        double s4 = (double)alpha * (double)beta[m];
        s4 = s4 / 7.0;
        float s = (float)s4;
        for (int64_t n = 0; n < N; ++n) {
            float v = (float)acc[m * N + n];
            v = v * s;
            if (bias) v = v + bias[n];
            y[m * N + n] = v;
        }
    }
}

/* ------------------------------------------------------------------------
 * Training with the straight-through estimator ([BitNet 三值权重实战] §3.3,
 * §6.3; [1.58 位大模型] §3.4).  The forward is the inference arithmetic with
 * the weights quantised afresh from the latent float weights every step (§4.2,
 * the training branch).  The backward of y = (x̃·β/127)·(Ŵ·α)ᵀ treats both
 * quantisers as the identity ("前向量化、反向恒等"), except that a weight
 * outside the clip range gets no gradient (§6.3): with g = ∂L/∂y,
 *   ∂L/∂x[m][k] = α · Σ_n g[m][n]·ŵ[n][k]
 *   ∂L/∂W[n][k] = [ |W[n][k]/α| <= 1 ] · Σ_m g[m][n]·(x̃[m][k]·β_m/127)
 * with α and β treated as constants.  Arithmetic: the sums in binary64 in
 * index order, each result rounded once to binary32; W/α is the forward's
 * binary32 quotient; β_m/127 is s_m = RN32(RN64(β_m/127)) and each product
 * g·s_m is rounded to binary32 before it multiplies x̃ (exact in binary64). */
int orc_ste_grad_x(const float* g, int64_t M, int64_t N, const int8_t* codes, int64_t K, float alpha, float* gx,
                   int threads) {
    (void)threads;
#ifdef _OPENMP
    int nt = threads > 0 ? threads : 1;
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt)
#endif
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                int8_t w = codes[n * K + k];
                if (w == 1) s += (double)g[m * N + n];
                else if (w == -1) s -= (double)g[m * N + n];
            }
            gx[m * K + k] = (float)((double)alpha * s);
        }
    return 0;
}

int orc_ste_grad_w(const float* g, int64_t M, int64_t N, const int8_t* xq, const float* beta, int64_t K,
                   const void* W, int dtype, float alpha, float* gw, int threads) {
    (void)threads;
#ifdef _OPENMP
    int nt = threads > 0 ? threads : 1;
#pragma omp parallel for collapse(2) schedule(static) num_threads(nt)
#endif
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float q = orc_load(W, dtype, n * K + k) / alpha;
            if (!(fabsf(q) <= 1.0f)) {  /* outside the clip range (or 0/0): no gradient */
                gw[n * K + k] = 0.0f;
                continue;
            }
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m) {
                double sm = (double)beta[m] / 127.0;
                float gs = g[m * N + n] * (float)sm;
                s += (double)gs * (double)xq[m * K + k];
            }
            gw[n * K + k] = (float)s;
        }
    return 0;
}
