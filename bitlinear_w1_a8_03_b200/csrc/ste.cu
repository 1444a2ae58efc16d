// Backward of the BitLinear layer with the straight-through estimator
// ("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §3.3: the forward
// quantises, the backward passes the gradient through the quantisers as if
// they were the identity; §6.3: a weight outside the clip range gets no
// gradient; "1.58 位大模型" §3.4: latent float weights are updated).
//
// For y = (x̃·β/127)·(Ŵ·α)ᵀ and g = ∂L/∂y [M][N]:
//   ∂L/∂x [M][K] = α · (g · Ŵ)                        (Ŵ ternary codes)
//   ∂L/∂W [N][K] = [|W/α| <= 1] ⊙ ((g·s)ᵀ · x̃)        (s_m = RN32(RN64(β_m/127)),
//                                                     each g·s_m rounded to binary32)
// Both are dense contractions of float32 data: g has arbitrary float32
// values, so the int8 / low-precision tensor-core kinds would not keep the
// products exact; they run as register-tiled float32 GEMMs on the CUDA cores.
// Each output is accumulated by one thread in index order (a fixed order, so
// results are reproducible), rounded once at the end.
#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {
namespace {

constexpr int kBM = 64;  // tile rows of the output
constexpr int kBN = 64;  // tile columns of the output
constexpr int kBR = 16;  // reduction depth per stage
constexpr int kT = 256;  // threads: 16 × 16, each 4 × 4 outputs

// ∂L/∂x: rows m (tokens), columns k, reduction over n.  A = g [M][N] float32,
// B = the codes of rows n, columns k (decoded to -1/0/+1 in shared memory).
__global__ void __launch_bounds__(kT) ste_grad_x_kernel(const float* __restrict__ g, int64_t M, int64_t N, int64_t K,
                                                        const uint8_t* __restrict__ W_packed, int64_t row_bytes,
                                                        const float* __restrict__ alpha_p, float* __restrict__ gx) {
    __shared__ float As[kBR][kBM + 4];  // [n][m]
    __shared__ float Bs[kBR][kBN + 4];  // [n][k]
    griddep_wait();
    griddep_launch_dependents();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t m0 = (int64_t)blockIdx.y * kBM, k0 = (int64_t)blockIdx.x * kBN;
    float acc[4][4] = {};
    for (int64_t n0 = 0; n0 < N; n0 += kBR) {
        // A tile: 64 tokens × 16 n (each thread 4 values)
        for (int i = threadIdx.x; i < kBM * kBR; i += kT) {
            const int mm = i / kBR, nn = i % kBR;
            const int64_t m = m0 + mm, n = n0 + nn;
            As[nn][mm] = (m < M && n < N) ? g[m * N + n] : 0.0f;
        }
        // B tile: 16 rows n × 64 columns k: one 16-byte chunk of codes per row
        for (int i = threadIdx.x; i < kBR * kBN; i += kT) {
            const int nn = i / kBN, kk = i % kBN;
            const int64_t n = n0 + nn, k = k0 + kk;
            float v = 0.0f;
            if (n < N && k < K) {
                // weight k = 16·word + 4·s + b lives in byte b of the word, bits 2s..2s+1
                const int64_t word = k / 16;
                const int sfield = (int)((k % 16) / 4), b = (int)(k % 4);
                const uint8_t byte = W_packed[n * row_bytes + 4 * word + b];
                const int c = (byte >> (2 * sfield)) & 3;
                v = c == 2 ? 1.0f : (c == 0 ? -1.0f : 0.0f);
            }
            Bs[nn][kk] = v;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kBR; ++r) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[r][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Bs[r][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    const float alpha = *alpha_p;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = k0 + tx * 4 + j;
            if (k < K) gx[m * K + k] = __fmul_rn(alpha, acc[i][j]);
        }
    }
}

// ∂L/∂W: rows n, columns k, reduction over m (tokens).  A = (g·s)ᵀ, B = x̃.
template <typename T>
__global__ void __launch_bounds__(kT) ste_grad_w_kernel(const float* __restrict__ g, int64_t M, int64_t N, int64_t K,
                                                        const int8_t* __restrict__ xq, const float* __restrict__ beta,
                                                        const T* __restrict__ W, const float* __restrict__ alpha_p,
                                                        float* __restrict__ gw) {
    __shared__ float As[kBR][kBM + 4];  // [m][n]
    __shared__ float Bs[kBR][kBN + 4];  // [m][k]
    __shared__ float ss[kBR];
    griddep_wait();
    griddep_launch_dependents();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t n0 = (int64_t)blockIdx.y * kBM, k0 = (int64_t)blockIdx.x * kBN;
    float acc[4][4] = {};
    for (int64_t mb = 0; mb < M; mb += kBR) {
        if (threadIdx.x < kBR) {
            const int64_t m = mb + threadIdx.x;
            ss[threadIdx.x] = m < M ? __double2float_rn(__ddiv_rn((double)beta[m], 127.0)) : 0.0f;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kBR * kBM; i += kT) {
            const int mm = i / kBM, nn = i % kBM;
            const int64_t m = mb + mm, n = n0 + nn;
            As[mm][nn] = (m < M && n < N) ? __fmul_rn(g[m * N + n], ss[mm]) : 0.0f;
        }
        for (int i = threadIdx.x; i < kBR * kBN; i += kT) {
            const int mm = i / kBN, kk = i % kBN;
            const int64_t m = mb + mm, k = k0 + kk;
            Bs[mm][kk] = (m < M && k < K) ? (float)xq[m * K + k] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kBR; ++r) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[r][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Bs[r][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    const float alpha = *alpha_p;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t n = n0 + ty * 4 + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = k0 + tx * 4 + j;
            if (k >= K) continue;
            const float q = __fdiv_rn(load_as_f32(W, n * K + k), alpha);  // the forward's quotient
            gw[n * K + k] = fabsf(q) <= 1.0f ? acc[i][j] : 0.0f;          // no gradient outside the clip range
        }
    }
}

}  // namespace

cudaError_t launch_ste_backward(const float* g, int64_t M, int64_t N, int64_t K, const uint8_t* W_packed,
                                const float* alpha, const int8_t* x_q, const float* beta, const void* W,
                                bitlinear_dtype w_dtype, float* grad_x, float* grad_W, cudaStream_t stream) {
    const int64_t row_bytes = (int64_t)bitlinear_packed_row_bytes(K);
    if (grad_x) {
        const dim3 grid((unsigned)((K + kBN - 1) / kBN), (unsigned)((M + kBM - 1) / kBM));
        ste_grad_x_kernel<<<grid, kT, 0, stream>>>(g, M, N, K, W_packed, row_bytes, alpha, grad_x);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (grad_W) {
        const dim3 grid((unsigned)((K + kBN - 1) / kBN), (unsigned)((N + kBM - 1) / kBM));
        if (w_dtype == BL_BF16)
            ste_grad_w_kernel<uint16_t><<<grid, kT, 0, stream>>>(g, M, N, K, x_q, beta,
                                                                 static_cast<const uint16_t*>(W), alpha, grad_W);
        else
            ste_grad_w_kernel<float><<<grid, kT, 0, stream>>>(g, M, N, K, x_q, beta, static_cast<const float*>(W),
                                                              alpha, grad_W);
    }
    return cudaGetLastError();
}

}  // namespace bl
