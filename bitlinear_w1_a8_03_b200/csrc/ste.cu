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

// Register-tiled float32 GEMM: a CTA computes a 128 × 128 output tile with
// 256 threads, each 8 × 8 outputs (rows ty·4 + {0..3, 64..67}, columns
// tx·4 + {0..3, 64..67}, so that the 16-byte shared-memory reads of a warp
// are broadcast or contiguous); the reduction runs in stages of 8 through two
// shared-memory buffers, the next stage's global values loaded into registers
// while the current one is multiplied.  Every output is accumulated by its
// thread in increasing reduction index with fused multiply-adds.
constexpr int kTile = 128;
constexpr int kBR = 8;    // reduction depth per stage
constexpr int kT = 256;   // threads (16 × 16)
constexpr int kPad = 4;   // row padding of the shared tiles (floats)

struct Tiles {
    float a[2][kBR][kTile + kPad];  // [stage buffer][r][output row]
    float b[2][kBR][kTile + kPad];  // [stage buffer][r][output column]
};

// acc += A(:, r) · B(r, :) over the 8 reduction steps of buffer `buf`.
__device__ __forceinline__ void tile_fma(const Tiles& T, int buf, int tx, int ty, float (&acc)[8][8]) {
#pragma unroll
    for (int r = 0; r < kBR; ++r) {
        const float4 a0 = *reinterpret_cast<const float4*>(&T.a[buf][r][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&T.a[buf][r][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&T.b[buf][r][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&T.b[buf][r][64 + tx * 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
}

// Output row / column of the thread's i-th (j-th) value in the tile.
__device__ __forceinline__ int tile_row(int ty, int i) { return (i < 4 ? ty * 4 : 64 + ty * 4) + (i & 3); }

// ∂L/∂x: rows m (tokens), columns k, reduction over n.  A = g [M][N] float32,
// B = the codes of rows n, columns k, decoded to -1/0/+1.
__global__ void __launch_bounds__(kT, 2) ste_grad_x_kernel(const float* __restrict__ g, int64_t M, int64_t N, int64_t K,
                                                        const uint8_t* __restrict__ W_packed, int64_t row_bytes,
                                                        const float* __restrict__ alpha_p, float* __restrict__ gx) {
    __shared__ __align__(16) Tiles T;
    griddep_wait();
    griddep_launch_dependents();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t m0 = (int64_t)blockIdx.y * kTile, k0 = (int64_t)blockIdx.x * kTile;
    // loader roles: A: token row am = tid / 2, reduction columns 4·(tid % 2) .. +3;
    // B: reduction row bn = tid / 32, output columns 4·(tid % 32) .. +3 (one packed word field)
    const int am = threadIdx.x / 2, ac = 4 * (threadIdx.x % 2);
    const int bn = threadIdx.x / 32, bc = 4 * (threadIdx.x % 32);
    float ra[4], rb[4];
    auto load = [&](int64_t n0) {
        const int64_t m = m0 + am;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t n = n0 + ac + e;
            ra[e] = (m < M && n < N) ? g[m * N + n] : 0.0f;
        }
        const int64_t n = n0 + bn, k = k0 + bc;  // k is a multiple of 4: four codes of one byte field
        uint32_t word = 0;
        if (n < N && k < K) word = *reinterpret_cast<const uint32_t*>(W_packed + n * row_bytes + 4 * (k / 16));
        const int sfield = (int)((k % 16) / 4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // weight k + e = 16·word + 4·s + e lives in byte e of the word, bits 2s..2s+1
            const int c = (int)((word >> (8 * e + 2 * sfield)) & 3u);
            rb[e] = (n < N && k + e < K) ? (c == 2 ? 1.0f : (c == 0 ? -1.0f : 0.0f)) : 0.0f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int e = 0; e < 4; ++e) T.a[buf][ac + e][am] = ra[e];
        *reinterpret_cast<float4*>(&T.b[buf][bn][bc]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    };
    float acc[8][8] = {};
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t n0 = 0; n0 < N; n0 += kBR) {
        const bool more = n0 + kBR < N;
        if (more) load(n0 + kBR);
        tile_fma(T, buf, tx, ty, acc);
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    const float alpha = *alpha_p;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t m = m0 + tile_row(ty, i);
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t k = k0 + tile_row(tx, j);
            if (k < K) gx[m * K + k] = __fmul_rn(alpha, acc[i][j]);
        }
    }
}

// ∂L/∂W: rows n, columns k, reduction over m (tokens).  A = (g·s)ᵀ, B = x̃.
template <typename T>
__global__ void __launch_bounds__(kT, 2) ste_grad_w_kernel(const float* __restrict__ g, int64_t M, int64_t N, int64_t K,
                                                        const int8_t* __restrict__ xq, const float* __restrict__ beta,
                                                        const T* __restrict__ W, const float* __restrict__ alpha_p,
                                                        float* __restrict__ gw) {
    __shared__ __align__(16) Tiles S;
    griddep_wait();
    griddep_launch_dependents();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t n0 = (int64_t)blockIdx.y * kTile, k0 = (int64_t)blockIdx.x * kTile;
    // loader roles: token row r = tid / 32 of the stage; A: output rows n 4·(tid % 32) .. +3;
    // B: output columns k 4·(tid % 32) .. +3
    const int lr = threadIdx.x / 32, lc = 4 * (threadIdx.x % 32);
    float ra[4], rb[4];
    auto load = [&](int64_t mb) {
        const int64_t m = mb + lr;
        const float s = m < M ? __double2float_rn(__ddiv_rn((double)beta[m], 127.0)) : 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t n = n0 + lc + e, k = k0 + lc + e;
            ra[e] = (m < M && n < N) ? __fmul_rn(g[m * N + n], s) : 0.0f;
            rb[e] = (m < M && k < K) ? (float)xq[m * K + k] : 0.0f;
        }
    };
    auto store = [&](int buf) {
        *reinterpret_cast<float4*>(&S.a[buf][lr][lc]) = make_float4(ra[0], ra[1], ra[2], ra[3]);
        *reinterpret_cast<float4*>(&S.b[buf][lr][lc]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    };
    float acc[8][8] = {};
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t mb = 0; mb < M; mb += kBR) {
        const bool more = mb + kBR < M;
        if (more) load(mb + kBR);
        tile_fma(S, buf, tx, ty, acc);
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    const float alpha = *alpha_p;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + tile_row(ty, i);
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t k = k0 + tile_row(tx, j);
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
        const dim3 grid((unsigned)((K + kTile - 1) / kTile), (unsigned)((M + kTile - 1) / kTile));
        ste_grad_x_kernel<<<grid, kT, 0, stream>>>(g, M, N, K, W_packed, row_bytes, alpha, grad_x);
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (grad_W) {
        const dim3 grid((unsigned)((K + kTile - 1) / kTile), (unsigned)((N + kTile - 1) / kTile));
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
