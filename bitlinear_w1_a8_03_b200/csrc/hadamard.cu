// Hadamard rotation of the activations before the absmax quantisation, and of
// the weights before the absmean quantisation.
//
// "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §6.2: a few
// activation dimensions carry outliers that blow up β = max|x| and crush the
// other dimensions to zero; multiplying the activations by an orthogonal
// (Hadamard) matrix first spreads an outlier's energy over all dimensions.
// The weights take the same rotation, W' = W·H/b, so that x'·W'ᵀ = x·Wᵀ.
//
// H is block-diagonal with Sylvester blocks of order b (a power of two
// dividing K): inside a block out[j] = Σ_i x[i]·(-1)^popcount(i & j).  It is
// evaluated by the fast Walsh–Hadamard butterfly network in binary32 with the
// stages in a fixed order, h = 1, 2, 4, …, b/2, each butterfly replacing the
// pair (i, i + h), i & h == 0, by (a + b, a - b).  Every butterfly is one
// binary32 add and one subtract of the same operands whichever thread does
// it, so the result is identical to any evaluation in that stage order.
//
// One CTA per row; each thread holds kE consecutive elements: stages h < kE
// run in registers, kE <= h < 32·kE between lanes by shuffles, larger ones as
// pair passes through shared memory.  Rows of up to 1024·kE elements stay in
// registers from the load to the store; longer rows are rotated twice (once
// for the absmax, once to quantise), which gives the same values both times.
#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {
namespace {

constexpr int kE = 16;                    // elements per thread
constexpr int kMaxThreads = 1024;
constexpr int kTile = kMaxThreads * kE;   // elements of one pass over a row
constexpr int kMaxBlock = 8192;           // largest rotation block

struct HadParams {
    HadJob p[kMaxGroup];
    int64_t row_begin[kMaxGroup + 1];
    int count;
};

template <typename T>
__device__ __forceinline__ void load_elems(const T* row, int64_t K, int64_t k0, bool vec, float (&v)[kE]) {
    if (vec && k0 + kE <= K) {
        constexpr int per = 16 / sizeof(T);  // elements per 16-byte vector
#pragma unroll
        for (int q = 0; q < kE / per; ++q) {
            const uint4 u = ld_shared_ro16(row + k0 + q * per);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (sizeof(T) == 4) {
                    v[q * per + i] = __uint_as_float(w[i]);
                } else {
                    v[q * per + 2 * i] = __uint_as_float(w[i] << 16);
                    v[q * per + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                }
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < kE; ++e) v[e] = (k0 + e < K) ? load_as_f32(row, k0 + e) : 0.0f;
    }
}

// Rotates the tile held by the CTA (thread t holds elements t·kE .. t·kE+kE-1
// of the tile) in place.  `s` is shared scratch of nthreads·kE floats.
__device__ void rotate_tile(float (&v)[kE], int block, float* s) {
    const int lane = threadIdx.x & 31;
    // stages inside a thread
#pragma unroll
    for (int h = 1; h < kE; h <<= 1) {
        if (h >= block) break;
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            if (e & h) continue;
            const float a = v[e], b = v[e + h];
            v[e] = __fadd_rn(a, b);
            v[e + h] = __fsub_rn(a, b);
        }
    }
    // stages between lanes of a warp
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        if (d * kE >= block) break;
        const bool upper = (lane & d) != 0;
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            const float o = __shfl_xor_sync(0xffffffffu, v[e], d);
            v[e] = upper ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
        }
    }
    // stages between warps: pair passes through shared memory
    if (block > 32 * kE) {
        const int t = threadIdx.x;
#pragma unroll
        for (int e = 0; e < kE; ++e) s[t * kE + e] = v[e];
        __syncthreads();
        for (int h = 32 * kE; h < block; h <<= 1) {
#pragma unroll
            for (int q = 0; q < kE / 2; ++q) {
                const int p = t * (kE / 2) + q;  // pair index within the tile
                const int i = (p / h) * 2 * h + (p % h), j = i + h;
                const float a = s[i], b = s[j];
                s[i] = __fadd_rn(a, b);
                s[j] = __fsub_rn(a, b);
            }
            __syncthreads();
        }
#pragma unroll
        for (int e = 0; e < kE; ++e) v[e] = s[t * kE + e];
        __syncthreads();  // s may be reused by the next tile
    }
}

__device__ __forceinline__ float block_max_h(float mx, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
    const int nw = blockDim.x >> 5;
    for (int w = 1; w < nw; ++w) mx = fmaxf(mx, red[w]);
    return mx;
}

// QUANT = false: out = rotate(x)·scale.  QUANT = true: x_q, β of rotate(x).
template <typename T, bool QUANT>
__global__ void __launch_bounds__(kMaxThreads) hadamard_kernel(const __grid_constant__ HadParams Q) {
    extern __shared__ float s_tile[];  // blockDim·kE floats (only for blocks > 32·kE)
    __shared__ float red[kMaxThreads / 32];
    griddep_wait();  // x may come from the preceding kernel
    griddep_launch_dependents();
    const int64_t grow = blockIdx.x;
    int pi = 0;
    while (pi + 1 < Q.count && grow >= Q.row_begin[pi + 1]) ++pi;
    const HadJob& P = Q.p[pi];
    const int64_t m = grow - Q.row_begin[pi];
    const T* row = static_cast<const T*>(P.x) + m * P.K;
    const int64_t tile = (int64_t)blockDim.x * kE;
    const int ntiles = (int)((P.K + tile - 1) / tile);
    const bool vec = (reinterpret_cast<uintptr_t>(P.x) & 15) == 0 && (P.K % kE) == 0;
    float v[kE];

    if constexpr (!QUANT) {
        float* orow = P.out + m * P.K;
        for (int ti = 0; ti < ntiles; ++ti) {
            const int64_t k0 = ti * tile + (int64_t)threadIdx.x * kE;
            load_elems(row, P.K, k0, vec, v);
            rotate_tile(v, P.block, s_tile);
            if (P.scale != 1.0f) {
#pragma unroll
                for (int e = 0; e < kE; ++e) v[e] = __fmul_rn(v[e], P.scale);
            }
            if (vec && k0 + kE <= P.K && (reinterpret_cast<uintptr_t>(P.out) & 15) == 0) {
#pragma unroll
                for (int q = 0; q < kE / 4; ++q)
                    *reinterpret_cast<float4*>(orow + k0 + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            } else {
#pragma unroll
                for (int e = 0; e < kE; ++e)
                    if (k0 + e < P.K) orow[k0 + e] = v[e];
            }
        }
    } else {
        // absmax over the rotated row
        float mx = 0.0f;
        for (int ti = 0; ti < ntiles; ++ti) {
            const int64_t k0 = ti * tile + (int64_t)threadIdx.x * kE;
            load_elems(row, P.K, k0, vec, v);
            rotate_tile(v, P.block, s_tile);
#pragma unroll
            for (int e = 0; e < kE; ++e) mx = fmaxf(mx, fabsf(v[e]));  // zeros past K do not change it
        }
        const float beta = __fadd_rn(block_max_h(mx, red), 1e-8f);
        const float qf = quant_factor(beta, 127.0f);
        if (threadIdx.x == 0) P.beta[m] = beta;
        int8_t* q = P.x_q + m * P.K;
        for (int ti = 0; ti < ntiles; ++ti) {
            const int64_t k0 = ti * tile + (int64_t)threadIdx.x * kE;
            if (ntiles > 1) {  // one tile: the rotated values are still in v
                load_elems(row, P.K, k0, vec, v);
                rotate_tile(v, P.block, s_tile);
            }
            uint32_t w[kE / 4];
            quantize_codes<kE>(v, beta, qf, w);
            if (vec && k0 + kE <= P.K && (reinterpret_cast<uintptr_t>(P.x_q) & 15) == 0) {
                *reinterpret_cast<uint4*>(q + k0) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int e = 0; e < kE; ++e)
                    if (k0 + e < P.K) q[k0 + e] = (int8_t)(uint8_t)(w[e / 4] >> (8 * (e % 4)));
            }
        }
    }
}

}  // namespace

int hadamard_max_block() { return kMaxBlock; }

cudaError_t launch_hadamard(const HadJob* jobs, int count, bitlinear_dtype dtype, cudaStream_t stream, bool pdl) {
    HadParams P{};
    P.count = count;
    int64_t rows = 0, kmax = 0;
    int bmax = 1;
    for (int i = 0; i < count; ++i) {
        P.p[i] = jobs[i];
        P.row_begin[i] = rows;
        rows += jobs[i].M;
        kmax = jobs[i].K > kmax ? jobs[i].K : kmax;
        bmax = jobs[i].block > bmax ? jobs[i].block : bmax;
    }
    P.row_begin[count] = rows;
    // threads: enough for one tile of the longest row, a multiple of 32 and
    // of bmax / kE, so that a tile holds whole blocks of every problem (the
    // shared-memory pair passes stay inside the tile); at most kMaxThreads,
    // whose tile (kTile, a multiple of every block) then takes several passes
    const int64_t step = bmax / kE > 32 ? bmax / kE : 32;
    int64_t want = (kmax + kE - 1) / kE;
    want = (want + step - 1) / step * step;
    if (want > kMaxThreads) want = kMaxThreads;
    const int threads = (int)want;
    const size_t smem = bmax > 32 * kE ? (size_t)threads * kE * sizeof(float) : 0;
    const bool quant = jobs[0].x_q != nullptr;
    const void* kernel;
    if (dtype == BL_BF16)
        kernel = quant ? reinterpret_cast<const void*>(hadamard_kernel<uint16_t, true>)
                       : reinterpret_cast<const void*>(hadamard_kernel<uint16_t, false>);
    else
        kernel = quant ? reinterpret_cast<const void*>(hadamard_kernel<float, true>)
                       : reinterpret_cast<const void*>(hadamard_kernel<float, false>);
    cudaError_t err = set_max_dynamic_smem(kernel, kTile * (int)sizeof(float));
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&P};
    return cudaLaunchKernelExC(&cfg, kernel, args);
}

}  // namespace bl
