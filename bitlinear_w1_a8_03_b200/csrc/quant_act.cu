// Per-token absmax int8 activation quantisation.
//
// "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.4 and §4.1:
// β = max|x| + 1e-8, x̃ = clip(round(127·x/β), -127, 127), taken per token
// (one row of x) as nxmr.cn/news/148658 §3.2 motivates.
//
// One CTA per token row.  The row is read twice (absmax, then quantise); the
// second read hits L1/L2, so HBM sees one read of x and one write of x̃.  The
// kernel is HBM-bound: 2 (bf16) or 4 (fp32) bytes in + 1 byte out per element.
#include "bl_common.cuh"
#include "bl_launch.h"

namespace bl {
namespace {

constexpr int kThreads = 256;

struct ActParams {
    bitlinear_act_problem p[kMaxGroup];
    int64_t row_begin[kMaxGroup + 1];
    int count;
};

__device__ __forceinline__ int8_t quantize_one(float v, float beta) {
    float t = __fdiv_rn(__fmul_rn(v, 127.0f), beta);
    float r = rintf(t);  // round half to even
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return (int8_t)__float2int_rn(r);
}

template <typename T>
struct Vec;  // 16-byte vector of T
template <>
struct Vec<float> {
    static constexpr int n = 4;
    __device__ static void load(const float* p, float* out) {
        uint4 v = ld_shared_ro16(p);
        out[0] = __uint_as_float(v.x);
        out[1] = __uint_as_float(v.y);
        out[2] = __uint_as_float(v.z);
        out[3] = __uint_as_float(v.w);
    }
};
template <>
struct Vec<uint16_t> {
    static constexpr int n = 8;
    __device__ static void load(const uint16_t* p, float* out) {
        uint4 v = ld_shared_ro16(p);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

template <typename T>
__global__ void __launch_bounds__(kThreads) act_quant_kernel(const __grid_constant__ ActParams P) {
    const int64_t row = blockIdx.x;
    int pi = 0;
    while (pi + 1 < P.count && row >= P.row_begin[pi + 1]) ++pi;
    const bitlinear_act_problem& pr = P.p[pi];
    const int64_t m = row - P.row_begin[pi];
    const int64_t K = pr.K;
    const T* x = static_cast<const T*>(pr.x) + m * K;
    int8_t* q = pr.x_q + m * K;
    constexpr int V = Vec<T>::n;
    const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && ((reinterpret_cast<uintptr_t>(q) & (V - 1)) == 0) &&
                     (K % V == 0);

    // absmax: max is exact and order-free
    float mx = 0.0f;
    if (vec) {
        for (int64_t i = (int64_t)threadIdx.x * V; i < K; i += (int64_t)kThreads * V) {
            float f[V];
            Vec<T>::load(x + i, f);
#pragma unroll
            for (int j = 0; j < V; ++j) mx = fmaxf(mx, fabsf(f[j]));
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += kThreads) mx = fmaxf(mx, fabsf(load_as_f32(x, i)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __shared__ float warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) mx = fmaxf(mx, warp_max[w]);
    const float beta = __fadd_rn(mx, 1e-8f);
    if (threadIdx.x == 0) pr.beta[m] = beta;

    if (vec) {
        for (int64_t i = (int64_t)threadIdx.x * V; i < K; i += (int64_t)kThreads * V) {
            float f[V];
            Vec<T>::load(x + i, f);
            uint32_t packed[V / 4];
#pragma unroll
            for (int j = 0; j < V / 4; ++j) {
                uint32_t w = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) w |= (uint32_t)(uint8_t)quantize_one(f[4 * j + b], beta) << (8 * b);
                packed[j] = w;
            }
            if constexpr (V == 4) {
                *reinterpret_cast<uint32_t*>(q + i) = packed[0];
            } else {
                *reinterpret_cast<uint2*>(q + i) = make_uint2(packed[0], packed[1]);
            }
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += kThreads) q[i] = quantize_one(load_as_f32(x, i), beta);
    }
}

}  // namespace

cudaError_t launch_quantize_act(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                cudaStream_t stream) {
    ActParams P{};
    P.count = count;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        P.p[i] = problems[i];
        P.row_begin[i] = rows;
        rows += problems[i].M;
    }
    P.row_begin[count] = rows;
    dim3 grid((unsigned)rows);
    if (dtype == BL_BF16)
        act_quant_kernel<uint16_t><<<grid, kThreads, 0, stream>>>(P);
    else
        act_quant_kernel<float><<<grid, kThreads, 0, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace bl
