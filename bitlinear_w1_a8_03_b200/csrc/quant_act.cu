// Per-token absmax int8 activation quantisation.
//
// "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.4 and §4.1:
// β = max|x| + 1e-8, x̃ = clip(round(127·x/β), -127, 127), taken per token
// (one row of x) as nxmr.cn/news/148658 §3.2 motivates.
//
// One CTA per token row.  Rows of up to kThreads·kVecPerThread 16-byte vectors
// are loaded once into registers (one HBM read of x, one write of x̃); longer
// or unaligned rows are read twice (the second read hits L1/L2).  The kernel
// is HBM-bound: 2 (bf16) or 4 (fp32) bytes in + 1 byte out per element.
#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {
namespace {

constexpr int kThreads = 512;
constexpr int kVecPerThread = 8;

struct ActParams {
    bitlinear_act_problem p[kMaxGroup];
    int64_t row_begin[kMaxGroup + 1];
    int count;
    int early_trigger;  // release the next PDL kernel before waiting on the previous one
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
    __device__ static void unpack(const uint4& v, float* out) {
        out[0] = __uint_as_float(v.x);
        out[1] = __uint_as_float(v.y);
        out[2] = __uint_as_float(v.z);
        out[3] = __uint_as_float(v.w);
    }
    __device__ static void load(const float* p, float* out) { unpack(ld_shared_ro16(p), out); }
};
template <>
struct Vec<uint16_t> {
    static constexpr int n = 8;
    __device__ static void unpack(const uint4& v, float* out) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ static void load(const uint16_t* p, float* out) { unpack(ld_shared_ro16(p), out); }
};

template <int V>
__device__ __forceinline__ void store_codes(int8_t* q, const float* f, float beta) {
    uint32_t packed[V / 4];
#pragma unroll
    for (int j = 0; j < V / 4; ++j) {
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) w |= (uint32_t)(uint8_t)quantize_one(f[4 * j + b], beta) << (8 * b);
        packed[j] = w;
    }
    if constexpr (V == 4) {
        *reinterpret_cast<uint32_t*>(q) = packed[0];
    } else {
        *reinterpret_cast<uint2*>(q) = make_uint2(packed[0], packed[1]);
    }
}

__device__ __forceinline__ float block_max(float mx) {
    __shared__ float warp_max[kThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) mx = fmaxf(mx, warp_max[w]);
    return mx;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) act_quant_kernel(const __grid_constant__ ActParams P) {
    // Programmatic dependent launch: the product kernel that follows may start
    // and stream its weights once this kernel triggers; it waits for x̃ and β
    // itself.  By default the trigger comes after this kernel's own wait, i.e.
    // after everything before it on the stream has finished; early_trigger
    // (constant weights) releases it at once.  x is read only after the wait,
    // whatever produced it.
    if (P.early_trigger) griddep_launch_dependents();
    griddep_wait();
    if (!P.early_trigger) griddep_launch_dependents();
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

    const int64_t nvec = K / V;
    if (vec && nvec <= (int64_t)kThreads * kVecPerThread) {
        // single pass: the row stays in registers between absmax and quantise
        uint4 buf[kVecPerThread];
        float mx = 0.0f;
#pragma unroll
        for (int j = 0; j < kVecPerThread; ++j) {
            const int64_t i = threadIdx.x + (int64_t)j * kThreads;
            if (i < nvec) {
                buf[j] = ld_shared_ro16(x + i * V);
                float f[V];
                Vec<T>::unpack(buf[j], f);
#pragma unroll
                for (int e = 0; e < V; ++e) mx = fmaxf(mx, fabsf(f[e]));  // exact, order-free
            }
        }
        const float beta = __fadd_rn(block_max(mx), 1e-8f);
        if (threadIdx.x == 0) pr.beta[m] = beta;
#pragma unroll
        for (int j = 0; j < kVecPerThread; ++j) {
            const int64_t i = threadIdx.x + (int64_t)j * kThreads;
            if (i < nvec) {
                float f[V];
                Vec<T>::unpack(buf[j], f);
                store_codes<V>(q + i * V, f, beta);
            }
        }
        return;
    }

    // two passes: absmax, then quantise (the second read hits L1/L2)
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
    const float beta = __fadd_rn(block_max(mx), 1e-8f);
    if (threadIdx.x == 0) pr.beta[m] = beta;

    if (vec) {
        for (int64_t i = (int64_t)threadIdx.x * V; i < K; i += (int64_t)kThreads * V) {
            float f[V];
            Vec<T>::load(x + i, f);
            store_codes<V>(q + i, f, beta);
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += kThreads) q[i] = quantize_one(load_as_f32(x, i), beta);
    }
}

}  // namespace

cudaError_t launch_quantize_act(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                cudaStream_t stream, bool pdl, bool early_trigger) {
    ActParams P{};
    P.count = count;
    P.early_trigger = early_trigger ? 1 : 0;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        P.p[i] = problems[i];
        P.row_begin[i] = rows;
        rows += problems[i].M;
    }
    P.row_begin[count] = rows;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dtype == BL_BF16) return cudaLaunchKernelEx(&cfg, act_quant_kernel<uint16_t>, P);
    return cudaLaunchKernelEx(&cfg, act_quant_kernel<float>, P);
}

}  // namespace bl
