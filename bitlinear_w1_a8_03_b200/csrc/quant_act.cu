// Per-token absmax int8 activation quantisation.
//
// "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.4 and §4.1:
// β = max|x| + 1e-8, x̃ = clip(round(127·x/β), -127, 127), taken per token
// (one row of x) as nxmr.cn/news/148658 §3.2 motivates.
//
// Optionally the input is the float32 sum of two activations (the residual
// addition between layers, which stays in floating point, §6.1), added
// element-wise with one binary32 rounding and optionally stored.
//
// One CTA per token row.  Rows of up to blockDim·kVecPerThread 16-byte vectors
// are loaded once into registers (one HBM read of x, one write of x̃); longer
// or unaligned rows are read twice (the second read hits L1/L2).  The kernel
// is HBM-bound: 2 (bf16) or 4 (fp32) bytes in + 1 byte out per element.  With
// few rows (decode) each CTA has 512 threads so a row finishes soonest; with
// many rows (prefill) the CTA is sized to the register buffer (kVecPerThread
// vectors per thread), so an SM holds many rows' loads in flight at once.
#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {
namespace {

constexpr int kMaxThreads = 512;
constexpr int kVecPerThread = 8;

struct ActParams {
    ActJob p[kMaxGroup];
    int64_t row_begin[kMaxGroup + 1];
    int count;
    int early_trigger;  // release the next PDL kernel before waiting on the previous one
};

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

// x (+ b) for one 16-byte vector of x; b only with float32 x.
template <typename T>
__device__ __forceinline__ uint4 load_sum16(const T* x, const float* b, int64_t i) {
    uint4 v = ld_shared_ro16(x + i);
    if constexpr (Vec<T>::n == 4) {
        if (b) {
            const uint4 w = ld_shared_ro16(b + i);
            v.x = __float_as_uint(__fadd_rn(__uint_as_float(v.x), __uint_as_float(w.x)));
            v.y = __float_as_uint(__fadd_rn(__uint_as_float(v.y), __uint_as_float(w.y)));
            v.z = __float_as_uint(__fadd_rn(__uint_as_float(v.z), __uint_as_float(w.z)));
            v.w = __float_as_uint(__fadd_rn(__uint_as_float(v.w), __uint_as_float(w.w)));
        }
    }
    return v;
}

template <typename T>
__device__ __forceinline__ float load_sum1(const T* x, const float* b, int64_t i) {
    const float v = load_as_f32(x, i);
    return b ? __fadd_rn(v, b[i]) : v;
}

template <int V>
__device__ __forceinline__ void store_codes(int8_t* q, const float (&f)[V], float beta, float qf) {
    uint32_t packed[V / 4];
    quantize_codes<V>(f, beta, qf, packed);
    if constexpr (V == 4) {
        *reinterpret_cast<uint32_t*>(q) = packed[0];
    } else {
        *reinterpret_cast<uint2*>(q) = make_uint2(packed[0], packed[1]);
    }
}

// blockDim.x is a multiple of 32
__device__ __forceinline__ float block_max(float mx) {
    __shared__ float warp_max[kMaxThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
    __syncthreads();
    const int nw = blockDim.x >> 5;
    mx = warp_max[0];
    for (int w = 1; w < nw; ++w) mx = fmaxf(mx, warp_max[w]);
    return mx;
}

template <typename T>
__global__ void __launch_bounds__(kMaxThreads) act_quant_kernel(const __grid_constant__ ActParams P) {
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
    const ActJob& pr = P.p[pi];
    const int64_t m = row - P.row_begin[pi];
    const int64_t K = pr.K;
    const T* x = static_cast<const T*>(pr.a) + m * K;
    const float* b = pr.b ? pr.b + m * K : nullptr;
    float* xs = pr.x_sum ? pr.x_sum + m * K : nullptr;
    int8_t* q = pr.x_q + m * K;
    constexpr int V = Vec<T>::n;
    const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && ((reinterpret_cast<uintptr_t>(q) & (V - 1)) == 0) &&
                     ((reinterpret_cast<uintptr_t>(b) & 15) == 0) && ((reinterpret_cast<uintptr_t>(xs) & 15) == 0) &&
                     (K % V == 0);

    const int64_t nvec = K / V;
    const int nt = blockDim.x;
    if (vec && nvec <= (int64_t)nt * kVecPerThread) {
        // single pass: the row stays in registers between absmax and quantise
        uint4 buf[kVecPerThread];
        float mx = 0.0f;
#pragma unroll
        for (int j = 0; j < kVecPerThread; ++j) {
            const int64_t i = threadIdx.x + (int64_t)j * nt;
            if (i < nvec) {
                buf[j] = load_sum16(x, b, i * V);
                if constexpr (V == 4) {  // only float32 x has a sum
                    if (xs) *reinterpret_cast<uint4*>(xs + i * V) = buf[j];
                }
                float f[V];
                Vec<T>::unpack(buf[j], f);
#pragma unroll
                for (int e = 0; e < V; ++e) mx = fmaxf(mx, fabsf(f[e]));  // exact, order-free
            }
        }
        const float beta = __fadd_rn(block_max(mx), 1e-8f);
        const float qf = quant_factor(beta, 127.0f);
        if (threadIdx.x == 0) pr.beta[m] = beta;
#pragma unroll
        for (int j = 0; j < kVecPerThread; ++j) {
            const int64_t i = threadIdx.x + (int64_t)j * nt;
            if (i < nvec) {
                float f[V];
                Vec<T>::unpack(buf[j], f);
                store_codes<V>(q + i * V, f, beta, qf);
            }
        }
        return;
    }

    // two passes: absmax, then quantise (the second read hits L1/L2)
    float mx = 0.0f;
    if (vec) {
        for (int64_t i = (int64_t)threadIdx.x * V; i < K; i += (int64_t)nt * V) {
            float f[V];
            Vec<T>::unpack(load_sum16(x, b, i), f);
#pragma unroll
            for (int j = 0; j < V; ++j) mx = fmaxf(mx, fabsf(f[j]));
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += nt) mx = fmaxf(mx, fabsf(load_sum1(x, b, i)));
    }
    const float beta = __fadd_rn(block_max(mx), 1e-8f);
    const float qf = quant_factor(beta, 127.0f);
    if (threadIdx.x == 0) pr.beta[m] = beta;

    if (vec) {
        for (int64_t i = (int64_t)threadIdx.x * V; i < K; i += (int64_t)nt * V) {
            const uint4 v = load_sum16(x, b, i);
            if constexpr (V == 4) {
                if (xs) *reinterpret_cast<uint4*>(xs + i) = v;
            }
            float f[V];
            Vec<T>::unpack(v, f);
            store_codes<V>(q + i, f, beta, qf);
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += nt) {
            const float v = load_sum1(x, b, i);
            if (xs) xs[i] = v;
            q[i] = quantize_one(v, beta, qf);
        }
    }
}

// Per-token absmax 4-bit quantisation ("BitNet CPU 实测", cf-1.com/news/5800143
// §2.1: later variants quantise the activations to 4 bits): β = max|x| + 1e-8,
// x̃ = clip(round((x·7)/β), -7, 7), two per byte (element k in byte k/2, the
// low nibble for even k; the high nibble of an odd row's last byte is 0).
// One CTA per row: absmax, then each thread quantises element pairs.
template <typename T>
__global__ void __launch_bounds__(kMaxThreads) act_quant_a4_kernel(const __grid_constant__ ActParams P) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t row = blockIdx.x;
    int pi = 0;
    while (pi + 1 < P.count && row >= P.row_begin[pi + 1]) ++pi;
    const ActJob& pr = P.p[pi];
    const int64_t m = row - P.row_begin[pi];
    const int64_t K = pr.K;
    const T* x = static_cast<const T*>(pr.a) + m * K;
    const int64_t rb = (K + 1) / 2;
    uint8_t* q = reinterpret_cast<uint8_t*>(pr.x_q) + m * rb;
    float mx = 0.0f;
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x) mx = fmaxf(mx, fabsf(load_as_f32(x, i)));
    const float beta = __fadd_rn(block_max(mx), 1e-8f);
    const float qf = quant_factor(beta, 7.0f);
    if (threadIdx.x == 0) pr.beta[m] = beta;
    for (int64_t j = threadIdx.x; j < rb; j += blockDim.x) {
        const int lo = quantize_one_a4(load_as_f32(x, 2 * j), beta, qf);
        const int hi = 2 * j + 1 < K ? quantize_one_a4(load_as_f32(x, 2 * j + 1), beta, qf) : 0;
        q[j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
    }
}

}  // namespace

cudaError_t launch_quantize_act_a4(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                   cudaStream_t stream, bool pdl) {
    ActParams P{};
    P.count = count;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        P.p[i] = ActJob{problems[i].x, nullptr, nullptr, problems[i].x_q, problems[i].beta, problems[i].M,
                        problems[i].K};
        P.row_begin[i] = rows;
        rows += problems[i].M;
    }
    P.row_begin[count] = rows;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dtype == BL_BF16) return cudaLaunchKernelEx(&cfg, act_quant_a4_kernel<uint16_t>, P);
    return cudaLaunchKernelEx(&cfg, act_quant_a4_kernel<float>, P);
}

cudaError_t launch_quantize_act(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                cudaStream_t stream, bool pdl, bool early_trigger) {
    ActJob jobs[kMaxGroup];
    for (int i = 0; i < count; ++i)
        jobs[i] = ActJob{problems[i].x, nullptr, nullptr, problems[i].x_q, problems[i].beta, problems[i].M, problems[i].K};
    return launch_quantize_act_jobs(jobs, count, dtype, stream, pdl, early_trigger);
}

namespace {

// One launch of act_quant_kernel over `count` jobs with `threads` per row.
cudaError_t launch_act_rows(const ActJob* jobs, int count, bitlinear_dtype dtype, cudaStream_t stream, bool pdl,
                            bool early_trigger, int threads) {
    ActParams P{};
    P.count = count;
    P.early_trigger = early_trigger ? 1 : 0;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        P.p[i] = jobs[i];
        P.row_begin[i] = rows;
        rows += jobs[i].M;
    }
    P.row_begin[count] = rows;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(threads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dtype == BL_BF16) return cudaLaunchKernelEx(&cfg, act_quant_kernel<uint16_t>, P);
    return cudaLaunchKernelEx(&cfg, act_quant_kernel<float>, P);
}

}  // namespace

cudaError_t launch_quantize_act_jobs(const ActJob* problems, int count, bitlinear_dtype dtype, cudaStream_t stream,
                                     bool pdl, bool early_trigger) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) rows += problems[i].M;
    // few rows: 512 threads per row.  Many rows: kVecPerThread vectors per
    // thread (at least 2 warps), sized for each problem's K; problems that
    // want different CTA sizes get a launch each (a 4096-wide row in CTAs
    // sized for an 11008-wide one leaves too few bytes in flight per SM).
    if (rows < 2 * (int64_t)dev.sm_count) return launch_act_rows(problems, count, dtype, stream, pdl, early_trigger,
                                                                 kMaxThreads);
    auto threads_for = [&](int64_t K) {
        const int64_t nvec = (K * (dtype == BL_BF16 ? 2 : 4) + 15) / 16;
        const int64_t want = ((nvec + kVecPerThread - 1) / kVecPerThread + 31) / 32 * 32;
        return (int)(want < 64 ? 64 : (want > kMaxThreads ? kMaxThreads : want));
    };
    ActJob group[kMaxGroup];
    bool done[kMaxGroup] = {};
    for (int i = 0; i < count; ++i) {
        if (done[i]) continue;
        const int t = threads_for(problems[i].K);
        int n = 0;
        for (int j = i; j < count; ++j)
            if (!done[j] && threads_for(problems[j].K) == t) {
                group[n++] = problems[j];
                done[j] = true;
            }
        err = launch_act_rows(group, n, dtype, stream, pdl, early_trigger, t);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace bl
