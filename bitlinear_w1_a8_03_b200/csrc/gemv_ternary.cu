// Ternary GEMV / skinny GEMM on CUDA cores: y = (x̃·Ŵᵀ)·(α·β/127) + bias.
//
// The product is the pages' add / subtract / skip ("1.58 位大模型",
// nxmr.cn/news/148658 §3.3): Y[m][n] = Σ_{W=+1} x̃ - Σ_{W=-1} x̃.  Here it is
// evaluated as Σ c·x̃ - Σ x̃ with the stored code c = w + 1 ∈ {0, 1, 2}: one
// mask of a packed word yields four codes as unsigned bytes, and one dp4a
// adds their products with four int8 activations, so a zero weight costs
// nothing extra and ±1 weights become adds and subtracts.  Dequantisation
// and bias follow "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html)
// §2.4–§2.5 and §4.2.
//
// Decode is bound by HBM bytes of the packed weights ("1.58-bit 大模型极限量化
// 实战" §5.1–§5.2; 2kiu.com/news/4928193 §3.1, §3.3): every weight byte is read
// once per token group, coalesced 16 bytes per lane, 512 bytes per warp.
//
// Work split: a warp owns R consecutive output rows and MT tokens; its lanes
// walk the row's 16-byte chunks (64 weights) with stride 32, keep exact int32
// partial sums, then a butterfly shuffle reduces them and R·MT lanes run the
// epilogue.  Warps take tasks from a grid-stride loop over all problems of a
// grouped launch, so several small matrices stream back to back.
#include <mutex>

#include "bl_common.cuh"
#include "bl_launch.h"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct GemvProblem {
    const int8_t* xq;
    const float* beta;
    const uint32_t* W;  // packed rows, row_words 32-bit words each
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int64_t M, N, K;
    int64_t row_words;
    int64_t row_groups;
    int64_t task_begin;
};

struct GemvParams {
    GemvProblem p[kMaxGroup];
    int count;
    int64_t total_tasks;
};

// The 16 activation words (64 int8) of chunk c of one token row; zero past K
// and for tokens past M.  Full chunks need a 16-byte aligned row.
__device__ __forceinline__ void load_act_chunk(const int8_t* xrow, int64_t K, int64_t c, bool full, bool valid,
                                               uint32_t (&a)[16]) {
    if (!valid) {
#pragma unroll
        for (int q = 0; q < 16; ++q) a[q] = 0u;
    } else if (full) {
        const int8_t* p = xrow + 64 * c;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_shared_ro16(p + 16 * v);
            a[4 * v + 0] = u.x;
            a[4 * v + 1] = u.y;
            a[4 * v + 2] = u.z;
            a[4 * v + 3] = u.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            uint32_t w = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int64_t k = 64 * c + 4 * q + b;
                if (k < K) w |= (uint32_t)(uint8_t)xrow[k] << (8 * b);
            }
            a[q] = w;
        }
    }
}

template <int MT, int R>
__global__ void __launch_bounds__(kThreads) gemv_ternary_kernel(const __grid_constant__ GemvParams P) {
    constexpr int NS = (MT == 1) ? 4 : 1;  // MT == 1: one accumulator per code field
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;

    for (int64_t t = warp0; t < P.total_tasks; t += nwarps) {
        int pi = 0;
        while (pi + 1 < P.count && t >= P.p[pi + 1].task_begin) ++pi;
        const GemvProblem& pr = P.p[pi];
        const int64_t lt = t - pr.task_begin;
        const int64_t tg = lt / pr.row_groups;
        const int64_t n0 = (lt - tg * pr.row_groups) * R;
        const int64_t m0 = tg * MT;
        const int64_t chunks = pr.row_words >> 2;
        const int64_t full_chunks = pr.K >> 6;

        int acc[R][MT][NS];
        int sx[MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int s = 0; s < NS; ++s) acc[r][m][s] = 0;
#pragma unroll
        for (int m = 0; m < MT; ++m) sx[m] = 0;

        for (int64_t c = lane; c < chunks; c += 32) {
            uint4 w[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r] = (n0 + r < pr.N) ? ld_stream16(pr.W + (n0 + r) * pr.row_words + 4 * c)
                                       : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
            uint32_t a[MT][16];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                load_act_chunk(pr.xq + (m0 + m) * pr.K, pr.K, c, c < full_chunks, m0 + m < pr.M, a[m]);
#pragma unroll
                for (int q = 0; q < 16; ++q) sx[m] = dp4a_s8s8(0x01010101u, a[m][q], sx[m]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t word = word_of(w[r], j);
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        if constexpr (MT == 1) {
                            // codes of weights 16j+4s .. 16j+4s+3, each times 4^s
                            const uint32_t codes = word & (0x03030303u << (2 * s));
                            acc[r][0][s] = dp4a_u8s8(codes, a[0][4 * j + s], acc[r][0][s]);
                        } else {
                            const uint32_t codes = (word >> (2 * s)) & 0x03030303u;
#pragma unroll
                            for (int m = 0; m < MT; ++m) acc[r][m][0] = dp4a_u8s8(codes, a[m][4 * j + s], acc[r][m][0]);
                        }
                    }
                }
            }
        }

        // Σ (c - 1)·x̃ per (row, token), exact in int32; then all-reduce over the warp.
        int v[R * MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int d;
                if constexpr (MT == 1)
                    d = acc[r][0][0] + (acc[r][0][1] >> 2) + (acc[r][0][2] >> 4) + (acc[r][0][3] >> 6);
                else
                    d = acc[r][m][0];
                v[m * R + r] = d - sx[m];
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int i = 0; i < R * MT; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], off);

        if (lane < R * MT) {
            int val = 0;
#pragma unroll
            for (int i = 0; i < R * MT; ++i)
                if (i == lane) val = v[i];
            const int r = lane % R, m = lane / R;
            const int64_t n = n0 + r, mm = m0 + m;
            if (n < pr.N && mm < pr.M) {
                const float s = dequant_scale(*pr.alpha, pr.beta[mm]);
                float out = __fmul_rn((float)val, s);
                if (pr.bias) out = __fadd_rn(out, pr.bias[n]);
                pr.y[mm * pr.N + n] = out;
                if (pr.acc_out) pr.acc_out[mm * pr.N + n] = val;
            }
        }
    }
}

// Any K and any x̃ alignment: one warp per output element, byte loads.
__global__ void __launch_bounds__(kThreads) gemv_generic_kernel(const __grid_constant__ GemvParams P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t t = warp0; t < P.total_tasks; t += nwarps) {
        int pi = 0;
        while (pi + 1 < P.count && t >= P.p[pi + 1].task_begin) ++pi;
        const GemvProblem& pr = P.p[pi];
        const int64_t lt = t - pr.task_begin;
        const int64_t m = lt / pr.N, n = lt - m * pr.N;
        const int8_t* xrow = pr.xq + m * pr.K;
        const uint32_t* wrow = pr.W + n * pr.row_words;
        int acc = 0;
        for (int64_t g = lane; g < pr.row_words; g += 32) {
            const uint32_t word = wrow[g];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t k = 16 * g + i;
                if (k < pr.K) {
                    const uint32_t code = (word >> (8 * (i & 3) + 2 * (i >> 2))) & 3u;
                    const int x = xrow[k];
                    acc += (code == 2u) ? x : ((code == 0u) ? -x : 0);
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            const float s = dequant_scale(*pr.alpha, pr.beta[m]);
            float out = __fmul_rn((float)acc, s);
            if (pr.bias) out = __fadd_rn(out, pr.bias[n]);
            pr.y[m * pr.N + n] = out;
            if (pr.acc_out) pr.acc_out[m * pr.N + n] = acc;
        }
    }
}

template <int MT, int R>
cudaError_t launch_fast(GemvParams& P, const DeviceInfo& dev, cudaStream_t stream) {
    int64_t total = 0;
    for (int i = 0; i < P.count; ++i) {
        GemvProblem& q = P.p[i];
        q.row_groups = (q.N + R - 1) / R;
        q.task_begin = total;
        total += q.row_groups * ((q.M + MT - 1) / MT);
    }
    P.total_tasks = total;
    static int occ[64] = {};
    static std::once_flag once;
    std::call_once(once, [] {
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ[0], gemv_ternary_kernel<MT, R>, kThreads, 0);
    });
    const int per_sm = occ[0] > 0 ? occ[0] : 1;
    int64_t blocks = (total + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)dev.sm_count * per_sm;
    if (blocks > cap) blocks = cap;
    gemv_ternary_kernel<MT, R><<<(unsigned)blocks, kThreads, 0, stream>>>(P);
    return cudaGetLastError();
}

cudaError_t launch_generic(GemvParams& P, const DeviceInfo& dev, cudaStream_t stream) {
    int64_t total = 0;
    for (int i = 0; i < P.count; ++i) {
        P.p[i].task_begin = total;
        total += P.p[i].M * P.p[i].N;
    }
    P.total_tasks = total;
    int64_t blocks = (total + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)dev.sm_count * 8;
    if (blocks > cap) blocks = cap;
    gemv_generic_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward(const bitlinear_forward_problem* problems, int count, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    GemvParams P{};
    P.count = count;
    bool fast = true;
    int64_t max_m = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        GemvProblem& q = P.p[i];
        q.xq = s.x_q;
        q.beta = s.beta;
        q.W = reinterpret_cast<const uint32_t*>(s.W_packed);
        q.alpha = s.alpha;
        q.bias = s.bias;
        q.y = s.y;
        q.acc_out = s.acc_out;
        q.M = s.M;
        q.N = s.N;
        q.K = s.K;
        q.row_words = (int64_t)bitlinear_packed_row_bytes(s.K) / 4;
        fast = fast && (s.K % 16 == 0) && ((reinterpret_cast<uintptr_t>(s.x_q) & 15) == 0);
        if (s.M > max_m) max_m = s.M;
    }
    if (!fast) return launch_generic(P, dev, stream);
    if (max_m == 1) return launch_fast<1, 8>(P, dev, stream);
    if (max_m == 2) return launch_fast<2, 4>(P, dev, stream);
    return launch_fast<4, 4>(P, dev, stream);
}

}  // namespace bl
