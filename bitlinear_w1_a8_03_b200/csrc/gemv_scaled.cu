// Ternary product with a finer scale granularity than the tensor: one α per
// output row ("1.58 位大模型", nxmr.cn/news/148658 §3.1, §4.2: alpha is the mean
// |w| of each row), or one α per block of `group` consecutive input features
// of a row (2kiu.com/news/4928193 §2.3, §4.2: one scale per 128 elements,
// scale[C_out][C_in / 128]).
//
// For each block b of row n the integer sum acc_b = Σ_{k in b} x̃·ŵ is exact
// (add / subtract / skip via masked dp4a, as in the streaming GEMV); then
// S = Σ_b α_{n,b}·acc_b and y = RN32( RN32(S)·RN32(RN64(β_m/127)) ) (+ bias):
// the activations' per-token dequantisation, then the weights' scale, which
// [1.58 位大模型] §4.3 applies to the product afterwards.  With one block per
// row S = α_n·acc is exact, so y is reproducible bit for bit; with several
// blocks S is summed in binary64 (each term α_b·acc_b is exact in binary64).
//
// The same kernel serves the 4-bit activations ("BitNet CPU 实测",
// cf-1.com/news/5800143 §2.1): x̃ ∈ [-7, 7] packed two per byte, with one α
// for the tensor and y = fp32(acc)·RN32(RN64(α·β/7)) (+ bias).
//
// CUDA cores, one warp per group of 4 rows × all K (no cross-warp sums), the
// rows' 16-byte words loaded straight into registers one chunk per lane, the
// next step's words requested before this step's arithmetic.  At most four
// tokens per pass; more tokens are taken four at a time.
#include <type_traits>

#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {
namespace {

constexpr int kRows = 4;     // rows per work item
// warps per CTA: 16 for one token (more loads in flight per SM: one α per
// 128-block went from 60 to 41 µs on the 7B set), 8 for more tokens, whose
// larger register sets would spill at 16
__host__ __device__ constexpr int warps_for(int MT) { return MT == 1 ? 16 : 8; }
constexpr int kPerSM = 3;    // CTAs per SM in the grid (one resident per SM by registers; later waves even out the end)

struct ScProblem {
    const int8_t* xq;
    const float* beta;
    const uint8_t* W;
    const float* alpha;  // [N][G]
    const float* bias;
    float* y;
    int32_t* acc_out;    // one block per row only
    int32_t M, N, K;
    int32_t row_bytes, C, full_chunks;
    int32_t G;           // blocks per row
    int32_t chunks_per_block;  // group / 64 (blocks of several rows' chunks), 0 when one block per row
    int32_t rgn, tgn;    // row groups, token groups
    int32_t x_stride;    // bytes per token row of x̃ (K, or ceil(K/2) for 4-bit activations)
    int64_t item_begin;  // first work item (token group, row group) of this problem
};

struct ScParams {
    ScProblem p[kMaxGroup];
    int count;
    int64_t total_items;
};

__device__ __forceinline__ void sc_load_rows(const ScProblem& pr, int rg, int chunk, bool valid, uint4 (&w)[kRows]) {
    const uint8_t* base = pr.W + (int64_t)chunk * 16;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int row = min(rg * kRows + r, pr.N - 1);
        w[r] = valid ? ld_stream16(base + (int64_t)row * pr.row_bytes) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// 64 activations (one chunk) of one token from global x̃, zero past K.
__device__ __forceinline__ void sc_load_x(const int8_t* xrow, int K, int chunk, bool full, uint32_t (&a)[16]) {
    if (full) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_shared_ro16(xrow + 64 * chunk + 16 * v);
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
                const int k = 64 * chunk + 4 * q + b;
                if (k < K) w |= (uint32_t)(uint8_t)xrow[k] << (8 * b);
            }
            a[q] = w;
        }
    }
}

template <typename T, int V>
__device__ __forceinline__ T sc_reduce_scatter(T (&v)[V], int lane, int& idx) {
    idx = 0;
#pragma unroll
    for (int half = V / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const T send = upper ? v[i] : v[i + half];
            const T keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
        if (upper) idx += half;
    }
    T r = v[0];
#pragma unroll
    for (int off = 16 / V; off >= 1; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    return r;
}

// 64 4-bit activations (one chunk, 32 bytes) of one token, as 16 words of
// four int8, zero past K.
__device__ __forceinline__ void sc_load_x4(const uint8_t* xrow, int K, int chunk, bool full, uint32_t (&a)[16]) {
    uint32_t w[8];
    if (full) {
        const uint4 u0 = ld_shared_ro16(xrow + 32 * chunk), u1 = ld_shared_ro16(xrow + 32 * chunk + 16);
        w[0] = u0.x, w[1] = u0.y, w[2] = u0.z, w[3] = u0.w, w[4] = u1.x, w[5] = u1.y, w[6] = u1.z, w[7] = u1.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t v = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int k = 64 * chunk + 8 * i + 2 * b;  // the byte's first element
                if (k < K) v |= (uint32_t)xrow[k / 2] << (8 * b);
            }
            w[i] = v;
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) unpack_a4(w[i], a[2 * i], a[2 * i + 1]);
}

enum ScaleMode { kTensor = 0, kRow = 1, kBlocks = 2 };

// MT tokens per pass; MODE: one α (tensor), one per row, several per row
// (binary64 sums of α_b·acc_b); A4: packed 4-bit activations.
template <int MT, int MODE, bool A4>
__global__ void __launch_bounds__(warps_for(MT) * 32, 1) gemv_scaled_kernel(const __grid_constant__ ScParams P) {
    constexpr int kWarps = warps_for(MT);
    constexpr int V = kRows * MT;
    constexpr bool BLOCKS = MODE == kBlocks;
    using Acc = typename std::conditional<BLOCKS, double, int>::type;
    __shared__ ScProblem prob[kMaxGroup];
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();
    for (int i = threadIdx.x; i < P.count; i += blockDim.x) prob[i] = P.p[i];
    __syncthreads();
    griddep_wait();  // x̃, β (and α) may come from the preceding kernels

    const int64_t warp0 = ((int64_t)blockIdx.x * kWarps) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    for (int64_t item = warp0; item < P.total_items; item += nwarps) {
        int p = 0;
        while (p + 1 < P.count && item >= prob[p + 1].item_begin) ++p;
        const ScProblem& pr = prob[p];
        const int64_t local = item - pr.item_begin;
        const int tg = (int)(local / pr.rgn), rg = (int)(local - (int64_t)tg * pr.rgn);
        const int m0 = tg * MT;

        Acc tot[kRows][MT];  // per lane: Σ over its chunks (int: Σ c·x̃ - Σ x̃; double: Σ α_b·(...))
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) tot[r][m] = 0;
        uint4 w[kRows];
        sc_load_rows(pr, rg, lane, lane < pr.C, w);
        for (int c = 0; c < pr.C; c += 32) {
            const int j = c + lane;
            const bool valid = j < pr.C;
            uint4 wn[kRows];
            if (c + 32 < pr.C) sc_load_rows(pr, rg, j + 32, j + 32 < pr.C, wn);
            uint32_t xa[MT][16];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (valid && m0 + m < pr.M) {
                    if constexpr (A4)
                        sc_load_x4(reinterpret_cast<const uint8_t*>(pr.xq) + (int64_t)(m0 + m) * pr.x_stride, pr.K, j,
                                   j < pr.full_chunks, xa[m]);
                    else
                        sc_load_x(pr.xq + (int64_t)(m0 + m) * pr.x_stride, pr.K, j, j < pr.full_chunks, xa[m]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) xa[m][q] = 0u;
                }
            }
            int acc[kRows][MT][4];
            int sx[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                sx[m] = 0;
#pragma unroll
                for (int q = 0; q < 16; ++q) sx[m] = dp4a_s8s8(0x01010101u, xa[m][q], sx[m]);
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[r][m][q] = 0;
            }
#pragma unroll
            for (int wj = 0; wj < 4; ++wj)
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        const uint32_t codes = word_of(w[r], wj) & (0x03030303u << (2 * q));
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[r][m][q] = dp4a_u8s8(codes, xa[m][4 * wj + q], acc[r][m][q]);
                    }
            // this chunk's exact partial of each (row, token)
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                float a_b = 0.0f;
                if constexpr (BLOCKS) {
                    const int row = min(rg * kRows + r, pr.N - 1);
                    if (valid) a_b = pr.alpha[(int64_t)row * pr.G + j / pr.chunks_per_block];
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const int d = acc[r][m][0] + (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) + (acc[r][m][3] >> 6) - sx[m];
                    if constexpr (BLOCKS)
                        tot[r][m] = __fma_rn((double)a_b, (double)d, tot[r][m]);  // α_b·d is exact in binary64
                    else
                        tot[r][m] += d;
                }
            }
#pragma unroll
            for (int r = 0; r < kRows; ++r) w[r] = wn[r];
        }
        // reduce over the lanes, dequantise, store
        Acc v[V];
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[m * kRows + r] = tot[r][m];
        int idx;
        const Acc val = sc_reduce_scatter<Acc, V>(v, lane, idx);
        const int r = idx % kRows, m = idx / kRows;
        const int row = rg * kRows + r, tok = m0 + m;
        if ((lane & (32 / V - 1)) == 0 && row < pr.N && tok < pr.M) {
            float out;
            if constexpr (MODE == kTensor) {
                const float s = A4 ? dequant_scale_a4(*pr.alpha, pr.beta[tok]) : dequant_scale(*pr.alpha, pr.beta[tok]);
                out = __fmul_rn((float)val, s);
            } else {
                const float s = __double2float_rn(__ddiv_rn((double)pr.beta[tok], 127.0));
                float S;
                if constexpr (BLOCKS)
                    S = __double2float_rn(val);
                else
                    S = __fmul_rn((float)val, pr.alpha[row]);  // α_n·acc, one binary32 rounding
                out = __fmul_rn(S, s);
            }
            if (pr.bias) out = __fadd_rn(out, pr.bias[row]);
            pr.y[(int64_t)tok * pr.N + row] = out;
            if constexpr (!BLOCKS) {
                if (pr.acc_out) pr.acc_out[(int64_t)tok * pr.N + row] = (int)val;
            }
        }
    }
}

template <int MT, int MODE, bool A4>
cudaError_t launch_scaled_mt(const ScaledProblem* problems, int count, cudaStream_t stream, bool pdl) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    ScParams P{};
    P.count = count;
    int64_t items = 0;
    for (int i = 0; i < count; ++i) {
        const ScaledProblem& s = problems[i];
        ScProblem& q = P.p[i];
        q.xq = s.x_q;
        q.beta = s.beta;
        q.W = s.W_packed;
        q.alpha = s.alpha;
        q.bias = s.bias;
        q.y = s.y;
        q.acc_out = s.acc_out;
        q.M = (int32_t)s.M;
        q.N = (int32_t)s.N;
        q.K = (int32_t)s.K;
        q.row_bytes = (int32_t)bitlinear_packed_row_bytes(s.K);
        q.C = q.row_bytes / 16;
        // 16-byte activation loads need 16-byte aligned x̃ rows; else bytes
        q.x_stride = A4 ? (int32_t)((s.K + 1) / 2) : q.K;
        const bool aligned = q.x_stride % 16 == 0 && (reinterpret_cast<uintptr_t>(s.x_q) & 15) == 0;
        q.full_chunks = aligned ? q.K / 64 : 0;
        q.G = (int32_t)((s.K + s.group - 1) / s.group);
        q.chunks_per_block = s.group >= s.K ? 0 : (int32_t)(s.group / 64);
        q.rgn = (q.N + kRows - 1) / kRows;
        q.tgn = (q.M + MT - 1) / MT;
        q.item_begin = items;
        items += (int64_t)q.rgn * q.tgn;
    }
    P.total_items = items;
    constexpr int kWarps = warps_for(MT);
    int64_t grid = (int64_t)dev.sm_count * kPerSM;
    const int64_t need = (items + kWarps - 1) / kWarps;
    if (grid > need) grid = need;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_scaled_kernel<MT, MODE, A4>, P);
}

}  // namespace

cudaError_t launch_forward_scaled(const ScaledProblem* problems, int count, cudaStream_t stream, bool pdl) {
    int64_t max_m = 0;
    bool blocks = false;
    for (int i = 0; i < count; ++i) {
        max_m = problems[i].M > max_m ? problems[i].M : max_m;
        blocks = blocks || problems[i].group < problems[i].K;
    }
    if (blocks) {
        if (max_m == 1) return launch_scaled_mt<1, kBlocks, false>(problems, count, stream, pdl);
        if (max_m == 2) return launch_scaled_mt<2, kBlocks, false>(problems, count, stream, pdl);
        return launch_scaled_mt<4, kBlocks, false>(problems, count, stream, pdl);
    }
    if (max_m == 1) return launch_scaled_mt<1, kRow, false>(problems, count, stream, pdl);
    if (max_m == 2) return launch_scaled_mt<2, kRow, false>(problems, count, stream, pdl);
    return launch_scaled_mt<4, kRow, false>(problems, count, stream, pdl);
}

cudaError_t launch_forward_a4(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl) {
    ScaledProblem sp[kMaxGroup];
    int64_t max_m = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& f = problems[i];
        sp[i] = ScaledProblem{f.x_q, f.beta, f.W_packed, f.alpha, f.bias, f.y, f.acc_out, f.M, f.N, f.K, f.K};
        max_m = f.M > max_m ? f.M : max_m;
    }
    if (max_m == 1) return launch_scaled_mt<1, kTensor, true>(sp, count, stream, pdl);
    if (max_m == 2) return launch_scaled_mt<2, kTensor, true>(sp, count, stream, pdl);
    return launch_scaled_mt<4, kTensor, true>(sp, count, stream, pdl);
}

}  // namespace bl
