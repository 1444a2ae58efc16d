// Ternary GEMV for at most four tokens on CUDA cores: y = (x̃·Ŵᵀ)·(α·β/127) + bias.
//
// The product is the pages' add / subtract / skip ("1.58 位大模型",
// nxmr.cn/news/148658 §3.3): Y[m][n] = Σ_{W=+1} x̃ - Σ_{W=-1} x̃.  It is
// evaluated as Σ c·x̃ - Σ x̃ with the stored code c = w + 1 ∈ {0, 1, 2}: one
// mask of a packed word yields four codes as unsigned bytes (×4^s), and one
// dp4a adds their products with four int8 activations, so a zero weight costs
// nothing extra and ±1 weights become adds and subtracts.  Σ x̃ is one number
// per token and problem, subtracted once per output.  Dequantisation and bias
// follow "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.4–§2.5
// and §4.2.
//
// Decode is bound by the HBM bytes of the packed weights ("1.58-bit 大模型极限
// 量化实战" §5.1–§5.2; 2kiu.com/news/4928193 §3.1, §3.3), so the kernel is built
// to keep HBM streaming while the arithmetic keeps up:
//  * persistent grid, one CTA per SM; the work (row groups of 8 rows × 16-byte
//    chunks, over every problem of a grouped launch) is cut into contiguous
//    CTA ranges of equal chunk count snapped to row-group boundaries, and each
//    CTA range into equal warp ranges; a row group split between warps is
//    summed exactly in shared memory and finished by its last contributor;
//  * each warp streams its segments (8 rows × up to SC chunks) through its own
//    ring of D shared-memory stages with 1-D bulk copies (TMA), one row per
//    lane, D segments ahead; the first D go out before the dependency wait
//    (programmatic dependent launch: the weights do not depend on the
//    previous kernel); the segment's activations are read before its wait;
//  * the arithmetic loads the 8 rows' words of a chunk first and then walks
//    (word, field) pairs with the rows innermost, so consecutive dp4a go to 8
//    independent accumulators; a reduce-scatter of shuffles leaves each
//    (row, token) sum in one lane.
//
// Fused mode (chosen by the host): the kernel also does the per-token
// activation quantisation.  Right after its dependency wait each CTA
// quantises the input rows of the (at most two) problems its range covers
// into shared-memory slots with the same arithmetic as the activation kernel;
// the CTA owning a problem's first row group writes x̃ and β (and a residual
// sum) out.  One launch then replaces the quantisation kernel and the product.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {

// Set (first error wins) by a kernel whose bounded wait expired; read and
// cleared by bitlinear_device_error().
static __device__ int g_device_error;

namespace {

constexpr int kRGMax = 8;          // most rows per row group
constexpr int kGemvMaxTokens = 4;  // more tokens go to the tensor-core GEMM
constexpr int kMaxSlots = 2;       // fused: input rows of at most two problems per CTA

struct GProblem {
    const int8_t* xq;
    const float* beta;
    const uint8_t* W;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int32_t M, N, K;
    int32_t row_bytes;    // 16·ceil(K/64)
    int32_t C;            // 16-byte chunks per row
    int32_t full_chunks;  // chunks entirely inside K (the activation tail needs guards)
    int32_t rgn;          // row groups
    int32_t alpha_rows;   // alpha is a per-row table [N] (else one α for the matrix)
    int32_t S;            // steps per row group: ceil(C / 32) (a step gives each lane one chunk)
    int64_t step_begin;   // first step of this problem in the launch
    // fused quantisation (x̃ made in shared memory from x):
    const void* x;          // activations, float32 or bfloat16 [M][K]
    const float* x2;        // nullable float32 second addend
    float* x_sum;           // nullable: stores x (+ x2)
    int32_t write_outputs;  // the owner CTA writes x̃ to xq and β to beta (and x_sum)
    int32_t had_block;      // > 0: x is rotated by the block-diagonal Hadamard first
};

constexpr int kMaxCta = 512;  // most CTAs of one launch

struct GParams {
    GProblem p[kMaxGroup];
    int count;
    int64_t total_steps;
    int32_t cta_begin[kMaxCta + 1];  // first step of each CTA (row-group boundaries), then the end
    int x_bf16;        // fused: activation dtype
    int a4;            // fused: 4-bit activations (codes in [-7, 7], x̃ written as nibbles, scale α·β/7)
    int had;           // fused: the inputs are rotated (every problem has a Hadamard block)
    int32_t slot_row;  // fused: bytes per token row of a shared x̃ slot (64·ceil(K/64) of the widest problem)
};

// ---------------------------------------------------------------- work split
// The work of a launch is a sequence of steps: problem by problem, row group
// by row group, S steps per row group (step s covers chunks 32s .. 32s+31 of
// the RG rows).  Each CTA takes a contiguous range of whole row groups (the
// host balances the ranges, see cta_ranges) and splits it into equal step
// ranges for its warps.
__host__ __device__ __forceinline__ int problem_of_step(const GProblem* P, int count, int64_t u) {
    int p = 0;
    while (p + 1 < count && u >= P[p + 1].step_begin) ++p;
    return p;
}

// ---------------------------------------------------------------- activations
// The last activation chunk of a row when K is not a multiple of 64: bytes
// past K read as zero.  Kept out of line so the full-chunk path stays lean.
__device__ __noinline__ void load_act_tail(const int8_t* xrow, int K, int chunk, uint32_t* a) {
    for (int q = 0; q < 16; ++q) {
        uint32_t w = 0;
        for (int b = 0; b < 4; ++b) {
            const int k = 64 * chunk + 4 * q + b;
            if (k < K) w |= (uint32_t)(uint8_t)xrow[k] << (8 * b);
        }
        a[q] = w;
    }
}

// Shared x̃ slot layout: the four 16-byte pieces of 64-byte chunk c are
// rotated by (c >> 1), so the 16-byte reads of 8 lanes on consecutive chunks
// fall in distinct banks.
__device__ __forceinline__ uint32_t xs_offset(int k) {
    const int c = k >> 6, v = (k >> 4) & 3;
    return (uint32_t)(64 * c + 16 * ((v + (c >> 1)) & 3) + (k & 15));
}

template <int NT>
__device__ __forceinline__ float block_max_n(float mx, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __syncthreads();  // red[] free from any previous use
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) mx = fmaxf(mx, red[w]);
    return mx;
}

// 16 bytes of x (+ x2): 8 bfloat16 or 4 float32 elements, kept raw in
// registers between the absmax and the quantisation (a float32 sum x + x2 is
// formed on load, one binary32 rounding).
// One input row the fused prologue quantises into a shared slot row; the
// fields are copied by value so the prologue reads them from registers.
struct QRow {
    const void* x;    // the problem's activations, float32 or bfloat16 [M][K]
    const float* x2;  // nullable float32 second addend
    int8_t* xq;       // x̃ out (with `out`)
    float* beta;      // β out (with `out`)
    float* x_sum;     // nullable x (+ x2) out (with `out`)
    uint32_t dst;     // shared address of the slot row
    int slot, m, K;
    int had;     // > 0: rotate by the block-diagonal Hadamard of this block size first
    bool valid;  // a row to quantise
    bool out;    // also write x̃, β (and x) to global memory
};

template <typename T>
struct FusedVec;
template <>
struct FusedVec<uint16_t> {
    static constexpr int n = 8;
    __device__ static uint4 load(const QRow& q, int64_t e) {
        return ld_shared_ro16(static_cast<const uint16_t*>(q.x) + e);
    }
    __device__ static void unpack(const uint4& u, float (&f)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct FusedVec<float> {
    static constexpr int n = 4;
    __device__ static uint4 load(const QRow& q, int64_t e) {
        uint4 u = ld_shared_ro16(static_cast<const float*>(q.x) + e);
        if (q.x2) {
            const uint4 v = ld_shared_ro16(q.x2 + e);
            u.x = __float_as_uint(__fadd_rn(__uint_as_float(u.x), __uint_as_float(v.x)));
            u.y = __float_as_uint(__fadd_rn(__uint_as_float(u.y), __uint_as_float(v.y)));
            u.z = __float_as_uint(__fadd_rn(__uint_as_float(u.z), __uint_as_float(v.z)));
            u.w = __float_as_uint(__fadd_rn(__uint_as_float(u.w), __uint_as_float(v.w)));
        }
        return u;
    }
    __device__ static void unpack(const uint4& u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
};

constexpr int kFuseVec = 8;  // 16-byte vectors per thread and row held in registers
constexpr int kFuseRows = 2;  // input rows quantised together (one block reduction)

// Quantises the kFuseRows input rows q[] at once (invalid ones are skipped)
// with the arithmetic of act_quant_kernel (β = max|x| + 1e-8, x̃ =
// quantize_one), zero past K: every load of the rows is issued before the
// first use, and one block reduction yields every β.  β and Σx̃ of a row go
// to xbeta / xsum[slot][m] (xsum zeroed before; the CTA's warps add their
// parts).  Each row must fit NT·kFuseVec 16-byte vectors (the host checks);
// K is a multiple of 16 and x, x2 are 16-byte aligned.
template <typename T, int NT>
__device__ void fused_quantize_rows(const QRow (&q)[kFuseRows], int32_t slot_row, float (*red)[32],
                                    float (*xbeta)[kGemvMaxTokens], int (*xsum)[kGemvMaxTokens], bool a4) {
    const float qmax = a4 ? 7.0f : 127.0f;
    constexpr int V = FusedVec<T>::n;
    uint4 raw[kFuseRows][kFuseVec];
    float mx[kFuseRows];
    int nv[kFuseRows];  // 16-byte vectors per thread (the same in every thread; the last may be empty)
#pragma unroll
    for (int i = 0; i < kFuseRows; ++i) {
        mx[i] = 0.0f;
        const int nvec = q[i].valid ? q[i].K / V : 0;
        nv[i] = (nvec + NT - 1) / NT;
        const int64_t base = (int64_t)q[i].m * q[i].K;
#pragma unroll
        for (int j = 0; j < kFuseVec; ++j) {
            if (j < nv[i]) {
                const int v = threadIdx.x + j * NT;
                raw[i][j] = v < nvec ? FusedVec<T>::load(q[i], base + (int64_t)v * V) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kFuseRows; ++i) {
#pragma unroll
        for (int j = 0; j < kFuseVec; ++j) {
            if (j < nv[i]) {  // zero vectors past K leave the max unchanged
                float f[V];
                FusedVec<T>::unpack(raw[i][j], f);
#pragma unroll
                for (int e = 0; e < V; ++e) mx[i] = fmaxf(mx[i], fabsf(f[e]));  // exact, order-free
            }
        }
    }
    // block max of each row
#pragma unroll
    for (int i = 0; i < kFuseRows; ++i)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], off));
    __syncthreads();  // red[] free from any previous use
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int i = 0; i < kFuseRows; ++i) red[i][threadIdx.x >> 5] = mx[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kFuseRows; ++i) {
        if (!q[i].valid) continue;
        float b = red[i][0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) b = fmaxf(b, red[i][w]);
        const float beta = __fadd_rn(b, 1e-8f);
        const float qf = quant_factor(beta, qmax);
        const int64_t base = (int64_t)q[i].m * q[i].K;
        const int nvec = q[i].K / V;
        int qsum = 0;  // this thread's part of Σx̃
#pragma unroll
        for (int j = 0; j < kFuseVec; ++j) {
            if (j < nv[i]) {
                // vectors past K give zero codes, which is what the slot holds
                // there, so they are stored too while inside it
                const int v = threadIdx.x + j * NT;
                float f[V];
                FusedVec<T>::unpack(raw[i][j], f);
                uint32_t wq[V / 4];
                quantize_codes<V>(f, beta, qf, wq, qmax);
#pragma unroll
                for (int g = 0; g < V / 4; ++g) {
                    if (v >= nvec) wq[g] = 0u;  // past K the codes are 0 whatever β is
                    qsum = dp4a_s8s8(0x01010101u, wq[g], qsum);
                }
                const int k = v * V;
                if (k < slot_row) {
#pragma unroll
                    for (int g = 0; g < V / 4; ++g) sts32(q[i].dst + xs_offset(k + 4 * g), wq[g]);
                }
                if (q[i].out && v < nvec && a4) {
                    // two codes per byte, element 2j in the low nibble ("BitNet CPU 实测" §2.1 variant)
                    uint8_t* o = reinterpret_cast<uint8_t*>(q[i].xq) + (int64_t)q[i].m * (q[i].K / 2) + k / 2;
                    const uint32_t lo = wq[0] & 0x0F0F0F0Fu;
                    const uint32_t t0 = lo | (lo >> 4);  // bytes 0 and 2: codes (0,1) and (2,3)
                    if constexpr (V == 8) {
                        const uint32_t hi = wq[1] & 0x0F0F0F0Fu;
                        *reinterpret_cast<uint32_t*>(o) = __byte_perm(t0, hi | (hi >> 4), 0x6420);
                    } else {
                        *reinterpret_cast<uint16_t*>(o) = (uint16_t)__byte_perm(t0, 0u, 0x0020);
                    }
                } else if (q[i].out && v < nvec) {
                    int8_t* o = q[i].xq + base + k;
                    if constexpr (V == 8)
                        *reinterpret_cast<uint2*>(o) = make_uint2(wq[0], wq[1]);
                    else
                        *reinterpret_cast<uint32_t*>(o) = wq[0];
                    if (q[i].x_sum) {
                        if constexpr (V == 4) {
                            *reinterpret_cast<uint4*>(q[i].x_sum + base + k) = raw[i][j];
                        } else {
#pragma unroll
                            for (int e = 0; e < V; ++e) q[i].x_sum[base + k + e] = f[e];
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, off);
        if ((threadIdx.x & 31) == 0) atomicAdd(&xsum[q[i].slot][q[i].m], qsum);  // integer: exact in any order
        if (threadIdx.x == 0) {
            xbeta[q[i].slot][q[i].m] = beta;
            if (q[i].out) q[i].beta[q[i].m] = beta;
        }
        for (int k = nv[i] * NT * V + 4 * threadIdx.x; k < slot_row; k += 4 * NT) sts32(q[i].dst + xs_offset(k), 0u);
    }
}

// A token's dequantisation factor: RN32(RN64(α·β/127)) for one α per matrix;
// with one α per row the row's α is applied first, y = RN32(RN32(acc·α_n)·s)
// with s = RN32(RN64(β/127)) ("1.58 位大模型", nxmr.cn/news/148658 §3.1, §4.2).
// With 4-bit activations the factor is RN32(RN64(α·β/7)).
__device__ __forceinline__ float token_scale(int alpha_rows, int a4, float alpha, float beta) {
    if (a4) return dequant_scale_a4(alpha, beta);
    return alpha_rows ? __double2float_rn(__ddiv_rn((double)beta, 127.0)) : dequant_scale(alpha, beta);
}

__host__ __device__ constexpr int ilog2_const(int v) { return v <= 1 ? 0 : 1 + ilog2_const(v / 2); }

// Scratch for a rotated row, in the stages that no copy targets before the
// main loop: segment s (SEG floats) is the last stage of warp s's ring.
struct RotScratch {
    uint32_t base;    // shared address of segment 0
    uint32_t stride;  // bytes from one segment to the next (one warp's ring)
    int seg_log2;     // log2 of the floats per segment
    __device__ __forceinline__ uint32_t addr(int e) const {
        return base + (uint32_t)(e >> seg_log2) * stride + 4u * (uint32_t)(e & ((1 << seg_log2) - 1));
    }
};

__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Butterfly stages h, 2h, …, h·R/2 of the rotation over the scratch in one
// pass: each item holds the R elements i + j·h (closed under those stages)
// in registers and runs the stages in order, so every butterfly is the same
// binary32 add or subtract as in a pass per stage.  Returns this thread's
// max |value| written.
template <int R>
__device__ __forceinline__ float rotate_pass(const RotScratch& sc, int K, int lh, int nt) {
    constexpr int r = R == 2 ? 1 : R == 4 ? 2 : 3;
    const int h = 1 << lh;
    float mx = 0.0f;
    for (int it = threadIdx.x; it < K / R; it += nt) {
        const int i = ((it >> lh) << (lh + r)) | (it & (h - 1));
        float f[R];
#pragma unroll
        for (int j = 0; j < R; ++j) f[j] = lds_f32(sc.addr(i + j * h));
#pragma unroll
        for (int st = 1; st < R; st <<= 1)
#pragma unroll
            for (int j = 0; j < R; ++j)
                if (!(j & st)) {
                    const float a = f[j], b = f[j + st];
                    f[j] = __fadd_rn(a, b);
                    f[j + st] = __fsub_rn(a, b);
                }
#pragma unroll
        for (int j = 0; j < R; ++j) {
            sts_f32(sc.addr(i + j * h), f[j]);
            mx = fmaxf(mx, fabsf(f[j]));
        }
    }
    return mx;
}

// One input row rotated, then quantised like fused_quantize_rows: x·H with H
// block-diagonal Sylvester Hadamard of block q.had ("1.58-bit 大模型极限量化实战",
// chenxutan.com/d/5049.html §6.2), butterfly stages h = 1, 2, 4, … each
// rounded to binary32, then β = max|x·H| + 1e-8 and the codes.  A lane holds
// 8 consecutive elements of a 256-element tile (a warp per tile): stages
// h < 8 run in its registers, 8 ≤ h < 256 between lanes by shuffles, and the
// tile goes to the scratch; larger stages run there, up to three per pass.
// K ≤ the scratch's floats, K·(element bytes) ≤ NT·kFuseVec·16, q.had ≥ 8
// (the host checks).
template <typename T, int NT>
__device__ void fused_rotate_quantize_row(const QRow& q, const RotScratch& sc, int32_t slot_row, float (*red)[32],
                                          float (*xbeta)[kGemvMaxTokens], int (*xsum)[kGemvMaxTokens], bool a4) {
    constexpr int V = FusedVec<T>::n;
    constexpr int kLd = 8 / V;                 // 16-byte loads per 8-element unit
    constexpr int kUnits = kFuseVec / kLd;     // units per thread at most
    constexpr int kW = NT / 32;
    const float qmax = a4 ? 7.0f : 127.0f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K = q.K, tiles = (K + 255) / 256;
    const int64_t base = (int64_t)q.m * K;
    // every load first: unit j of this lane is elements 256·(warp + j·kW) + 8·lane + [0, 8)
    uint4 raw[kUnits][kLd];
#pragma unroll
    for (int j = 0; j < kUnits; ++j) {
        const int e = 256 * (warp + j * kW) + 8 * lane;
        if (warp + j * kW < tiles) {
#pragma unroll
            for (int l = 0; l < kLd; ++l)
                raw[j][l] = e < K ? FusedVec<T>::load(q, base + e + l * V) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    const int lhad = 31 - __clz(q.had);
    const int lsh = lhad < 8 ? lhad : 8;  // stages below 2^lsh stay in the warp
    float mx = 0.0f;
#pragma unroll
    for (int j = 0; j < kUnits; ++j) {
        if (warp + j * kW >= tiles) continue;  // the same in every lane of the warp
        float f[8];
#pragma unroll
        for (int l = 0; l < kLd; ++l) {
            float g[V];
            FusedVec<T>::unpack(raw[j][l], g);
#pragma unroll
            for (int e = 0; e < V; ++e) f[l * V + e] = g[e];
        }
#pragma unroll
        for (int h = 1; h < 8; h <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (!(e & h)) {
                    const float a = f[e], b = f[e + h];
                    f[e] = __fadd_rn(a, b);
                    f[e + h] = __fsub_rn(a, b);
                }
        for (int lh = 3; lh < lsh; ++lh) {
            // pair (i, i + h) across lanes lane and lane ^ h/8: the lower lane keeps
            // a + b, the upper one a - b (a from the lower lane)
            const int mask = 1 << (lh - 3);
            const bool upper = (lane & mask) != 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float o = __shfl_xor_sync(0xffffffffu, f[e], mask);
                f[e] = upper ? __fsub_rn(o, f[e]) : __fadd_rn(f[e], o);
            }
        }
        const int e0 = 256 * (warp + j * kW) + 8 * lane;
        if (e0 < K) {
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
            sts128(sc.addr(e0), make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                           __float_as_uint(f[3])));
            sts128(sc.addr(e0 + 4), make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]),
                                               __float_as_uint(f[6]), __float_as_uint(f[7])));
        }
    }
    // the stages from 256 up, two or three per pass (5 → 3 + 2, 4 → 2 + 2)
    for (int lh = lsh; lh < lhad;) {
        const int rest = lhad - lh;
        const int r = rest == 4 ? 2 : rest < 3 ? rest : 3;
        __syncthreads();
        mx = r == 1 ? rotate_pass<2>(sc, K, lh, NT) : r == 2 ? rotate_pass<4>(sc, K, lh, NT) : rotate_pass<8>(sc, K, lh, NT);
        lh += r;
    }
    // β of the rotated row: the max over the last values every thread wrote
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __syncthreads();  // red[] free from any previous use; the scratch is complete
    if (lane == 0) red[0][warp] = mx;
    __syncthreads();
    float bmax = red[0][0];
#pragma unroll
    for (int w = 1; w < kW; ++w) bmax = fmaxf(bmax, red[0][w]);
    const float beta = __fadd_rn(bmax, 1e-8f);
    const float qf = quant_factor(beta, qmax);
    // codes, eight elements per item
    int qsum = 0;
    for (int v = threadIdx.x; v < K / 8; v += NT) {
        const uint4 u0 = lds128_after(sc.addr(8 * v)), u1 = lds128_after(sc.addr(8 * v + 4));
        const float f[8] = {__uint_as_float(u0.x), __uint_as_float(u0.y), __uint_as_float(u0.z), __uint_as_float(u0.w),
                            __uint_as_float(u1.x), __uint_as_float(u1.y), __uint_as_float(u1.z), __uint_as_float(u1.w)};
        uint32_t wq[2];
        quantize_codes<8>(f, beta, qf, wq, qmax);
        qsum = dp4a_s8s8(0x01010101u, wq[0], qsum);
        qsum = dp4a_s8s8(0x01010101u, wq[1], qsum);
        const int k = 8 * v;
        sts32(q.dst + xs_offset(k), wq[0]);
        sts32(q.dst + xs_offset(k + 4), wq[1]);
        if (q.out) {
            if (a4) {
                // two codes per byte, element 2j in the low nibble ("BitNet CPU 实测" §2.1 variant)
                const uint32_t lo = wq[0] & 0x0F0F0F0Fu, hi = wq[1] & 0x0F0F0F0Fu;
                *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(q.xq) + (int64_t)q.m * (K / 2) + k / 2) =
                    __byte_perm(lo | (lo >> 4), hi | (hi >> 4), 0x6420);
            } else {
                *reinterpret_cast<uint2*>(q.xq + base + k) = make_uint2(wq[0], wq[1]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, off);
    if (lane == 0) atomicAdd(&xsum[q.slot][q.m], qsum);  // integer: exact in any order
    if (threadIdx.x == 0) {
        xbeta[q.slot][q.m] = beta;
        if (q.out) q.beta[q.m] = beta;
    }
    for (int k = K + 4 * threadIdx.x; k < slot_row; k += 4 * NT) sts32(q.dst + xs_offset(k), 0u);
    __syncthreads();  // the scratch is free again (for a next row)
}

// ---------------------------------------------------------------- reductions
// Sums v[0..V-1] over the 32 lanes of the warp (V a power of two <= 32).
// Returns the total of index idx in every lane; lanes whose low 5-log2(V)
// bits are zero hold distinct indices 0..V-1.  V-1 + 5-log2(V) shuffles.
template <int V>
__device__ __forceinline__ int reduce_scatter(int (&v)[V], int lane, int& idx) {
    idx = 0;
#pragma unroll
    for (int half = V / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const int send = upper ? v[i] : v[i + half];
            const int keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
        if (upper) idx += half;
    }
    int r = v[0];
#pragma unroll
    for (int off = 16 / V; off >= 1; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    return r;
}

// ---------------------------------------------------------------- the kernel
// 128-byte aligned, so the fused x̃ slots that follow it in shared memory start
// on a 16-byte boundary (they are read with 16-byte loads).
template <int W>
struct alignas(128) GShared {
    int64_t bound[W + 1];                     // warp step ranges inside the CTA
    int part[W][2][kRGMax * kGemvMaxTokens];  // a warp's sums of row groups shared with its neighbours
    GProblem prob[kMaxGroup];  // copy of the problem table (indexed reads of it are cheap here)
    float xbeta[kMaxSlots][kGemvMaxTokens];  // fused: β of each slot's tokens
    int xsum[kMaxSlots][kGemvMaxTokens];     // fused: Σx̃ of each slot's tokens
    float red[kFuseRows][32];                // fused: block reduction scratch
    uint4 zero[4];                           // 64 zero bytes: what idle lanes read as activations
};

// 64 zero bytes in global memory: the activations idle lanes read when x̃
// comes from global memory.
__device__ const uint4 g_zero_chunk[4] = {};

// Where a warp's next weight request comes from: problem p, row group rg,
// step s, the steps left in the warp's range, the problem's fields, and this
// lane's source address in row 0 of the row group for step s (chunk
// 32s + lane) with the other rows' offsets (rows past N repeat row N-1, whose
// results are never written).  The fields and offsets are re-derived only
// when the position enters a new row group; a step moves the address by 512.
template <int RG, int CPL>
struct Feed {
    int p, rg, s, rem;
    int32_t C, S, rgn, N, rb;
    const uint8_t* W;
    const uint8_t* src;    // row 0 of the row group, this lane's chunk of step s
    uint32_t off[RG];      // row r at src + off[r]

    __device__ __forceinline__ void fields(const GProblem* T) {
        const GProblem& q = T[p];
        C = q.C;
        S = q.S;
        rgn = q.rgn;
        N = q.N;
        rb = q.row_bytes;
        W = q.W;
    }
    __device__ __forceinline__ void rows(int lane) {
        const int row0 = rg * RG;
        const int rlast = min(RG, N - row0) - 1;
        src = W + (int64_t)row0 * rb + 16 * (32 * CPL * s + lane);
#pragma unroll
        for (int r = 0; r < RG; ++r) off[r] = (uint32_t)(min(r, rlast) * rb);
    }
    // Requests step s into this lane's column of a stage: chunk 32·CPL·s +
    // 32j + lane of row r at dst + 512·(j·RG + r).  In a row's last step
    // chunks past the end are replaced by the last chunk: their words meet
    // zero activations.
    __device__ __forceinline__ void request(uint32_t dst, int lane) const {
        const int n = C - 32 * CPL * s;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const uint8_t* b =
                src + 512 * j - (n >= 32 * CPL ? 0u : 16u * (uint32_t)max(0, 32 * j + lane - (n - 1)));
#pragma unroll
            for (int r = 0; r < RG; ++r) cp_async16(dst + 512u * (j * RG + r), b + off[r]);
        }
    }
    __device__ __forceinline__ void advance(const GProblem* T, int lane) {
        --rem;
        if (++s < S) {
            src += 512 * CPL;
            return;
        }
        s = 0;
        if (++rg == rgn) {
            rg = 0;
            ++p;
            if (rem > 0) fields(T);
        }
        if (rem > 0) rows(lane);
    }
};

// Problem, row group and step of global step u.
__device__ __forceinline__ void locate_step(const GProblem* T, int count, int64_t u, int& p, int& rg, int& s) {
    p = problem_of_step(T, count, u);
    const int32_t local = (int32_t)(u - T[p].step_begin);
    rg = local / T[p].S;
    s = local - rg * T[p].S;
}

// MT tokens' activations of chunk ch from the shared slot rows (token m at
// xrow + m·slot_row, pieces rotated as xs_offset lays them out); idle lanes
// read the zero block.  Tokens past M read rows the prologue did not write:
// their sums are never stored.
template <int MT>
__device__ __forceinline__ void lds_x(uint32_t xrow, int32_t slot_row, int ch, bool active, uint32_t zero,
                                      uint32_t (&a)[MT][16]) {
    const uint32_t rot = (uint32_t)(ch >> 1);
    const uint32_t b0 = active ? xrow + 64u * (uint32_t)ch : zero;
    const uint32_t dm = active ? (uint32_t)slot_row : 0u;
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = lds128(b0 + (uint32_t)m * dm + 16u * ((v + rot) & 3u));
            a[m][4 * v + 0] = u.x;
            a[m][4 * v + 1] = u.y;
            a[m][4 * v + 2] = u.z;
            a[m][4 * v + 3] = u.w;
        }
}

// MT tokens' activations of chunk ch from global x̃ [M][K] (tokens past M
// read token M-1; their sums are never stored); idle lanes read zeros.  The
// chunk holding the end of a row when K % 64 != 0 goes through
// load_act_tail, which reads nothing past K.
template <int MT>
__device__ __forceinline__ void ldg_x(const int8_t* xq, int M, int K, int full_chunks, int ch, bool active,
                                      uint32_t (&a)[MT][16]) {
    const bool tail = active && ch >= full_chunks;
    if (__any_sync(0xffffffffu, tail)) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int8_t* row = xq + (int64_t)min(m, M - 1) * K;
            if (tail) {
                uint32_t tmp[16];
                load_act_tail(row, K, ch, tmp);
#pragma unroll
                for (int q = 0; q < 16; ++q) a[m][q] = tmp[q];
            } else {
                const uint8_t* p = active ? reinterpret_cast<const uint8_t*>(row) + 64 * ch
                                          : reinterpret_cast<const uint8_t*>(g_zero_chunk);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 u = ld_shared_ro16(p + 16 * v);
                    a[m][4 * v + 0] = u.x;
                    a[m][4 * v + 1] = u.y;
                    a[m][4 * v + 2] = u.z;
                    a[m][4 * v + 3] = u.w;
                }
            }
        }
        return;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const uint8_t* p = active ? reinterpret_cast<const uint8_t*>(xq + (int64_t)min(m, M - 1) * K) + 64 * ch
                                  : reinterpret_cast<const uint8_t*>(g_zero_chunk);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_shared_ro16(p + 16 * v);
            a[m][4 * v + 0] = u.x;
            a[m][4 * v + 1] = u.y;
            a[m][4 * v + 2] = u.z;
            a[m][4 * v + 3] = u.w;
        }
    }
}

// acc[r][m][q] += codes × x̃ for one step: per (word, field) the RG rows'
// codes are masked first, then their dp4a go to RG independent accumulators.
// With NQ = 4 field q keeps its codes in place (×4^q, summed with a shift at
// the end); with NQ = 1 the codes are shifted down.
template <int RG, int MT, int NQ>
__device__ __forceinline__ void step_math(const uint4 (&w)[RG], const uint32_t (&xa)[MT][16],
                                          int (&acc)[RG][MT][NQ]) {
#pragma unroll
    for (int wj = 0; wj < 4; ++wj) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t codes[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const uint32_t word = word_of(w[r], wj);
                codes[r] = NQ == 4 ? (word & (0x03030303u << (2 * q))) : ((word >> (2 * q)) & 0x03030303u);
            }
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    int& a = acc[r][m][NQ == 4 ? q : 0];
                    a = dp4a_u8s8(codes[r], xa[m][4 * wj + q], a);
                }
        }
    }
}

// MT tokens (M <= MT), W warps per CTA, MINB CTAs per SM, row groups of RG
// rows, CPL chunks per lane, D stages.  A warp walks its range one step at a
// time (up to 32·CPL chunks of one row group).  Each warp has a ring of D
// shared-memory stages (CPL·RG·512 bytes): lane l copies its own 16-byte
// pieces with cp.async and later reads back only those, so the wait is per
// thread and needs no warp barrier.  D-1 steps are in flight while one is
// computed; the first D-1 are requested before the dependency wait.  With
// the fused prologue Σx̃ is not accumulated per step: the warp that holds a
// row group's first chunk subtracts the token's whole-row Σx̃ (summed while
// quantising) once, so every row's total is Σ c·x̃ - Σ x̃ over the full row.
// With x̃ from global memory each lane adds up the Σx̃ of the chunks it
// multiplies and subtracts it from its own partial sums.  FUSE: 0 x̃ from
// global memory, 1 the prologue quantises x, 2 it rotates x, then quantises
// (a separate instance, so the rotation's code does not weigh on the others).
template <int MT, int W, int MINB, int RG, int CPL, int D, int FUSE>
__global__ void __launch_bounds__(W * 32, MINB) gemv_stream_kernel(const __grid_constant__ GParams P) {
    constexpr int NQ = MT <= 2 ? 4 : 1;  // one accumulator per code field (no shifts) for few tokens
    constexpr int V = RG * MT;           // sums per lane when a row group is done
    constexpr uint32_t kStage = CPL * RG * 512;
    static_assert(RG <= kRGMax && V <= 32, "row group too large");
    static_assert(D >= 2, "at least one step in flight");
    using Shared = GShared<W>;
    static_assert(sizeof(Shared) % 16 == 0, "the stages after the shared block need 16-byte alignment");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Shared& S = *reinterpret_cast<Shared*>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the next kernel on the stream may be scheduled now; it waits for this
    // grid before touching memory this grid writes
    griddep_launch_dependents();

    // ---- CTA range (from the host, on row-group edges) and equal warp step ranges
    for (int i = threadIdx.x; i < P.count; i += W * 32) S.prob[i] = P.p[i];
    if (threadIdx.x < 16) reinterpret_cast<uint32_t*>(S.zero)[threadIdx.x] = 0u;
    if (threadIdx.x < kMaxSlots * kGemvMaxTokens) (&S.xsum[0][0])[threadIdx.x] = 0;
    __syncthreads();
    const GProblem* T = S.prob;
    const int count = P.count;
    const int64_t ca = P.cta_begin[blockIdx.x], cb = P.cta_begin[blockIdx.x + 1];
    if (threadIdx.x <= W) S.bound[threadIdx.x] = ca + ((cb - ca) * threadIdx.x) / W;
    __syncthreads();
    const int64_t wu0 = S.bound[warp], wu1 = S.bound[warp + 1];

    // ---- the first D-1 steps' weights do not depend on the previous kernel
    const uint32_t ring = smem_addr(smem_raw + sizeof(Shared)) + (uint32_t)warp * (D * kStage) + 16u * lane;
    int p0 = 0, rg0 = 0, s0 = 0;
    if (wu1 > wu0) locate_step(T, count, wu0, p0, rg0, s0);
    Feed<RG, CPL> fd;
    fd.p = p0;
    fd.rg = rg0;
    fd.s = s0;
    fd.rem = (int)(wu1 - wu0);
    if (fd.rem > 0) {
        fd.fields(T);
        fd.rows(lane);
    }
#pragma unroll
    for (int d = 0; d < D - 1; ++d) {
        if (fd.rem > 0) {
            fd.request(ring + d * kStage, lane);
            fd.advance(T, lane);
        }
        cp_async_commit();
    }
    // ---- fused quantisation: x̃ of the (at most two) problems of this CTA;
    // the rows are set up before the dependency wait (they need only the table)
    int p_first = 0;
    int second_slot = 1;  // slot of the CTA's second problem (0 when it shares the first one's input)
    uint32_t xs_base = 0;
    // rows[slot·MT + m]: token m of the slot's problem (static indices keep them in registers)
    QRow rows[FUSE ? kMaxSlots * MT : 1];
    if constexpr (FUSE) {
        xs_base = smem_addr(smem_raw + sizeof(Shared) + W * D * kStage);
        p_first = problem_of_step(T, count, ca);
        const int p_last = cb > ca ? problem_of_step(T, count, cb - 1) : p_first;
#pragma unroll
        for (int slot = 0; slot < kMaxSlots; ++slot) {
            const int p = p_first + slot;
            bool use = ca < cb && p <= p_last;
            bool owner = false;
            if (use) {
                const GProblem& pr = T[p];
                owner = ca <= pr.step_begin && pr.step_begin < cb;
                if (slot == 1) {
                    const GProblem& p0 = T[p_first];
                    if (pr.x == p0.x && pr.x2 == p0.x2 && pr.K == p0.K && pr.M == p0.M) {
                        // same input as slot 0: reuse it (the owner still publishes x̃, β)
                        second_slot = 0;
                        if (owner && pr.write_outputs && (pr.xq != p0.xq || pr.beta != p0.beta || pr.x_sum != p0.x_sum))
                            second_slot = 1;  // distinct output buffers: quantise again to write them
                        use = second_slot == 1;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                QRow& r = rows[slot * MT + m];
                r.valid = false;
                if (use) {
                    const GProblem& pr = T[p];
                    r.valid = m < pr.M;
                    r.x = pr.x;
                    r.x2 = pr.x2;
                    r.xq = const_cast<int8_t*>(pr.xq);
                    r.beta = const_cast<float*>(pr.beta);
                    r.x_sum = pr.x_sum;
                    r.dst = xs_base + (uint32_t)((slot * MT + m) * P.slot_row);
                    r.slot = slot;
                    r.m = m;
                    r.K = pr.K;
                    r.had = pr.had_block;
                    r.out = owner && pr.write_outputs != 0;
                }
            }
        }
    }
    griddep_wait();  // x̃, β (and α) may come from the preceding kernels
    if constexpr (FUSE) {
#pragma unroll
        for (int i = 0; i < kMaxSlots * MT; i += kFuseRows) {
            const QRow(&pair)[kFuseRows] = *reinterpret_cast<const QRow(*)[kFuseRows]>(&rows[i]);
            if constexpr (FUSE == 2) {  // rotated rows one at a time through the scratch
                const RotScratch sc{smem_addr(smem_raw + sizeof(Shared)) + (uint32_t)((D - 1) * kStage),
                                    (uint32_t)(D * kStage), ilog2_const(kStage / 4)};
#pragma unroll
                for (int e = 0; e < kFuseRows; ++e) {
                    if (!pair[e].valid) continue;  // the same in every thread of the CTA
                    if (P.x_bf16)
                        fused_rotate_quantize_row<uint16_t, W * 32>(pair[e], sc, P.slot_row, S.red, S.xbeta, S.xsum,
                                                                    P.a4 != 0);
                    else
                        fused_rotate_quantize_row<float, W * 32>(pair[e], sc, P.slot_row, S.red, S.xbeta, S.xsum,
                                                                 P.a4 != 0);
                }
            } else if (pair[0].valid || pair[1].valid) {  // the same in every thread of the CTA
                if (P.x_bf16)
                    fused_quantize_rows<uint16_t, W * 32>(pair, P.slot_row, S.red, S.xbeta, S.xsum, P.a4 != 0);
                else
                    fused_quantize_rows<float, W * 32>(pair, P.slot_row, S.red, S.xbeta, S.xsum, P.a4 != 0);
            }
        }
        __syncthreads();
    }
    const uint32_t zero_addr = smem_addr(S.zero);

    // ---- state of the problem of the current step
    int sp = -1;                          // that problem
    float alpha_v = 0.0f, beta_v = 0.0f;  // lane m < MT: α and token m's β
    int sx[MT];  // fused: Σx̃ of each token over the whole row; else this lane's part of the row group's
    uint32_t xrow = 0;                    // fused: shared address of the problem's slot
    const int8_t* xq = nullptr;           // unfused: the problem's x̃ and its shape
    int xM = 1, xK = 0, xfull = 0;
    int cC = 0, cS = 1, crgn = 1;  // the problem's chunks per row, steps per row group, row groups
    int scale_p = -1;       // problem of my_scale
    float my_scale = 0.0f;  // lane m < MT: dequant scale of token m
#pragma unroll
    for (int m = 0; m < MT; ++m) sx[m] = 0;

    int acc[RG][MT][NQ];
    bool fresh = true;           // the next step begins a row group for this warp
    bool rg_own = false;         // this warp holds the current row group's first chunk
    int own_p = -1, own_rg = 0;  // a shared row group this warp finishes after the loop
    uint32_t stage = ring;       // the current step's stage
    uint32_t fill = ring + (D - 1) * kStage;  // the stage the next request goes to
    int cp = p0, crg = rg0, cs = s0;          // the current step
    int crem = (int)(wu1 - wu0);              // steps left, the current one included

    while (crem > 0) {
        if (cp != sp) {  // entering a problem: its α, β, Σx̃, activations and shape
            sp = cp;
            const GProblem& pr = T[sp];
            alpha_v = pr.alpha_rows ? 0.0f : *pr.alpha;
            cC = pr.C;
            cS = pr.S;
            crgn = pr.rgn;
            if constexpr (FUSE) {
                const int slot = sp == p_first ? 0 : second_slot;
                xrow = xs_base + (uint32_t)(slot * MT) * (uint32_t)P.slot_row;
                if (lane < MT) beta_v = S.xbeta[slot][lane];
#pragma unroll
                for (int m = 0; m < MT; ++m) sx[m] = S.xsum[slot][m];
            } else {
                xq = pr.xq;
                xM = pr.M;
                xK = pr.K;
                xfull = pr.full_chunks;
                if (lane < MT && lane < pr.M) beta_v = pr.beta[lane];
            }
        }
        if (fresh) {
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int q = 0; q < NQ; ++q) acc[r][m][q] = 0;
            rg_own = cs == 0;
            fresh = false;
            if constexpr (!FUSE) {
#pragma unroll
                for (int m = 0; m < MT; ++m) sx[m] = 0;
            }
        }
        // request the step D-1 ahead into the stage freed by the previous step
        if (fd.rem > 0) {
            fd.request(fill, lane);
            fd.advance(T, lane);
        }
        cp_async_commit();
        cp_async_wait<D - 1>();  // this lane's copies of the current step have landed
        const int nc = min(32 * CPL, cC - 32 * CPL * cs);  // chunks of this step
#pragma unroll 1
        for (int j = 0; j < CPL; ++j) {  // not unrolled: one copy of the arithmetic keeps the loop in the instruction cache
            uint4 w[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) w[r] = lds128_after(stage + 512u * (j * RG + r));
            const bool active = 32 * j + lane < nc;
            const int ch = 32 * CPL * cs + 32 * j + lane;
            uint32_t xa[MT][16];
            if constexpr (FUSE)
                lds_x<MT>(xrow, P.slot_row, ch, active, zero_addr, xa);
            else
                ldg_x<MT>(xq, xM, xK, xfull, ch, active, xa);
            step_math<RG, MT, NQ>(w, xa, acc);
            if constexpr (!FUSE) {  // this lane's Σx̃ over the chunks it added
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int q = 0; q < 16; ++q) sx[m] = dp4a_s8s8(0x01010101u, xa[m][q], sx[m]);
            }
        }

        const bool rg_end = cs + 1 == cS;
        if (rg_end || crem == 1) {
            // this warp's sums of the row group.  Fused: the holder of its
            // first chunk takes the row's Σx̃ off (in one lane, so once);
            // otherwise every lane takes off the Σx̃ of the chunks it added.
            const bool sub = FUSE ? (lane == 0 && rg_own) : true;
            int v[V];
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    int t = acc[r][m][0];
                    if constexpr (NQ == 4) t += (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) + (acc[r][m][3] >> 6);
                    v[m * RG + r] = t - (sub ? sx[m] : 0);
                }
            int idx;
            const int val = reduce_scatter<V>(v, lane, idx);
            const bool writer = (lane & (32 / V - 1)) == 0;
            const int r = idx % RG, m = idx / RG;
            if (rg_own && rg_end) {  // the whole row group: write y
                if (scale_p != sp) {
                    scale_p = sp;
                    my_scale = token_scale(T[sp].alpha_rows, P.a4, alpha_v, beta_v);
                }
                const float sc = __shfl_sync(0xffffffffu, my_scale, m);
                const GProblem& pr = T[sp];
                const int row = crg * RG + r;
                if (writer && row < pr.N && m < pr.M) {
                    float out = pr.alpha_rows ? __fmul_rn(__fmul_rn((float)val, pr.alpha[row]), sc)
                                              : __fmul_rn((float)val, sc);
                    if (pr.bias) out = __fadd_rn(out, pr.bias[row]);
                    pr.y[(int64_t)m * pr.N + row] = out;
                    if (pr.acc_out) pr.acc_out[(int64_t)m * pr.N + row] = val;
                }
            } else {
                // a row group shared with the neighbouring warps: keep this
                // warp's part; the holder of its first chunk adds the parts up
                // after the main loop
                if (writer) S.part[warp][rg_own ? 1 : 0][idx] = val;
                if (rg_own) {
                    own_p = sp;
                    own_rg = crg;
                }
            }
            fresh = true;
        }
        // the next step
        --crem;
        if (++cs == cS) {
            cs = 0;
            if (++crg == crgn) {
                crg = 0;
                ++cp;
            }
        }
        fill = stage;
        stage = stage + kStage == ring + D * kStage ? ring : stage + kStage;
    }
    cp_async_wait<0>();

    // ---- row groups shared between warps: the warp holding the first chunk
    // adds the parts of the warps after it that worked on the same row group
    __syncthreads();
    if (own_p >= 0) {
        const GProblem& pr = T[own_p];
        const int64_t rg_end = pr.step_begin + (int64_t)(own_rg + 1) * pr.S;
        int idx = 0;
#pragma unroll
        for (int half = V / 2, off = 16; half >= 1; half >>= 1, off >>= 1)
            if (lane & off) idx += half;
        const bool writer = (lane & (32 / V - 1)) == 0;
        int val = writer ? S.part[warp][1][idx] : 0;
        for (int w2 = warp + 1; w2 < W && S.bound[w2] < rg_end; ++w2)
            if (writer && S.bound[w2 + 1] > S.bound[w2]) val += S.part[w2][0][idx];  // skip empty ranges
        if (scale_p != own_p) my_scale = token_scale(pr.alpha_rows, P.a4, alpha_v, beta_v);
        const int r = idx % RG, m = idx / RG;
        const float sc = __shfl_sync(0xffffffffu, my_scale, m);
        const int row = own_rg * RG + r;
        if (writer && row < pr.N && m < pr.M) {
            float out = pr.alpha_rows ? __fmul_rn(__fmul_rn((float)val, pr.alpha[row]), sc)
                                      : __fmul_rn((float)val, sc);
            if (pr.bias) out = __fadd_rn(out, pr.bias[row]);
            pr.y[(int64_t)m * pr.N + row] = out;
            if (pr.acc_out) pr.acc_out[(int64_t)m * pr.N + row] = val;
        }
    }
}

// ---------------------------------------------------------------- any K, any alignment
// One warp per output element, byte loads.
struct GenericProblem {
    const int8_t* xq;
    const float* beta;
    const uint32_t* W;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int64_t M, N, K, row_words, task_begin;
};
struct GenericParams {
    GenericProblem p[kMaxGroup];
    int count;
    int64_t total_tasks;
};

__global__ void __launch_bounds__(256) gemv_generic_kernel(const __grid_constant__ GenericParams P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * 256 + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * 256) >> 5;
    for (int64_t t = warp0; t < P.total_tasks; t += nwarps) {
        int pi = 0;
        while (pi + 1 < P.count && t >= P.p[pi + 1].task_begin) ++pi;
        const GenericProblem& pr = P.p[pi];
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

// Waits on an mbarrier that nothing ever completes, with a caller-chosen
// bound, to exercise the timeout path (sets the device error, then returns).
__global__ void wait_timeout_selftest_kernel(uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    __syncthreads();
    bool ok = false;
    for (uint32_t i = 0; i < polls && !ok; ++i) ok = mbar_try_wait(smem_addr(&bar), 0, 1000);
    if (!ok && threadIdx.x == 0) atomicCAS(&g_device_error, 0, (int)BL_ERR_TIMEOUT);
}

// ---------------------------------------------------------------- launch
// Shape of the streaming kernel for MT tokens: warps per CTA, CTAs per SM.
template <int MT>
struct StreamCfg;
template <>
struct StreamCfg<1> {
    static constexpr int W = 12, MINB = 1, RG = 8, CPL = 2, D = 2;
};
template <>
struct StreamCfg<2> {
    static constexpr int W = 12, MINB = 1, RG = 8, CPL = 1, D = 3;
};
template <>
struct StreamCfg<4> {
    static constexpr int W = 8, MINB = 1, RG = 4, CPL = 1, D = 4;
};

constexpr size_t kSmemOptIn = 232448;  // opt-in dynamic shared memory per block on sm_100

void fill_params(GParams& P, const bitlinear_forward_problem* problems, int count, int RG, int CPL,
                 bool alpha_rows = false) {
    P = GParams{};
    P.count = count;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        GProblem& q = P.p[i];
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
        q.full_chunks = q.K / 64;
        q.rgn = (q.N + RG - 1) / RG;
        q.alpha_rows = alpha_rows ? 1 : 0;
        q.S = (q.C + 32 * CPL - 1) / (32 * CPL);
        q.step_begin = total;
        total += (int64_t)q.rgn * q.S;
    }
    P.total_steps = total;
}

// Prologue cost of quantising one input row of K elements in a CTA of W
// warps, in warp-steps (the time one warp takes for one step of CPL chunks
// per lane): measured on B200 with 12 warps and one chunk per lane as about
// 1.27 + K / 4930 step times.
inline double prologue_cost(int W, int CPL, int64_t K) { return W * (1.27 + (double)K / 4930.0) / CPL; }

// Splits the steps of P into at most G contiguous CTA ranges of whole row
// groups whose costs (their steps, plus, with `pro`, the prologue cost of
// each distinct input they quantise) are as even as a greedy fill allows:
// the smallest cost bound T for which the fill needs at most G CTAs is found
// by bisection.  Writes P.cta_begin[0..n] and returns n (the CTAs to launch).
int cta_ranges(GParams& P, int G, const double* pro) {
    const int count = P.count;
    auto same_input = [&](int a, int b) {
        return P.p[a].x == P.p[b].x && P.p[a].x2 == P.p[b].x2 && P.p[a].K == P.p[b].K && P.p[a].M == P.p[b].M;
    };
    auto fill = [&](double T, bool write) {
        int c = 0;
        double cost = 0.0;
        int64_t pos = 0;
        int last = -1;  // the last problem the current CTA took
        if (write) P.cta_begin[0] = 0;
        for (int p = 0; p < count; ++p) {
            const GProblem& q = P.p[p];
            int64_t left = q.rgn;
            while (left > 0) {
                const double pc = (!pro || last == p || (last >= 0 && same_input(p, last))) ? 0.0 : pro[p];
                const double room = T - cost - pc;
                int64_t k = room >= q.S ? (int64_t)(room / q.S) : 0;
                if (k == 0) {
                    if (cost == 0.0) {
                        k = 1;  // an empty CTA takes one row group even above T
                    } else {
                        ++c;
                        if (write && c <= kMaxCta) P.cta_begin[c] = (int32_t)pos;
                        cost = 0.0;
                        last = -1;
                        continue;
                    }
                }
                if (k > left) k = left;
                cost += pc + (double)k * q.S;
                last = p;
                pos += k * q.S;
                left -= k;
            }
        }
        if (write && c + 1 <= kMaxCta) P.cta_begin[c + 1] = (int32_t)pos;
        return c + 1;
    };
    double lo = 0.0, hi = 0.0;
    for (int p = 0; p < count; ++p) hi += (double)P.p[p].rgn * P.p[p].S + (pro ? pro[p] : 0.0);
    hi += 1.0;
    for (int it = 0; it < 40 && hi - lo > 0.5; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (fill(mid, false) <= G)
            hi = mid;
        else
            lo = mid;
    }
    return fill(hi, true);
}

// cta_ranges for a call whose shapes match a recent call's: the split
// depends only on G, the problems' row-group counts, steps per row group,
// prologue costs and which neighbours share an input, so it is looked up
// (the bisection costs several microseconds of host time per call).
int cta_ranges_cached(GParams& P, int G, const double* pro) {
    struct Key {
        int G, count, fused;
        uint64_t same;  // bit p: problem p has the input of problem p-1
        int32_t rgn[kMaxGroup], S[kMaxGroup];
        double pro[kMaxGroup];
    };
    struct Entry {
        Key key;
        int grid;
        int32_t begin[kMaxCta + 1];
    };
    constexpr int kEntries = 8;
    static std::mutex mu;
    static Entry cache[kEntries];
    static int used = 0, next = 0;
    Key k;
    std::memset(&k, 0, sizeof(k));
    k.G = G;
    k.count = P.count;
    k.fused = pro ? 1 : 0;
    for (int p = 0; p < P.count; ++p) {
        k.rgn[p] = P.p[p].rgn;
        k.S[p] = P.p[p].S;
        k.pro[p] = pro ? pro[p] : 0.0;
        if (p > 0 && P.p[p].x == P.p[p - 1].x && P.p[p].x2 == P.p[p - 1].x2 && P.p[p].K == P.p[p - 1].K &&
            P.p[p].M == P.p[p - 1].M)
            k.same |= (uint64_t)1 << p;
    }
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int e = 0; e < used; ++e)
            if (std::memcmp(&cache[e].key, &k, sizeof(Key)) == 0) {
                std::memcpy(P.cta_begin, cache[e].begin, sizeof(int32_t) * (cache[e].grid + 1));
                return cache[e].grid;
            }
    }
    const int grid = cta_ranges(P, G, pro);
    std::lock_guard<std::mutex> lock(mu);
    Entry& e = cache[next];
    next = (next + 1) % kEntries;
    if (used < kEntries) ++used;
    e.key = k;
    e.grid = grid;
    std::memcpy(e.begin, P.cta_begin, sizeof(int32_t) * (grid + 1));
    return grid;
}

// Launches gemv_stream_kernel<MT, W, MINB, RG, CPL, D, fused>; with `fused` (one entry per
// problem) the kernel quantises x itself, if every CTA's range meets at most
// two problems, the slots fit shared memory and the CTAs' input reads stay
// small next to the weights (else *launched = false and nothing runs).
template <int MT, int W, int MINB, int RG, int CPL, int D>
cudaError_t launch_stream_cfg(const bitlinear_forward_problem* problems, int count, const DeviceInfo& dev,
                              cudaStream_t stream, bool pdl, const FusedInput* fused, bool x_bf16, bool* launched,
                              bool fuse_always, bool alpha_rows = false, bool a4 = false) {
    using Shared = GShared<W>;
    if (launched) *launched = true;
    if (a4 && !fused) return cudaErrorInvalidValue;  // 4-bit activations only with the fused prologue
    GParams P;
    fill_params(P, problems, count, RG, CPL, alpha_rows);
    int64_t weight_bytes = 0;
    for (int i = 0; i < count; ++i) weight_bytes += (int64_t)P.p[i].N * P.p[i].row_bytes;
    if (P.total_steps >= INT32_MAX) return cudaErrorInvalidValue;  // over 8 TB of weights in one call
    const int G = (int)std::min<int64_t>((int64_t)dev.sm_count * MINB, kMaxCta);
    int grid = 0;
    size_t smem = sizeof(Shared) + (size_t)W * D * CPL * RG * 512;  // the table, then the warps' stage rings
    const size_t smem_cap = kSmemOptIn / MINB - (MINB > 1 ? 1024 : 0);
    if (fused) {
        int32_t slot_row = 0;
        for (int i = 0; i < count; ++i) {
            GProblem& q = P.p[i];
            q.x = fused[i].x;
            q.x2 = fused[i].x2;
            q.x_sum = fused[i].x_sum;
            q.write_outputs = fused[i].write_outputs ? 1 : 0;
            q.had_block = fused[i].had_block;
            slot_row = std::max(slot_row, 64 * q.C);
        }
        P.x_bf16 = x_bf16 ? 1 : 0;
        P.a4 = a4 ? 1 : 0;
        P.had = fused[0].had_block > 0 ? 1 : 0;
        P.slot_row = slot_row;
        bool fits = smem + (size_t)kMaxSlots * MT * slot_row <= smem_cap;
        for (int i = 0; i < count; ++i) {
            // all problems rotated or none; a rotated row fits the scratch in the
            // last stage of every warp's ring, which nothing fills before the loop
            fits = fits && (fused[i].had_block > 0) == (P.had != 0);
            if (P.had)  // (built for one token; blocks of at least 8 dividing K)
                fits = fits && MT == 1 && D >= 2 && fused[i].had_block >= 8 &&
                       (fused[i].had_block & (fused[i].had_block - 1)) == 0 && P.p[i].K % fused[i].had_block == 0 && (int64_t)P.p[i].K <= (int64_t)W * (CPL * RG * 512 / 4) && !fused[i].x2 &&
                       !fused[i].x_sum;
        }
        // the prologue holds a row in registers: at most W·32·kFuseVec 16-byte vectors
        for (int i = 0; i < count; ++i)
            fits = fits && (int64_t)P.p[i].K * (x_bf16 ? 2 : 4) <= (int64_t)W * 32 * kFuseVec * 16;
        double pro[kMaxGroup];
        for (int i = 0; i < count; ++i)  // a rotation about doubles the prologue
            pro[i] = prologue_cost(W, CPL, P.p[i].K) * std::min<int>(P.p[i].M, MT) * (P.had ? 2 : 1);
        grid = cta_ranges_cached(P, G, pro);
        // Every CTA reads its problems' whole input rows before its main loop;
        // that pays off only while those reads are small next to the weights.
        auto input_bytes = [&](const GProblem& q) {
            return (int64_t)q.M * q.K * (x_bf16 ? 2 : 4) * (q.x2 ? 2 : 1);
        };
        int64_t prologue_bytes = 0;
        for (int c = 0; c < grid && fits; ++c) {
            const int64_t a = P.cta_begin[c], b = P.cta_begin[c + 1];
            if (a >= b) continue;
            const int pa = problem_of_step(P.p, count, a), pb = problem_of_step(P.p, count, b - 1);
            fits = pb - pa <= 1;
            prologue_bytes += input_bytes(P.p[pa]);
            if (pb != pa && !(P.p[pb].x == P.p[pa].x && P.p[pb].x2 == P.p[pa].x2)) prologue_bytes += input_bytes(P.p[pb]);
        }
        if (!fuse_always && 2 * prologue_bytes > weight_bytes) fits = false;
        if (!fits) {
            *launched = false;
            return cudaSuccess;
        }
        smem += (size_t)kMaxSlots * MT * slot_row;
    } else {
        grid = cta_ranges_cached(P, G, nullptr);
    }
    if (smem > smem_cap) return cudaErrorInvalidConfiguration;  // a shape that does not fit (not built)
    const void* kernel = fused ? reinterpret_cast<const void*>(gemv_stream_kernel<MT, W, MINB, RG, CPL, D, 1>)
                               : reinterpret_cast<const void*>(gemv_stream_kernel<MT, W, MINB, RG, CPL, D, 0>);
    if constexpr (MT == 1)
        if (fused && P.had) kernel = reinterpret_cast<const void*>(gemv_stream_kernel<MT, W, MINB, RG, CPL, D, 2>);
    // the opt-in is per device: set once on each device that launches the kernel
    cudaError_t err = set_max_dynamic_smem(kernel, (int)smem_cap);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(W * 32);
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

template <int MT>
cudaError_t launch_stream(const bitlinear_forward_problem* problems, int count, const DeviceInfo& dev,
                          cudaStream_t stream, bool pdl, const FusedInput* fused = nullptr, bool x_bf16 = false,
                          bool* launched = nullptr, bool fuse_always = false, bool alpha_rows = false,
                          bool a4 = false) {
    using C = StreamCfg<MT>;
    return launch_stream_cfg<MT, C::W, C::MINB, C::RG, C::CPL, C::D>(problems, count, dev, stream, pdl, fused, x_bf16,
                                                                     launched, fuse_always, alpha_rows, a4);
}

cudaError_t launch_generic(const bitlinear_forward_problem* problems, int count, const DeviceInfo& dev,
                           cudaStream_t stream) {
    GenericParams P{};
    P.count = count;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        GenericProblem& q = P.p[i];
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
        q.task_begin = total;
        total += s.M * s.N;
    }
    P.total_tasks = total;
    int64_t blocks = (total + 7) / 8;
    const int64_t cap = (int64_t)dev.sm_count * 8;
    if (blocks > cap) blocks = cap;
    gemv_generic_kernel<<<(unsigned)blocks, 256, 0, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace

// Three or four tokens on large weights: the tensor-core GEMM (x̃ quantised by
// its own launch) is faster than the streaming GEMV, whose dp4a work grows
// with the token count (100B-shaped matrices at four tokens: 33 against 46 µs).
constexpr int64_t kGemmFewTokenMinBytes = 8 << 20;

bool prefer_gemm_few_tokens(const bitlinear_forward_problem* problems, int count, int64_t max_m) {
    if (max_m < 3 || max_m > kGemvMaxTokens) return false;
    int64_t bytes = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        if (s.K % 16 != 0 || (reinterpret_cast<uintptr_t>(s.x_q) & 15) != 0 || !gemm_tc_supported(s)) return false;
        bytes += s.N * (int64_t)bitlinear_packed_row_bytes(s.K);
    }
    return bytes >= kGemmFewTokenMinBytes;
}

cudaError_t launch_forward(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl,
                           bool alpha_rows) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    bool fast = true;
    int64_t max_m = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        fast = fast && (s.K % 16 == 0) && ((reinterpret_cast<uintptr_t>(s.x_q) & 15) == 0);
        if (s.M > max_m) max_m = s.M;
    }
    if (alpha_rows) {  // per-row α: the streaming GEMV only (the caller checked shape and alignment)
        if (max_m == 1) return launch_stream<1>(problems, count, dev, stream, pdl, nullptr, false, nullptr, false, true);
        if (max_m == 2) return launch_stream<2>(problems, count, dev, stream, pdl, nullptr, false, nullptr, false, true);
        return launch_stream<4>(problems, count, dev, stream, pdl, nullptr, false, nullptr, false, true);
    }
    if (max_m > kGemvMaxTokens || (!alpha_rows && prefer_gemm_few_tokens(problems, count, max_m))) {
        // many tokens: the int8 tensor cores, all problems in one launch
        bool tc = fast;
        for (int i = 0; i < count; ++i) tc = tc && gemm_tc_supported(problems[i]);
        if (tc) return launch_gemm_tc(problems, count, stream, pdl);
        return launch_generic(problems, count, dev, stream);
    }
    if (!fast) return launch_generic(problems, count, dev, stream);
    if (max_m == 1) return launch_stream<1>(problems, count, dev, stream, pdl);
    if (max_m == 2) return launch_stream<2>(problems, count, dev, stream, pdl);
    return launch_stream<4>(problems, count, dev, stream, pdl);
}

cudaError_t launch_linear_fused(const bitlinear_forward_problem* problems, const FusedInput* in, int count,
                                bitlinear_dtype dtype, cudaStream_t stream, bool pdl, bool* launched,
                                bool alpha_rows, bool a4) {
    *launched = false;
    // BITLINEAR_LINEAR_FUSION=off never fuses, =on fuses whenever the
    // problems fit the kernel (skipping the byte-ratio rule); default: auto
    const char* mode = std::getenv("BITLINEAR_LINEAR_FUSION");
    if (mode && std::strcmp(mode, "off") == 0) return cudaSuccess;
    const bool always = mode && std::strcmp(mode, "on") == 0;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    int64_t max_m = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        if (s.K % 16 != 0 || (reinterpret_cast<uintptr_t>(s.x_q) & 15) != 0) return cudaSuccess;
        // the fused prologue reads x (and x2) and writes x_sum in 16-byte vectors
        if ((reinterpret_cast<uintptr_t>(in[i].x) & 15) != 0 || (reinterpret_cast<uintptr_t>(in[i].x2) & 15) != 0 ||
            (reinterpret_cast<uintptr_t>(in[i].x_sum) & 15) != 0)
            return cudaSuccess;
        if (s.M > max_m) max_m = s.M;
    }
    // three or four tokens on large weights: act quant + tensor-core GEMM instead
    if (!always && !alpha_rows && !a4 && prefer_gemm_few_tokens(problems, count, max_m)) return cudaSuccess;
    const bool bf16 = dtype == BL_BF16;
    if (max_m == 1)
        return launch_stream<1>(problems, count, dev, stream, pdl, in, bf16, launched, always, alpha_rows, a4);
    if (max_m == 2)
        return launch_stream<2>(problems, count, dev, stream, pdl, in, bf16, launched, always, alpha_rows, a4);
    if (max_m <= 4)
        return launch_stream<4>(problems, count, dev, stream, pdl, in, bf16, launched, always, alpha_rows, a4);
    return cudaSuccess;
}

cudaError_t read_device_error(int* code) {
    int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(code, g_device_error, sizeof(int));
    if (err != cudaSuccess) return err;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

cudaError_t launch_wait_timeout_selftest(uint32_t polls, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(polls);
    return cudaGetLastError();
}

}  // namespace bl
