// Ternary GEMV / skinny GEMM on CUDA cores: y = (x̃·Ŵᵀ)·(α·β/127) + bias.
//
// The product is the pages' add / subtract / skip ("1.58 位大模型",
// nxmr.cn/news/148658 §3.3): Y[m][n] = Σ_{W=+1} x̃ - Σ_{W=-1} x̃.  It is
// evaluated as Σ c·x̃ - Σ x̃ with the stored code c = w + 1 ∈ {0, 1, 2}: one
// mask of a packed word yields four codes as unsigned bytes (×4^s), and one
// dp4a adds their products with four int8 activations, so a zero weight costs
// nothing extra and ±1 weights become adds and subtracts.  Dequantisation and
// bias follow "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.4–§2.5
// and §4.2.
//
// Decode is bound by the HBM bytes of the packed weights ("1.58-bit 大模型极限
// 量化实战" §5.1–§5.2; 2kiu.com/news/4928193 §3.1, §3.3), so the kernel is built
// to keep HBM streaming while the arithmetic runs:
//  * persistent grid, one CTA per SM; the work (row groups of 8 rows × 16-byte
//    chunks, over every problem of a grouped launch) is cut into contiguous
//    ranges of equal chunk count, snapped to row-group boundaries;
//  * inside a CTA the range is split evenly over 8 warps at chunk
//    granularity; a row group shared by several warps is summed exactly in
//    shared memory (int32 atomics) and finished by its last contributor;
//  * each warp streams its own segments (8 rows × up to 64 chunks) into two
//    private shared-memory stages with 1-D bulk copies (TMA), the rows issued
//    by eight lanes at once; a waiting warp sleeps in the mbarrier (bounded);
//  * everything a segment needs from global memory besides its weights (the
//    activations, α, β) is requested before the warp waits for the weights,
//    so those latencies overlap the copy;
//  * lanes read staged rows with conflict-free 16-byte shared loads, the
//    activations serve all 8 rows, and a reduce-scatter of shuffles leaves
//    each row's sum in one lane.
// The weight stream does not depend on the previous kernel, so it starts
// before griddepcontrol.wait (programmatic dependent launch).
//
// Fused mode (at most four tokens, chosen by the host): the kernel also does
// the per-token activation quantisation.  Right after its dependency wait each
// CTA quantises the input rows of the (at most two) problems its range covers
// into shared-memory slots with the same arithmetic as the activation kernel,
// and the main loop reads x̃ and β from there; the CTA owning a problem's first
// unit writes x̃ and β (and a residual sum) out.  One launch then replaces the
// quantisation kernel and the product kernel.

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {

// Set (first error wins) by a kernel whose bounded wait expired; read and
// cleared by bitlinear_device_error().
static __device__ int g_device_error;

namespace {

#ifndef BL_GEMV_WARPS
#define BL_GEMV_WARPS 8
#endif
#ifndef BL_GEMV_STAGES
#define BL_GEMV_STAGES 2
#endif
constexpr int kWarps = BL_GEMV_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = BL_GEMV_STAGES;         // private stages per warp
constexpr int kRG = 8;                          // rows per row group
// CTAs per SM the streaming kernel is compiled for: 2 lets the next launch's
// CTAs start streaming weights beside the current ones (needs small stages)
#ifndef BL_GEMV_MIN_BLOCKS
#define BL_GEMV_MIN_BLOCKS 1
#endif
#ifndef BL_GEMV_SEG_CHUNKS
#define BL_GEMV_SEG_CHUNKS 64
#endif
constexpr int kSegChunks = BL_GEMV_SEG_CHUNKS;  // 16-byte chunks per row per segment (multiple of 32)
constexpr int kIt = kSegChunks / 32;            // chunks per lane per row per segment
constexpr int kRowStride = kSegChunks * 16;     // bytes per staged row
constexpr int kStageBytes = kRG * kRowStride;   // 8 KiB at 64 chunks
static_assert(kSegChunks % 32 == 0, "whole chunks per lane");
constexpr int kSlots = kWarps;                  // row groups shared between warps
constexpr int kMaxMT = 4;
constexpr int kGemvMaxTokens = 4;  // more tokens go to the tensor-core GEMM

struct SProblem {
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
    int32_t rgn;          // row groups of kRG rows
    int32_t tgn;          // token groups of MT tokens
    int64_t unit_begin;   // first unit (token group, row group, chunk) of this problem
    // fused quantisation (x̃ made in shared memory from x, see below):
    const void* x;        // activations, float32 or bfloat16 [M][K]
    const float* x2;      // nullable float32 second addend
    float* x_sum;         // nullable: stores x (+ x2)
    int32_t write_outputs;  // the owner CTA writes x̃ to xq and β to beta (and x_sum)
};

struct SParams {
    SProblem p[kMaxGroup];
    int count;
    int64_t total_units;
    int x_bf16;         // fused: activation dtype
    int32_t slot_row;   // fused: bytes per token row of a shared x̃ slot (64·ceil(K/64) of the widest problem)
};

// Fused quantisation keeps two problems' x̃ (up to kMaxMT token rows each) in
// shared memory after SharedLayout.
constexpr int kFuseSlotBytes = 45056;

struct SharedLayout {
    alignas(128) uint8_t stage[kWarps][kStages][kStageBytes];
    alignas(8) uint64_t full[kWarps][kStages];
    int64_t bound[kWarps + 1];  // warp unit ranges inside the CTA
    int slot_acc[kSlots][kRG * kMaxMT];
    int slot_count[kSlots];
    SProblem prob[kMaxGroup];  // copy of the problem table (indexed reads of it are cheap here)
    float xbeta[2][kMaxMT];  // fused: β of each slot's tokens
    float red[kWarps];       // fused: block reduction scratch
};

// The problem table as the kernel reads it after copying it to shared memory.
struct ProbTable {
    const SProblem* p;
    int count;
};

// Position in the unit sequence: problem, (token group, row group), chunk.
struct Cursor {
    int p;
    int tgrg;
    int c;
    int64_t u, end;
};

template <typename Tab>
__device__ __forceinline__ void cursor_seek(const Tab& P, Cursor& cur, int64_t u, int64_t end) {
    int p = 0;
    while (p + 1 < P.count && u >= P.p[p + 1].unit_begin) ++p;
    const int64_t local = u - P.p[p].unit_begin;
    cur.p = p;
    cur.tgrg = (int)(local / P.p[p].C);
    cur.c = (int)(local - (int64_t)cur.tgrg * P.p[p].C);
    cur.u = u;
    cur.end = end;
}

// Length (chunks) of the segment starting at the cursor.
template <typename Tab>
__device__ __forceinline__ int cursor_len(const Tab& P, const Cursor& cur) {
    int64_t n = P.p[cur.p].C - cur.c;
    if (n > kSegChunks) n = kSegChunks;
    if (n > cur.end - cur.u) n = (int)(cur.end - cur.u);
    return (int)n;
}

template <typename Tab>
__device__ __forceinline__ void cursor_advance(const Tab& P, Cursor& cur, int n) {
    cur.u += n;
    cur.c += n;
    if (cur.c == P.p[cur.p].C) {
        cur.c = 0;
        if (++cur.tgrg == P.p[cur.p].tgn * P.p[cur.p].rgn) {
            cur.tgrg = 0;
            ++cur.p;
        }
    }
}

// Start of the row group containing unit t, rounded to the nearer boundary.
__host__ __device__ int64_t snap_to_row_group(const SParams& P, int64_t t) {
    if (t >= P.total_units) return P.total_units;
    int p = 0;
    while (p + 1 < P.count && t >= P.p[p + 1].unit_begin) ++p;
    const int64_t local = t - P.p[p].unit_begin;
    int64_t g = local / P.p[p].C;
    if (2 * (local - g * P.p[p].C) >= P.p[p].C) ++g;
    return P.p[p].unit_begin + g * P.p[p].C;
}

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

__device__ __forceinline__ void load_act_chunk(const int8_t* xrow, int K, int chunk, bool full, bool valid,
                                               uint32_t (&a)[16]) {
    if (valid && full) {
        const int8_t* p = xrow + 64 * chunk;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = ld_shared_ro16(p + 16 * v);
            a[4 * v + 0] = u.x;
            a[4 * v + 1] = u.y;
            a[4 * v + 2] = u.z;
            a[4 * v + 3] = u.w;
        }
    } else if (valid) {
        uint32_t tmp[16];  // only this rare path goes through local memory
        load_act_tail(xrow, K, chunk, tmp);
#pragma unroll
        for (int q = 0; q < 16; ++q) a[q] = tmp[q];
    } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) a[q] = 0u;
    }
}

// Shared x̃ slot layout: the four 16-byte pieces of 64-byte chunk c are
// rotated by (c >> 1), so the 16-byte reads of 8 lanes on consecutive chunks
// fall in distinct banks.
__device__ __forceinline__ uint32_t xs_offset(int k) {
    const int c = k >> 6, v = (k >> 4) & 3;
    return (uint32_t)(64 * c + 16 * ((v + (c >> 1)) & 3) + (k & 15));
}

__device__ __forceinline__ void lds_act_chunk(uint32_t row, int chunk, uint32_t (&a)[16]) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 u = lds128(row + 64 * chunk + 16 * ((v + (chunk >> 1)) & 3));
        a[4 * v + 0] = u.x;
        a[4 * v + 1] = u.y;
        a[4 * v + 2] = u.z;
        a[4 * v + 3] = u.w;
    }
}

__device__ __forceinline__ float block_max_fused(float mx, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    __syncthreads();  // red[] free from any previous use
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, red[w]);
    return mx;
}

// 16 bytes of x (+ x2) as binary32 values: 8 bfloat16 or 4 float32 elements.
template <typename T>
struct FusedVec;
template <>
struct FusedVec<uint16_t> {
    static constexpr int n = 8;
    __device__ static void load(const SProblem& pr, int64_t e, float (&f)[8]) {
        const uint4 u = ld_shared_ro16(static_cast<const uint16_t*>(pr.x) + e);
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
    __device__ static void load(const SProblem& pr, int64_t e, float (&f)[4]) {
        const uint4 u = ld_shared_ro16(static_cast<const float*>(pr.x) + e);
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
        if (pr.x2) {
            const uint4 v = ld_shared_ro16(pr.x2 + e);
            f[0] = __fadd_rn(f[0], __uint_as_float(v.x));
            f[1] = __fadd_rn(f[1], __uint_as_float(v.y));
            f[2] = __fadd_rn(f[2], __uint_as_float(v.z));
            f[3] = __fadd_rn(f[3], __uint_as_float(v.w));
        }
    }
};

constexpr int kFuseVec = 8;  // 16-byte vectors per thread held in registers

// Quantises V consecutive values into the slot (and, for the owner, global).
template <int V>
__device__ __forceinline__ void fused_store(const SProblem& pr, const float (&f)[V], int64_t base, int k,
                                            uint8_t* dst_row, float beta, float rbeta, bool out) {
    uint32_t w[V / 4];
#pragma unroll
    for (int j = 0; j < V / 4; ++j) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) x |= (uint32_t)(uint8_t)quantize_one(f[4 * j + b], beta, rbeta) << (8 * b);
        w[j] = x;
    }
#pragma unroll
    for (int j = 0; j < V / 4; ++j) *reinterpret_cast<uint32_t*>(dst_row + xs_offset(k + 4 * j)) = w[j];
    if (out) {
        int8_t* q = const_cast<int8_t*>(pr.xq) + base + k;
        if constexpr (V == 8)
            *reinterpret_cast<uint2*>(q) = make_uint2(w[0], w[1]);
        else
            *reinterpret_cast<uint32_t*>(q) = w[0];
        if (pr.x_sum) {
#pragma unroll
            for (int j = 0; j < V; ++j) pr.x_sum[base + k + j] = f[j];
        }
    }
}

// Per-token quantisation of one activation row into a shared slot row (the
// same arithmetic as act_quant_kernel: β = max|x| + 1e-8, x̃ = quantize_one),
// zero past K.  Rows of up to kThreads·kFuseVec vectors are read once into
// registers; longer rows are read twice.  The owner also writes x̃, β (and x)
// to global memory.  K is a multiple of 16 and x, x2 are 16-byte aligned.
template <typename T>
__device__ void fused_quantize_row(const SProblem& pr, int m, uint8_t* dst_row, int32_t row_bytes, float* beta_slot,
                                   float* red, bool owner) {
    constexpr int V = FusedVec<T>::n;
    const int64_t base = (int64_t)m * pr.K;
    const int nvec = pr.K / V;
    const bool out = owner && pr.write_outputs;
    float mx = 0.0f;
    if (nvec <= kThreads * kFuseVec) {
        float f[kFuseVec][V];
#pragma unroll
        for (int j = 0; j < kFuseVec; ++j) {
            const int i = threadIdx.x + j * kThreads;
            if (i < nvec) {
                FusedVec<T>::load(pr, base + (int64_t)i * V, f[j]);
#pragma unroll
                for (int e = 0; e < V; ++e) mx = fmaxf(mx, fabsf(f[j][e]));
            }
        }
        const float beta = __fadd_rn(block_max_fused(mx, red), 1e-8f);
        const float rbeta = __frcp_rn(beta);
#pragma unroll
        for (int j = 0; j < kFuseVec; ++j) {
            const int i = threadIdx.x + j * kThreads;
            if (i < nvec) fused_store<V>(pr, f[j], base, i * V, dst_row, beta, rbeta, out);
        }
        if (threadIdx.x == 0) {
            *beta_slot = beta;
            if (out) const_cast<float*>(pr.beta)[m] = beta;
        }
    } else {
        for (int i = threadIdx.x; i < nvec; i += kThreads) {
            float f[V];
            FusedVec<T>::load(pr, base + (int64_t)i * V, f);
#pragma unroll
            for (int e = 0; e < V; ++e) mx = fmaxf(mx, fabsf(f[e]));
        }
        const float beta = __fadd_rn(block_max_fused(mx, red), 1e-8f);
        const float rbeta = __frcp_rn(beta);
        for (int i = threadIdx.x; i < nvec; i += kThreads) {
            float f[V];
            FusedVec<T>::load(pr, base + (int64_t)i * V, f);
            fused_store<V>(pr, f, base, i * V, dst_row, beta, rbeta, out);
        }
        if (threadIdx.x == 0) {
            *beta_slot = beta;
            if (out) const_cast<float*>(pr.beta)[m] = beta;
        }
    }
    for (int k = pr.K + 4 * threadIdx.x; k < row_bytes; k += 4 * kThreads)
        *reinterpret_cast<uint32_t*>(dst_row + xs_offset(k)) = 0u;
}

// Issues the bulk copies of one segment (rows of one row group, chunks
// [c, c+n)) into a stage.  Called by the whole warp: lane 0 arms the
// barrier, then lane r copies row r, so the rows go out in one instruction.
__device__ __forceinline__ void issue_segment(const SProblem& pr, int rg, int c, int n, uint32_t dst, uint32_t bar,
                                              uint64_t policy, int lane) {
    const int row0 = rg * kRG;
    const int rows = min(kRG, pr.N - row0);
    const uint32_t bytes = (uint32_t)n * 16u;
    if (lane == 0) mbar_arrive_expect_tx(bar, bytes * (uint32_t)rows);
    __syncwarp();
    if (lane < rows)
        bulk_copy_g2s(dst + lane * kRowStride, pr.W + (int64_t)(row0 + lane) * pr.row_bytes + (int64_t)c * 16, bytes,
                      bar, policy);
}

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

// The token a lane finishes after reduce_scatter over kRG·MT values.
template <int MT>
__device__ __forceinline__ int lane_token(int lane) {
    constexpr int V = kRG * MT;
    int idx = 0;
#pragma unroll
    for (int half = V / 2, off = 16; half >= 1; half >>= 1, off >>= 1)
        if (lane & off) idx += half;
    return idx / kRG;
}

template <int MT, bool FUSE>
__global__ void __launch_bounds__(kThreads, BL_GEMV_MIN_BLOCKS) gemv_stream_kernel(const __grid_constant__ SParams P) {
    constexpr bool kMask = MT <= 2;  // one accumulator per code field (no shifts)
    constexpr int NS = kMask ? 4 : 1;
    constexpr int V = kRG * MT;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SharedLayout& S = *reinterpret_cast<SharedLayout*>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the next kernel on the stream (the next step's activation quantisation)
    // may be scheduled now; it waits for this grid before touching memory
    griddep_launch_dependents();

    // ---- CTA and warp ranges (equal chunk counts, CTA edges on row groups)
    const int64_t G = gridDim.x;
    const int64_t a = snap_to_row_group(P, (P.total_units * (int64_t)blockIdx.x) / G);
    const int64_t b = snap_to_row_group(P, (P.total_units * ((int64_t)blockIdx.x + 1)) / G);
    if (threadIdx.x <= kWarps) S.bound[threadIdx.x] = a + ((b - a) * threadIdx.x) / kWarps;
    for (int i = threadIdx.x; i < kSlots * kRG * kMaxMT; i += kThreads) (&S.slot_acc[0][0])[i] = 0;
    if (threadIdx.x < kSlots) S.slot_count[threadIdx.x] = 0;
    if (threadIdx.x < kWarps * kStages) mbar_init(smem_addr(&S.full[0][0] + threadIdx.x), 1);
    for (int i = threadIdx.x; i < P.count; i += kThreads) S.prob[i] = P.p[i];
    fence_mbar_init();
    __syncthreads();
    const ProbTable T{S.prob, P.count};

    const int64_t wu0 = S.bound[warp], wu1 = S.bound[warp + 1];
    const uint64_t policy = policy_evict_first();
    const uint32_t stage0 = smem_addr(&S.stage[warp][0][0]);
    const uint32_t bar0 = smem_addr(&S.full[warp][0]);

    // ---- prologue: weights do not depend on the previous kernel
    Cursor prod;
    cursor_seek(T, prod, wu0, wu1);
    int issued = 0;  // segments whose copies this warp has issued
    for (int st = 0; st < kStages && prod.u < prod.end; ++st, ++issued) {
        const int n = cursor_len(T, prod);
        const SProblem& pr = S.prob[prod.p];
        issue_segment(pr, prod.tgrg % pr.rgn, prod.c, n, stage0 + st * kStageBytes, bar0 + 8 * st, policy, lane);
        cursor_advance(T, prod, n);
    }
    griddep_wait();  // x̃, β (and α) may come from the preceding kernels

    // ---- fused quantisation: x̃ of the (at most two) problems of this CTA
    int p_first = 0;
    int second_slot = 1;  // slot of the CTA's second problem (0 when it shares the first one's input)
    uint32_t xs_base = 0;
    if constexpr (FUSE) {
        uint8_t* xs = smem_raw + sizeof(SharedLayout);
        xs_base = smem_addr(xs);
        Cursor c0, c1;
        cursor_seek(T, c0, a, b);
        cursor_seek(T, c1, b > a ? b - 1 : a, b);
        p_first = c0.p;
        for (int slot = 0; slot < 2 && a < b; ++slot) {
            const int p = p_first + slot;
            if (p > c1.p) break;
            const SProblem& pr = S.prob[p];
            const bool owner = a <= pr.unit_begin && pr.unit_begin < b;
            if (slot == 1) {
                const SProblem& p0 = S.prob[p_first];
                if (pr.x == p0.x && pr.x2 == p0.x2 && pr.K == p0.K && pr.M == p0.M) {
                    // same input as slot 0: reuse it (the owner still publishes x̃, β)
                    second_slot = 0;
                    if (owner && pr.write_outputs && (pr.xq != p0.xq || pr.beta != p0.beta || pr.x_sum != p0.x_sum))
                        second_slot = 1;  // distinct output buffers: quantise again to write them
                    if (second_slot == 0) break;
                }
            }
            for (int m = 0; m < pr.M && m < MT; ++m) {
                uint8_t* row = xs + (slot * MT + m) * P.slot_row;
                if (P.x_bf16)
                    fused_quantize_row<uint16_t>(pr, m, row, P.slot_row, &S.xbeta[slot][m], S.red, owner);
                else
                    fused_quantize_row<float>(pr, m, row, P.slot_row, &S.xbeta[slot][m], S.red, owner);
            }
        }
        __syncthreads();
    }

    // ---- main loop over this warp's segments
    Cursor cons;
    cursor_seek(T, cons, wu0, wu1);
    const int my_tok = lane_token<MT>(lane);
    int acc[kRG][MT][NS];
    int sx[MT];
    int sx_cache[MT];
    int cache_p = -1, cache_tg = -1;
    int scale_p = -1, scale_tg = -1;
    float scale = 0.0f;                   // dequant scale of this lane's output token
    float alpha_v = 0.0f, beta_v = 0.0f;  // this lane's α and β, loaded ahead of use
    bool sx_from_cache = false;
    int rg_chunks = 0;  // chunks of the current row group done by this warp
#pragma unroll
    for (int m = 0; m < MT; ++m) sx_cache[m] = 0;

    for (int seg = 0; cons.u < cons.end; ++seg) {
        const int st = seg % kStages;
        const uint32_t phase = (uint32_t)((seg / kStages) & 1);
        const SProblem& pr = S.prob[cons.p];
        const int n = cursor_len(T, cons);
        const int tg = cons.tgrg / pr.rgn;
        const int rg = cons.tgrg - tg * pr.rgn;
        const int m0 = tg * MT;

        if (rg_chunks == 0) {  // first segment of a row group for this warp
#pragma unroll
            for (int r = 0; r < kRG; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int q = 0; q < NS; ++q) acc[r][m][q] = 0;
            // Σx̃ over this lane's chunks: reuse the cached value when the whole
            // row group is ours with the usual lane-to-chunk mapping.
            const bool whole = cons.c == 0 && (cons.end - cons.u) >= pr.C;
            sx_from_cache = whole && cache_p == cons.p && cache_tg == tg;
#pragma unroll
            for (int m = 0; m < MT; ++m) sx[m] = sx_from_cache ? sx_cache[m] : 0;
        }
        if (scale_p != cons.p || scale_tg != tg) {  // start the α, β loads early
            const int tok = m0 + my_tok;
            alpha_v = *pr.alpha;
            if constexpr (FUSE)
                beta_v = tok < pr.M ? S.xbeta[cons.p == p_first ? 0 : second_slot][tok] : 0.0f;
            else
                beta_v = tok < pr.M ? pr.beta[tok] : 0.0f;
        }

        // This segment's activations do not depend on the stage: load them
        // before the wait so their latency overlaps it (single token).
        constexpr bool kPreload = (MT == 1);
        uint32_t pre[kPreload ? kIt : 1][16];
        if constexpr (kPreload) {
#pragma unroll
            for (int it = 0; it < kIt; ++it) {
                const int chunk = cons.c + it * 32 + lane;
                if constexpr (FUSE) {
                    if (it * 32 + lane < n) {
                        lds_act_chunk(xs_base + (uint32_t)((cons.p == p_first ? 0 : second_slot) * MT) * P.slot_row,
                                      chunk, pre[it]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) pre[it][q] = 0u;
                    }
                } else {
                    load_act_chunk(pr.xq + (int64_t)m0 * pr.K, pr.K, chunk, chunk < pr.full_chunks,
                                   it * 32 + lane < n && m0 < pr.M, pre[it]);
                }
            }
        }

        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8 * st, phase))) {
            // Give up: record the error, let this warp's copies in flight land
            // (bounded again), then leave.
            if (lane == 0) atomicCAS(&g_device_error, 0, (int)BL_ERR_TIMEOUT);
            for (int i = seg + 1; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % kStages), (i / kStages) & 1);
            return;
        }
        const uint32_t sbase = stage0 + st * kStageBytes;
        constexpr int kItUnroll = (MT == 1) ? kIt : 1;  // keep MT > 1 within registers
#pragma unroll(kItUnroll)
        for (int it = 0; it < kIt; ++it) {
            const int j = it * 32 + lane;
            if (j < n) {
                const int chunk = cons.c + j;
                uint32_t av[MT][16];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if constexpr (kPreload) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) av[m][q] = pre[it][q];
                    } else if constexpr (FUSE) {
                        if (m0 + m < pr.M) {
                            lds_act_chunk(xs_base + (uint32_t)((cons.p == p_first ? 0 : second_slot) * MT + m) *
                                                        P.slot_row,
                                          chunk, av[m]);
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q) av[m][q] = 0u;
                        }
                    } else {
                        load_act_chunk(pr.xq + (int64_t)(m0 + m) * pr.K, pr.K, chunk, chunk < pr.full_chunks,
                                       m0 + m < pr.M, av[m]);
                    }
                    if (!sx_from_cache) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) sx[m] = dp4a_s8s8(0x01010101u, av[m][q], sx[m]);
                    }
                }
#pragma unroll
                for (int r = 0; r < kRG; ++r) {
                    const uint4 w = lds128(sbase + r * kRowStride + j * 16);
#pragma unroll
                    for (int wj = 0; wj < 4; ++wj) {
                        const uint32_t word = word_of(w, wj);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if constexpr (kMask) {
                                const uint32_t codes = word & (0x03030303u << (2 * q));
#pragma unroll
                                for (int m = 0; m < MT; ++m)
                                    acc[r][m][q] = dp4a_u8s8(codes, av[m][4 * wj + q], acc[r][m][q]);
                            } else {
                                const uint32_t codes = (word >> (2 * q)) & 0x03030303u;
#pragma unroll
                                for (int m = 0; m < MT; ++m)
                                    acc[r][m][0] = dp4a_u8s8(codes, av[m][4 * wj + q], acc[r][m][0]);
                            }
                        }
                    }
                }
            }
        }
        rg_chunks += n;
        const bool rg_whole = (cons.c + n == pr.C) && (rg_chunks == pr.C);
        const bool rg_done = (cons.c + n == pr.C) || (cons.u + n == cons.end);
        const int seg_p = cons.p;
        const int64_t rg_u0 = pr.unit_begin + (int64_t)cons.tgrg * pr.C;

        // refill this stage with the segment kStages ahead
        __syncwarp();
        if (prod.u < prod.end) {
            const int pn = cursor_len(T, prod);
            const SProblem& pp = S.prob[prod.p];
            issue_segment(pp, prod.tgrg % pp.rgn, prod.c, pn, sbase, bar0 + 8 * st, policy, lane);
            cursor_advance(T, prod, pn);
            ++issued;
        }
        cursor_advance(T, cons, n);

        if (rg_done) {
            if (rg_whole && !sx_from_cache) {
                // a whole row group from chunk 0 (segments at multiples of 64
                // chunks, so chunk j always fell to lane j mod 32): cache Σx̃
                cache_p = seg_p;
                cache_tg = tg;
#pragma unroll
                for (int m = 0; m < MT; ++m) sx_cache[m] = sx[m];
            }
            int v[V];
#pragma unroll
            for (int r = 0; r < kRG; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    int d;
                    if constexpr (kMask)
                        d = acc[r][m][0] + (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) + (acc[r][m][3] >> 6);
                    else
                        d = acc[r][m][0];
                    v[m * kRG + r] = d - sx[m];
                }
            int idx;
            int val = reduce_scatter<V>(v, lane, idx);
            const bool writer = (lane & (32 / V - 1)) == 0;

            bool finish = rg_whole;
            if (!rg_whole) {
                // shared row group: add into its slot; the last contributor finishes it
                int slot = 0;
                for (int w = 1; w <= kWarps - 1; ++w) {
                    const int64_t bw = S.bound[w];
                    if (bw > rg_u0 && bw < rg_u0 + pr.C) {
                        slot = w;
                        break;
                    }
                }
                if (writer) atomicAdd(&S.slot_acc[slot][idx], val);
                __threadfence_block();
                __syncwarp();
                int last = 0;
                if (lane == 0) last = (atomicAdd(&S.slot_count[slot], rg_chunks) + rg_chunks == pr.C);
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence_block();
                    if (writer) val = atomicAdd(&S.slot_acc[slot][idx], 0);
                    finish = true;
                }
            }
            if (finish) {
                const int r = idx % kRG, m = idx / kRG;
                const int row = rg * kRG + r, tok = m0 + m;
                if (scale_p != seg_p || scale_tg != tg) {  // once per (problem, token group)
                    scale_p = seg_p;
                    scale_tg = tg;
                    scale = dequant_scale(alpha_v, beta_v);
                }
                if (writer && row < pr.N && tok < pr.M) {
                    float out = __fmul_rn((float)val, scale);
                    if (pr.bias) out = __fadd_rn(out, pr.bias[row]);
                    pr.y[(int64_t)tok * pr.N + row] = out;
                    if (pr.acc_out) pr.acc_out[(int64_t)tok * pr.N + row] = val;
                }
            }
            rg_chunks = 0;
        }
    }
}

// Any K and any x̃ alignment: one warp per output element, byte loads.
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

int problem_of(const SParams& P, int64_t u) {
    int p = 0;
    while (p + 1 < P.count && u >= P.p[p + 1].unit_begin) ++p;
    return p;
}

// launches the streaming kernel; with `fused` (one entry per problem) the
// kernel quantises x itself, if every CTA's range meets at most two problems
// and a slot holds the widest row (else *launched = false and nothing runs)
template <int MT>
cudaError_t launch_stream(const bitlinear_forward_problem* problems, int count, const DeviceInfo& dev,
                          cudaStream_t stream, bool pdl, const FusedInput* fused = nullptr, bool x_bf16 = false,
                          bool* launched = nullptr, bool fuse_always = false) {
    if (launched) *launched = true;
    SParams P{};
    P.count = count;
    int64_t total = 0, row_groups = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        SProblem& q = P.p[i];
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
        q.rgn = (q.N + kRG - 1) / kRG;
        q.tgn = (q.M + MT - 1) / MT;
        q.unit_begin = total;
        total += (int64_t)q.tgn * q.rgn * q.C;
        row_groups += (int64_t)q.tgn * q.rgn;
    }
    P.total_units = total;
    int64_t grid = dev.sm_count;
    if (grid > row_groups) grid = row_groups;
    size_t smem = sizeof(SharedLayout);
    if (fused) {
        int32_t slot_row = 0;
        for (int i = 0; i < count; ++i) {
            SProblem& q = P.p[i];
            if (q.M > MT) {
                *launched = false;
                return cudaSuccess;
            }
            q.x = fused[i].x;
            q.x2 = fused[i].x2;
            q.x_sum = fused[i].x_sum;
            q.write_outputs = fused[i].write_outputs ? 1 : 0;
            slot_row = std::max(slot_row, 64 * q.C);
        }
        P.x_bf16 = x_bf16 ? 1 : 0;
        P.slot_row = slot_row;
        bool fits = (int64_t)MT * slot_row <= kFuseSlotBytes;
        // Every CTA reads its problems' whole input rows before its main loop;
        // that pays off only while those reads are small next to the weights.
        int64_t prologue_bytes = 0, weight_bytes = 0;
        for (int i = 0; i < count; ++i) weight_bytes += (int64_t)P.p[i].N * P.p[i].row_bytes;
        auto input_bytes = [&](const SProblem& q) {
            return (int64_t)q.M * q.K * (x_bf16 ? 2 : 4) * (q.x2 ? 2 : 1);
        };
        for (int64_t c = 0; c < grid && fits; ++c) {
            const int64_t a = snap_to_row_group(P, (total * c) / grid);
            const int64_t b = snap_to_row_group(P, (total * (c + 1)) / grid);
            if (a >= b) continue;
            const int pa = problem_of(P, a), pb = problem_of(P, b - 1);
            fits = pb - pa <= 1;
            prologue_bytes += input_bytes(P.p[pa]);
            if (pb != pa && !(P.p[pb].x == P.p[pa].x && P.p[pb].x2 == P.p[pa].x2))
                prologue_bytes += input_bytes(P.p[pb]);
        }
        if (!fuse_always && 8 * prologue_bytes > weight_bytes) fits = false;
        if (!fits) {
            *launched = false;
            return cudaSuccess;
        }
        smem += (size_t)2 * MT * slot_row;
    }
    const void* kernel = fused ? reinterpret_cast<const void*>(gemv_stream_kernel<MT, true>)
                               : reinterpret_cast<const void*>(gemv_stream_kernel<MT, false>);
    // the opt-in is per device: set once on each device that launches the kernel
    cudaError_t attr_err = set_max_dynamic_smem(
        kernel, fused ? (int)(sizeof(SharedLayout) + 2 * kFuseSlotBytes) : (int)sizeof(SharedLayout));
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
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

cudaError_t launch_forward(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    bool fast = true;
    int64_t max_m = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& s = problems[i];
        fast = fast && (s.K % 16 == 0) && ((reinterpret_cast<uintptr_t>(s.x_q) & 15) == 0);
        // the streaming kernel indexes (token group, row group) pairs in 32 bits
        fast = fast && ((s.M + 3) / 4) * ((s.N + kRG - 1) / kRG) < ((int64_t)1 << 30);
        if (s.M > max_m) max_m = s.M;
    }
    if (!fast) return launch_generic(problems, count, dev, stream);
    if (max_m > kGemvMaxTokens) {
        // many tokens: the int8 tensor cores, all problems in one launch
        bool tc = true;
        for (int i = 0; i < count; ++i) tc = tc && gemm_tc_supported(problems[i]);
        if (tc) return launch_gemm_tc(problems, count, stream, pdl);
    }
    if (max_m == 1) return launch_stream<1>(problems, count, dev, stream, pdl);
    if (max_m == 2) return launch_stream<2>(problems, count, dev, stream, pdl);
    return launch_stream<4>(problems, count, dev, stream, pdl);
}

cudaError_t launch_linear_fused(const bitlinear_forward_problem* problems, const FusedInput* in, int count,
                                bitlinear_dtype dtype, cudaStream_t stream, bool pdl, bool* launched) {
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
        // the fused prologue reads x (and x2) in 16-byte vectors
        if ((reinterpret_cast<uintptr_t>(in[i].x) & 15) != 0 || (reinterpret_cast<uintptr_t>(in[i].x2) & 15) != 0)
            return cudaSuccess;
        if (((s.M + 3) / 4) * ((s.N + kRG - 1) / kRG) >= ((int64_t)1 << 30)) return cudaSuccess;
        if (s.M > max_m) max_m = s.M;
    }
    const bool bf16 = dtype == BL_BF16;
    if (max_m == 1) return launch_stream<1>(problems, count, dev, stream, pdl, in, bf16, launched, always);
    if (max_m == 2) return launch_stream<2>(problems, count, dev, stream, pdl, in, bf16, launched, always);
    if (max_m <= 4) return launch_stream<4>(problems, count, dev, stream, pdl, in, bf16, launched, always);
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
