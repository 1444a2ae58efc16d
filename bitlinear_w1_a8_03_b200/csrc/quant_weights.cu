// Absmean ternary weight quantisation and 2-bit packing.
//
// "1.58-bit 大模型极限量化实战" (chenxutan.com/d/5049.html) §2.3 and §4.1:
// α = mean(|W|) over the tensor, Ŵ = clip(round(W/α), -1, 1); stored at two
// bits per weight with codes 00/01/10 for -1/0/+1 (§5.3).  Done once per
// weight matrix and cached (§3.2).
//
// α is exact: every |w| is a 24-bit significand times a power of two, so the
// kernels add them into a 320-bit fixed-point integer (the sum scaled by
// 2^149), held as ten 32-bit limbs in 64-bit lanes with deferred carries.  The
// sum therefore does not depend on the order or the grid, and the mean is
// rounded once to binary64 and once to binary32: α = RN32(RN64(Σ|W| / count)).
//
// Three launches: per-CTA partial sums -> one-CTA finalise (writes α) ->
// quantise + pack (reads α).  All are HBM-bound on W; the matrix is read twice.
#include <mutex>

#include "bl_common.cuh"
#include "bl_launch.h"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kLimbs = 10;          // 320 bits: 2^-149 .. 2^128 times up to 2^40 terms
constexpr int kMaxPartials = 1024;  // partial sums written to the workspace

// Adds |w|·2^149 into the limb accumulator.  The significand lands in limbs
// li and li + 1 (li = p / 32 ≤ 7 for every finite w); a switch on li keeps
// the accumulator in registers and costs a few instructions per element where
// a select over all ten limbs cost about forty (the weights of a matrix have
// few distinct li, so a warp rarely diverges on it).
__device__ __forceinline__ void add_abs(uint64_t (&acc)[kLimbs], float w) {
    const uint32_t bits = __float_as_uint(w) & 0x7FFFFFFFu;
    const uint32_t e = bits >> 23;
    uint32_t sig = bits & 0x7FFFFFu;
    if (e != 0) sig |= 0x800000u;
    const uint32_t p = (e != 0 ? e : 1u) - 1u;  // bit position of the significand
    const uint32_t li = p >> 5;
    const uint64_t v = (uint64_t)sig << (p & 31u);
    const uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    switch (li) {
#define BL_ADD_AT(L)       \
    case L:                \
        acc[L] += lo;      \
        acc[L + 1] += hi;  \
        break;
        BL_ADD_AT(0)
        BL_ADD_AT(1)
        BL_ADD_AT(2)
        BL_ADD_AT(3)
        BL_ADD_AT(4)
        BL_ADD_AT(5)
        BL_ADD_AT(6)
        BL_ADD_AT(7)
#undef BL_ADD_AT
        default:  // not reached: p <= 254, so li <= 7
            break;
    }
}

__device__ __forceinline__ void normalize(uint64_t (&acc)[kLimbs]) {
#pragma unroll
    for (int j = 0; j + 1 < kLimbs; ++j) {
        acc[j + 1] += acc[j] >> 32;
        acc[j] &= 0xFFFFFFFFull;
    }
}

// Sums the per-thread limb vectors of the CTA into thread 0 (normalised).
__device__ void block_sum(uint64_t (&acc)[kLimbs]) {
    __shared__ uint64_t sm[kThreads][kLimbs + 1];
    normalize(acc);
#pragma unroll
    for (int j = 0; j < kLimbs; ++j) sm[threadIdx.x][j] = acc[j];
    __syncthreads();
    for (int stride = kThreads / 2; stride > 0; stride >>= 1) {
        if ((int)threadIdx.x < stride) {
#pragma unroll
            for (int j = 0; j < kLimbs; ++j) sm[threadIdx.x][j] += sm[threadIdx.x + stride][j];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < kLimbs; ++j) acc[j] = sm[0][j];
        normalize(acc);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) absmean_partial_kernel(const T* __restrict__ W, int64_t count,
                                                                   unsigned long long* __restrict__ partials) {
    uint64_t acc[kLimbs];
#pragma unroll
    for (int j = 0; j < kLimbs; ++j) acc[j] = 0;
    const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    constexpr int V = 16 / sizeof(T);
    const bool vec = (reinterpret_cast<uintptr_t>(W) & 15) == 0;
    int64_t done = 0;
    if (vec) {
        const int64_t nvec = count / V;
        for (int64_t u = tid; u < nvec; u += stride) {
            const uint4 v = ld_stream16(W + u * V);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (sizeof(T) == 4) {
                    add_abs(acc, __uint_as_float(w4[i]));
                } else {
                    add_abs(acc, __uint_as_float(w4[i] << 16));
                    add_abs(acc, __uint_as_float(w4[i] & 0xFFFF0000u));
                }
            }
        }
        done = nvec * V;
    }
    for (int64_t i = done + tid; i < count; i += stride) add_abs(acc, load_as_f32(W, i));
    block_sum(acc);
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < kLimbs; ++j) partials[(int64_t)blockIdx.x * kLimbs + j] = acc[j];
    }
}

// Bits [lo, lo+n) of a little-endian array of 32-bit limbs (n <= 53, lo >= 0).
__device__ uint64_t extract_bits(const uint32_t* q, int nlimbs, int lo, int n) {
    uint64_t r = 0;
    for (int b = 0; b < n; ++b) {
        const int pos = lo + b;
        const int li = pos >> 5;
        if (li < nlimbs && ((q[li] >> (pos & 31)) & 1u)) r |= 1ull << b;
    }
    return r;
}

// RN32(RN64(S / count)) for S·2^149 = acc (normalised 32-bit digits in
// 64-bit lanes).  T = S·2^128; Q = floor(T / count), R = T mod count.
__device__ float limbs_mean(const uint64_t (&acc)[kLimbs], int64_t count) {
    constexpr int kT = kLimbs + 4;
    uint32_t t[kT], q[kT];
    for (int j = 0; j < 4; ++j) t[j] = 0;
    for (int j = 0; j < kLimbs; ++j) t[4 + j] = (uint32_t)acc[j];
    unsigned __int128 rem = 0;
    const unsigned __int128 d = (unsigned __int128)(uint64_t)count;
    for (int j = kT - 1; j >= 0; --j) {
        const unsigned __int128 cur = (rem << 32) | t[j];
        q[j] = (uint32_t)(cur / d);
        rem = cur % d;
    }
    int top = -1;
    for (int j = kT - 1; j >= 0 && top < 0; --j)
        if (q[j] != 0) top = 32 * j + 31 - __clz(q[j]);
    if (top < 0) return 0.0f;  // Σ|W| = 0
    // mean = (Q + R/count)·2^-277.  Round Q to 53 significant bits, half to even;
    // S >= 1 gives Q >= 2^88, so top >= 88 and all shifts below are valid.
    uint64_t mant = extract_bits(q, kT, top - 52, 53);
    const bool round_bit = extract_bits(q, kT, top - 53, 1) != 0;
    bool sticky = rem != 0;
    for (int pos = 0; pos < top - 53 && !sticky; ++pos)
        if ((q[pos >> 5] >> (pos & 31)) & 1u) sticky = true;
    int e = top - 52 - 277;
    if (round_bit && (sticky || (mant & 1ull))) {
        ++mant;
        if (mant == (1ull << 53)) {
            mant >>= 1;
            ++e;
        }
    }
    const double mean = ldexp((double)mant, e);  // exact: a normal binary64
    return __double2float_rn(mean);
}

__global__ void __launch_bounds__(kThreads) absmean_finalize_kernel(const unsigned long long* __restrict__ partials,
                                                                    int nparts, int64_t count,
                                                                    float* __restrict__ alpha) {
    uint64_t acc[kLimbs];
#pragma unroll
    for (int j = 0; j < kLimbs; ++j) acc[j] = 0;
    for (int g = threadIdx.x; g < nparts; g += kThreads) {
#pragma unroll
        for (int j = 0; j < kLimbs; ++j) acc[j] += partials[(int64_t)g * kLimbs + j];
    }
    block_sum(acc);
    if (threadIdx.x != 0) return;
    *alpha = limbs_mean(acc, count);
}

// One α per group of `group` consecutive elements of each row (the last group
// of a row may be shorter): the same exact mean as for the tensor, one warp
// per group, the limb vectors of the lanes summed by shuffles.
template <typename T>
__global__ void __launch_bounds__(kThreads) absmean_groups_kernel(const T* __restrict__ W, int64_t N, int64_t K,
                                                                  int64_t group, float* __restrict__ alpha) {
    const int lane = threadIdx.x & 31;
    const int64_t G = (K + group - 1) / group;
    const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t gi = warp0; gi < N * G; gi += nwarps) {
        const int64_t n = gi / G, g = gi - n * G;
        const int64_t k0 = g * group, k1 = min(K, k0 + group);
        uint64_t acc[kLimbs];
#pragma unroll
        for (int j = 0; j < kLimbs; ++j) acc[j] = 0;
        for (int64_t k = k0 + lane; k < k1; k += 32) add_abs(acc, load_as_f32(W + n * K, k));
        normalize(acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int j = 0; j < kLimbs; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
        if (lane == 0) {
            normalize(acc);
            alpha[gi] = limbs_mean(acc, k1 - k0);
        }
    }
}

__device__ __forceinline__ uint32_t ternary_code(float w, float alpha) {
    const float q = __fdiv_rn(w, alpha);
    if (q != q) return 1u;  // 0/0 when α underflowed to 0: the zero weight
    float r = rintf(q);     // round half to even
    r = fminf(fmaxf(r, -1.0f), 1.0f);
    return (uint32_t)(__float2int_rn(r) + 1);
}

// One thread per packed 32-bit word (16 weights).  Weight 16g + 4s + b sits
// in byte b, bits 2s..2s+1 of word g; weights past K carry the zero code 01.
// group == 0: one α for the tensor; otherwise α[n][k / group] (group a
// multiple of 16, so a word's 16 weights share one α).
template <typename T>
__global__ void __launch_bounds__(kThreads) ternary_pack_kernel(const T* __restrict__ W, int64_t N, int64_t K,
                                                                int64_t row_words, const float* __restrict__ alpha_p,
                                                                int64_t group, uint32_t* __restrict__ out) {
    const float alpha_t = group == 0 ? *alpha_p : 0.0f;
    const int64_t G = group == 0 ? 1 : (K + group - 1) / group;
    const int64_t total = N * row_words;
    constexpr int V = 16 / sizeof(T);
    const bool vec_rows = ((reinterpret_cast<uintptr_t>(W) & 15) == 0) && (K % V == 0);
    for (int64_t wi = (int64_t)blockIdx.x * kThreads + threadIdx.x; wi < total; wi += (int64_t)gridDim.x * kThreads) {
        const int64_t n = wi / row_words;
        const int64_t k0 = (wi - n * row_words) * 16;
        const T* row = W + n * K;
        const float alpha = group == 0 ? alpha_t : alpha_p[n * G + min(k0, K - 1) / group];
        float f[16];
        if (vec_rows && k0 + 16 <= K) {
#pragma unroll
            for (int v = 0; v < 16 / V; ++v) {
                const uint4 u = ld_stream16(row + k0 + v * V);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if constexpr (sizeof(T) == 4) {
                        f[v * 4 + i] = __uint_as_float(w4[i]);
                    } else {
                        f[v * 8 + 2 * i] = __uint_as_float(w4[i] << 16);
                        f[v * 8 + 2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) f[i] = (k0 + i < K) ? load_as_f32(row, k0 + i) : 0.0f;
        }
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t code = (k0 + i < K) ? ternary_code(f[i], alpha) : 1u;
            word |= code << (8 * (i & 3) + 2 * (i >> 2));
        }
        out[wi] = word;
    }
}

int partial_blocks(int64_t count) {
    const int64_t want = (count + (int64_t)kThreads * 64 - 1) / ((int64_t)kThreads * 64);
    return (int)(want < 1 ? 1 : (want > kMaxPartials ? kMaxPartials : want));
}

}  // namespace

size_t quantize_weights_workspace_bytes(int64_t N, int64_t K) {
    return (size_t)partial_blocks(N * K) * kLimbs * sizeof(unsigned long long);
}

cudaError_t launch_quantize_weights(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K, uint8_t* W_packed,
                                    float* alpha, void* workspace, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t count = N * K;
    const int nparts = partial_blocks(count);
    auto* partials = static_cast<unsigned long long*>(workspace);
    const int64_t row_words = (int64_t)bitlinear_packed_row_bytes(K) / 4;
    const int64_t words = N * row_words;
    int64_t pack_blocks = (words + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)dev.sm_count * 16;
    if (pack_blocks > cap) pack_blocks = cap;
    if (dtype == BL_BF16) {
        const auto* w = static_cast<const uint16_t*>(W);
        absmean_partial_kernel<uint16_t><<<nparts, kThreads, 0, stream>>>(w, count, partials);
        absmean_finalize_kernel<<<1, kThreads, 0, stream>>>(partials, nparts, count, alpha);
        ternary_pack_kernel<uint16_t><<<(unsigned)pack_blocks, kThreads, 0, stream>>>(
            w, N, K, row_words, alpha, 0, reinterpret_cast<uint32_t*>(W_packed));
    } else {
        const auto* w = static_cast<const float*>(W);
        absmean_partial_kernel<float><<<nparts, kThreads, 0, stream>>>(w, count, partials);
        absmean_finalize_kernel<<<1, kThreads, 0, stream>>>(partials, nparts, count, alpha);
        ternary_pack_kernel<float><<<(unsigned)pack_blocks, kThreads, 0, stream>>>(
            w, N, K, row_words, alpha, 0, reinterpret_cast<uint32_t*>(W_packed));
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_weights_groups(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K, int64_t group,
                                           uint8_t* W_packed, float* alpha, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t G = (K + group - 1) / group;
    int64_t blocks = (N * G + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)dev.sm_count * 16;
    if (blocks > cap) blocks = cap;
    const int64_t row_words = (int64_t)bitlinear_packed_row_bytes(K) / 4;
    int64_t pack_blocks = (N * row_words + kThreads - 1) / kThreads;
    if (pack_blocks > cap) pack_blocks = cap;
    if (dtype == BL_BF16) {
        const auto* w = static_cast<const uint16_t*>(W);
        absmean_groups_kernel<uint16_t><<<(unsigned)blocks, kThreads, 0, stream>>>(w, N, K, group, alpha);
        ternary_pack_kernel<uint16_t><<<(unsigned)pack_blocks, kThreads, 0, stream>>>(
            w, N, K, row_words, alpha, group, reinterpret_cast<uint32_t*>(W_packed));
    } else {
        const auto* w = static_cast<const float*>(W);
        absmean_groups_kernel<float><<<(unsigned)blocks, kThreads, 0, stream>>>(w, N, K, group, alpha);
        ternary_pack_kernel<float><<<(unsigned)pack_blocks, kThreads, 0, stream>>>(
            w, N, K, row_words, alpha, group, reinterpret_cast<uint32_t*>(W_packed));
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant (bitlinear_quantize_weights_static).
//
// Some callers may not allocate device memory at all: a plugin running inside
// a host application that owns the whole device-memory budget, or a
// latency-critical loop in which cudaMalloc/cudaFree (which can synchronise
// the device) are not allowed.  For them the partial sums of α live in this
// fixed module-scope array instead of a caller workspace.  Its size is fixed:
// kMaxPartials × kLimbs 64-bit words (80 KiB), which covers every accepted
// matrix because the partial-sum grid never exceeds kMaxPartials CTAs.  Every
// GPU that loads the library holds the array until the process exits.
//
// Each call overwrites the partial sums it reads (nothing has to start at
// zero), and every call on a device shares the one array: calls that overlap
// on the GPU (for example on two streams without ordering) race and give
// wrong α.  In host code the array's name is only a host-side handle, so its
// device address is looked up once per device with cudaGetSymbolAddress, on
// that device's first call; that first call should therefore come before any
// stream capture.
static __device__ __align__(256) unsigned long long g_static_partials[kMaxPartials * kLimbs];
static_assert(sizeof(g_static_partials) == (size_t)kMaxPartials * kLimbs * sizeof(unsigned long long),
              "the static scratch holds the largest partial-sum grid (partial_blocks never exceeds kMaxPartials)");

namespace {

cudaError_t static_partials(unsigned long long** out) {
    static std::mutex mu;
    static unsigned long long* addr[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_static_partials);
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<unsigned long long*>(p);
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

size_t quantize_weights_static_scratch_bytes() { return sizeof(g_static_partials); }

cudaError_t launch_quantize_weights_static(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                           uint8_t* W_packed, float* alpha, cudaStream_t stream) {
    if (quantize_weights_workspace_bytes(N, K) > sizeof(g_static_partials)) return cudaErrorInvalidValue;
    unsigned long long* scratch = nullptr;
    cudaError_t err = static_partials(&scratch);
    if (err != cudaSuccess) return err;
    return launch_quantize_weights(W, dtype, N, K, W_packed, alpha, scratch, stream);
}

}  // namespace bl
