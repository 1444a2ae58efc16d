// C ABI of libbitlinear.so (declared in include/bitlinear.h).
//
// Every entry point validates its arguments on the host first and returns an
// error before touching the device, then checks that the current device is
// compute capability 10.0, then enqueues kernels on the caller's stream.
#include <mutex>

#include "bl_attr.h"
#include "bl_launch.h"

namespace bl {

cudaError_t device_info(DeviceInfo* out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        DeviceInfo d;
        err = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        cache[dev] = d;
        have[dev] = true;
    }
    *out = cache[dev];
    return cudaSuccess;
}

cudaError_t set_max_dynamic_smem(const void* func, int bytes) {
    static AttrOnce once;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const int rc = once.ensure(func, dev, [&] {
        return (int)cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
    return rc < 0 ? cudaErrorInvalidDevice : static_cast<cudaError_t>(rc);
}

}  // namespace bl

namespace {

constexpr int64_t kMaxRows = (int64_t)1 << 31;
constexpr int64_t kMaxWeights = (int64_t)1 << 40;

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

bitlinear_status check_device() {
    bl::DeviceInfo d;
    cudaError_t err = bl::device_info(&d);
    if (err != cudaSuccess) {
        cudaGetLastError();
        return BL_ERR_CUDA;
    }
    if (d.major != 10 || d.minor != 0) return BL_ERR_ARCH;
    return BL_OK;
}

bitlinear_status from_cuda(cudaError_t err) {
    if (err == cudaSuccess) return BL_OK;
    cudaGetLastError();
    return BL_ERR_CUDA;
}

bitlinear_status check_act(const bitlinear_act_problem& p) {
    if (!p.x || !p.x_q || !p.beta) return BL_ERR_NULL;
    if (p.M < 1 || p.K < 1 || p.K > BITLINEAR_MAX_K || p.M > kMaxRows) return BL_ERR_SHAPE;
    if (misaligned(p.beta, 4)) return BL_ERR_ALIGN;
    return BL_OK;
}

bitlinear_status check_forward(const bitlinear_forward_problem& p) {
    if (!p.x_q || !p.beta || !p.W_packed || !p.alpha || !p.y) return BL_ERR_NULL;
    if (p.M < 1 || p.N < 1 || p.K < 1 || p.K > BITLINEAR_MAX_K || p.M > kMaxRows || p.N > kMaxRows)
        return BL_ERR_SHAPE;
    if (misaligned(p.W_packed, 16) || misaligned(p.beta, 4) || misaligned(p.alpha, 4) || misaligned(p.y, 4) ||
        misaligned(p.bias, 4) || misaligned(p.acc_out, 4))
        return BL_ERR_ALIGN;
    return BL_OK;
}

bool valid_dtype(bitlinear_dtype d) { return d == BL_F32 || d == BL_BF16; }

// Byte ranges [p, p + n) and [q, q + m) intersect.
bool ranges_overlap(const void* p, int64_t n, const void* q, int64_t m) {
    if (!p || !q) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + (uintptr_t)m && b < a + (uintptr_t)n;
}

// Some x_sum of the call overlaps some a or b of the call.
bool sums_overlap_inputs(const bitlinear_act_sum_problem* acts, int n) {
    for (int i = 0; i < n; ++i) {
        if (!acts[i].x_sum) continue;
        const int64_t bytes_i = acts[i].M * acts[i].K * 4;
        for (int j = 0; j < n; ++j) {
            const int64_t bytes_j = acts[j].M * acts[j].K * 4;
            if (ranges_overlap(acts[i].x_sum, bytes_i, acts[j].a, bytes_j) ||
                ranges_overlap(acts[i].x_sum, bytes_i, acts[j].b, bytes_j))
                return true;
        }
    }
    return false;
}

}  // namespace

extern "C" {

size_t bitlinear_packed_row_bytes(int64_t K) {
    if (K < 1) return 0;
    return (size_t)(16 * ((K + 63) / 64));
}

size_t bitlinear_quantize_weights_workspace_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < 1) return 0;
    return bl::quantize_weights_workspace_bytes(N, K);
}

bitlinear_status bitlinear_quantize_weights(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                            uint8_t* W_packed, float* alpha, void* workspace,
                                            size_t workspace_bytes, bitlinear_stream_t stream) {
    if (!W || !W_packed || !alpha) return BL_ERR_NULL;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (N < 1 || K < 1 || K > BITLINEAR_MAX_K || N > kMaxWeights / K) return BL_ERR_SHAPE;
    if (misaligned(W_packed, 16) || misaligned(alpha, 4) || misaligned(W, dtype == BL_F32 ? 4 : 2))
        return BL_ERR_ALIGN;
    if (!workspace || workspace_bytes < bl::quantize_weights_workspace_bytes(N, K)) return BL_ERR_WORKSPACE;
    if (misaligned(workspace, 8)) return BL_ERR_ALIGN;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_quantize_weights(W, dtype, N, K, W_packed, alpha, workspace,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

bitlinear_status bitlinear_quantize_weights_static(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                                   uint8_t* W_packed, float* alpha, bitlinear_stream_t stream) {
    if (!W || !W_packed || !alpha) return BL_ERR_NULL;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (N < 1 || K < 1 || K > BITLINEAR_MAX_K || N > kMaxWeights / K) return BL_ERR_SHAPE;
    if (bl::quantize_weights_workspace_bytes(N, K) > bl::quantize_weights_static_scratch_bytes()) return BL_ERR_SHAPE;
    if (misaligned(W_packed, 16) || misaligned(alpha, 4) || misaligned(W, dtype == BL_F32 ? 4 : 2))
        return BL_ERR_ALIGN;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_quantize_weights_static(W, dtype, N, K, W_packed, alpha,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

bitlinear_status bitlinear_quantize_act(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K, int8_t* x_q,
                                        float* beta, bitlinear_stream_t stream) {
    bitlinear_act_problem p{x, x_q, beta, M, K};
    return bitlinear_quantize_act_grouped(&p, 1, dtype, stream);
}

bitlinear_status bitlinear_quantize_act_grouped(const bitlinear_act_problem* problems, int count,
                                                bitlinear_dtype dtype, bitlinear_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        bitlinear_status st = check_act(problems[i]);
        if (st != BL_OK) return st;
        if (misaligned(problems[i].x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
        rows += problems[i].M;
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_quantize_act(problems, count, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

bitlinear_status bitlinear_forward(const int8_t* x_q, const float* beta, int64_t M, int64_t K,
                                   const uint8_t* W_packed, const float* alpha, int64_t N, const float* bias,
                                   float* y, int32_t* acc_out, bitlinear_stream_t stream) {
    bitlinear_forward_problem p{x_q, beta, W_packed, alpha, bias, y, acc_out, M, N, K};
    return bitlinear_forward_grouped(&p, 1, stream);
}

bitlinear_status bitlinear_forward_grouped(const bitlinear_forward_problem* problems, int count,
                                           bitlinear_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    for (int i = 0; i < count; ++i) {
        bitlinear_status st = check_forward(problems[i]);
        if (st != BL_OK) return st;
    }
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_forward(problems, count, reinterpret_cast<cudaStream_t>(stream), false));
}

bitlinear_status bitlinear_linear(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                  const uint8_t* W_packed, const float* alpha, int64_t N, const float* bias,
                                  int8_t* x_q, float* beta, float* y, int32_t* acc_out, bitlinear_stream_t stream) {
    bitlinear_linear_problem p{x, x_q, beta, W_packed, alpha, bias, y, acc_out, M, N, K};
    return bitlinear_linear_grouped(&p, 1, dtype, 0u, stream);
}

bitlinear_status bitlinear_linear_grouped(const bitlinear_linear_problem* problems, int count, bitlinear_dtype dtype,
                                          uint32_t flags, bitlinear_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (flags & ~(uint32_t)(BL_LINEAR_WEIGHTS_STATIC | BL_LINEAR_HADAMARD)) return BL_ERR_FLAGS;
    const bool rotate = (flags & BL_LINEAR_HADAMARD) != 0;
    bitlinear_act_problem act[BITLINEAR_MAX_GROUP];
    bitlinear_forward_problem fwd[BITLINEAR_MAX_GROUP];
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_linear_problem& q = problems[i];
        act[i] = bitlinear_act_problem{q.x, q.x_q, q.beta, q.M, q.K};
        fwd[i] = bitlinear_forward_problem{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K};
        bitlinear_status st = check_act(act[i]);
        if (st == BL_OK) st = check_forward(fwd[i]);
        if (st != BL_OK) return st;
        if (misaligned(q.x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
        if (rotate && bitlinear_hadamard_block(q.K) < 2) return BL_ERR_SHAPE;
        rows += q.M;
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool weights_static = (flags & BL_LINEAR_WEIGHTS_STATIC) != 0;
    if (rotate) {
        // one token: rotation and quantisation in the product kernel's prologue
        bl::FusedInput rin[BITLINEAR_MAX_GROUP];
        for (int i = 0; i < count; ++i)
            rin[i] = bl::FusedInput{problems[i].x, nullptr, nullptr, true,
                                    (int32_t)bitlinear_hadamard_block(problems[i].K)};
        bool fused = false;
        st = from_cuda(bl::launch_linear_fused(fwd, rin, count, dtype, s, weights_static, &fused));
        if (st != BL_OK || fused) return st;
        // else rotation + quantisation in one grouped launch, then the product
        // (the product kernel streams weights early only under the flag)
        bl::HadJob jobs[BITLINEAR_MAX_GROUP];
        for (int i = 0; i < count; ++i)
            jobs[i] = bl::HadJob{problems[i].x, nullptr, problems[i].x_q, problems[i].beta, problems[i].M,
                                 problems[i].K, (int)bitlinear_hadamard_block(problems[i].K), 1.0f};
        st = from_cuda(bl::launch_hadamard(jobs, count, dtype, s, true));
        if (st != BL_OK) return st;
        return from_cuda(bl::launch_forward(fwd, count, s, true));
    }
    // few tokens: one launch that quantises in the product kernel's prologue
    bl::FusedInput fin[BITLINEAR_MAX_GROUP];
    for (int i = 0; i < count; ++i) fin[i] = bl::FusedInput{problems[i].x, nullptr, nullptr, true, 0};
    bool launched = false;
    st = from_cuda(bl::launch_linear_fused(fwd, fin, count, dtype, s, weights_static, &launched));
    if (st != BL_OK || launched) return st;
    st = from_cuda(bl::launch_quantize_act(act, count, dtype, s, true, weights_static));
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_forward(fwd, count, s, true));
}

// Copies `count` (dst[i], src[i], bytes[i]) on `stream`, one cudaMemcpyAsync
// per run of pairs that are adjacent on both sides, skipping a pair equal to an
// earlier one (problems sharing an input).
static cudaError_t copy_runs(void* const* dst, const void* const* src, const size_t* bytes, int count,
                             cudaMemcpyKind kind, cudaStream_t s) {
    int i = 0;
    while (i < count) {
        bool repeat = false;
        for (int j = 0; j < i && !repeat; ++j) repeat = dst[j] == dst[i] && src[j] == src[i] && bytes[j] == bytes[i];
        if (repeat) {
            ++i;
            continue;
        }
        size_t run = bytes[i];
        int k = i + 1;
        while (k < count && static_cast<const char*>(dst[i]) + run == dst[k] &&
               static_cast<const char*>(src[i]) + run == src[k]) {
            run += bytes[k];
            ++k;
        }
        cudaError_t err = cudaMemcpyAsync(dst[i], src[i], run, kind, s);
        if (err != cudaSuccess) return err;
        i = k;
    }
    return cudaSuccess;
}

bitlinear_status bitlinear_linear_grouped_host(const bitlinear_linear_problem* problems, const bitlinear_host_io* io,
                                               int count, bitlinear_dtype dtype, uint32_t flags,
                                               bitlinear_stream_t stream) {
    if (!problems || !io) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (flags & ~(uint32_t)(BL_LINEAR_WEIGHTS_STATIC | BL_LINEAR_HADAMARD)) return BL_ERR_FLAGS;
    void* xd[BITLINEAR_MAX_GROUP];
    const void* xh[BITLINEAR_MAX_GROUP];
    void* yh[BITLINEAR_MAX_GROUP];
    const void* yd[BITLINEAR_MAX_GROUP];
    size_t xb[BITLINEAR_MAX_GROUP], yb[BITLINEAR_MAX_GROUP];
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_linear_problem& q = problems[i];
        if (!io[i].x_host || !io[i].y_host) return BL_ERR_NULL;
        // the shapes are checked by the grouped call below; the copy sizes are
        // only formed once M, N, K are known to be in range
        const bitlinear_act_problem a{q.x, q.x_q, q.beta, q.M, q.K};
        const bitlinear_forward_problem f{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K};
        bitlinear_status st = check_act(a);
        if (st == BL_OK) st = check_forward(f);
        if (st != BL_OK) return st;
        if (misaligned(q.x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
        if ((flags & BL_LINEAR_HADAMARD) && bitlinear_hadamard_block(q.K) < 2) return BL_ERR_SHAPE;
        rows += q.M;
        xd[i] = const_cast<void*>(q.x);
        xh[i] = io[i].x_host;
        xb[i] = (size_t)q.M * (size_t)q.K * (dtype == BL_F32 ? 4 : 2);
        yd[i] = q.y;
        yh[i] = io[i].y_host;
        yb[i] = (size_t)q.M * (size_t)q.N * 4;
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = from_cuda(copy_runs(xd, xh, xb, count, cudaMemcpyHostToDevice, s));
    if (st != BL_OK) return st;
    st = bitlinear_linear_grouped(problems, count, dtype, flags, stream);
    if (st != BL_OK) return st;
    return from_cuda(copy_runs(yh, yd, yb, count, cudaMemcpyDeviceToHost, s));
}

bitlinear_status bitlinear_linear_block(const bitlinear_act_sum_problem* acts, int n_acts,
                                        const bitlinear_forward_problem* fwd, int n_fwd, uint32_t flags,
                                        bitlinear_stream_t stream) {
    if ((n_acts > 0 && !acts) || (n_fwd > 0 && !fwd)) return BL_ERR_NULL;
    if (n_acts < 0 || n_fwd < 0 || n_acts > BITLINEAR_MAX_GROUP || n_fwd > BITLINEAR_MAX_GROUP || n_acts + n_fwd == 0)
        return BL_ERR_COUNT;
    if (flags & ~(uint32_t)BL_LINEAR_WEIGHTS_STATIC) return BL_ERR_FLAGS;
    bl::ActJob jobs[BITLINEAR_MAX_GROUP];
    int64_t rows = 0;
    for (int i = 0; i < n_acts; ++i) {
        const bitlinear_act_sum_problem& p = acts[i];
        if (!p.a || !p.x_q || !p.beta) return BL_ERR_NULL;
        if (p.M < 1 || p.K < 1 || p.K > BITLINEAR_MAX_K || p.M > kMaxRows) return BL_ERR_SHAPE;
        if (misaligned(p.a, 4) || misaligned(p.b, 4) || misaligned(p.x_sum, 4) || misaligned(p.beta, 4))
            return BL_ERR_ALIGN;
        jobs[i] = bl::ActJob{p.a, p.b, p.x_sum, p.x_q, p.beta, p.M, p.K};
        rows += p.M;
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    for (int i = 0; i < n_fwd; ++i) {
        bitlinear_status st = check_forward(fwd[i]);
        if (st != BL_OK) return st;
    }
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool weights_static = (flags & BL_LINEAR_WEIGHTS_STATIC) != 0;
    // Fused single launch when every product reads one of this call's inputs
    // and every input feeds a product: each product quantises its input in its
    // prologue; the first product of each input writes that input's outputs.
    if (n_acts > 0 && n_fwd > 0) {
        bl::FusedInput fin[BITLINEAR_MAX_GROUP];
        bool used[BITLINEAR_MAX_GROUP] = {};
        // In the fused form other CTAs still read a and b while the owner of an
        // input writes its x_sum, so an x_sum that overlaps any input rules it out.
        bool ok = !sums_overlap_inputs(acts, n_acts);
        for (int i = 0; i < n_fwd && ok; ++i) {
            int j = 0;
            while (j < n_acts && !(acts[j].x_q == fwd[i].x_q && acts[j].beta == fwd[i].beta && acts[j].M == fwd[i].M &&
                                   acts[j].K == fwd[i].K))
                ++j;
            if (j == n_acts) {
                ok = false;
                break;
            }
            fin[i] = bl::FusedInput{acts[j].a, acts[j].b, used[j] ? nullptr : acts[j].x_sum, !used[j], 0};
            used[j] = true;
        }
        for (int j = 0; j < n_acts && ok; ++j) ok = used[j];
        if (ok) {
            bool launched = false;
            st = from_cuda(bl::launch_linear_fused(fwd, fin, n_fwd, BL_F32, s, weights_static, &launched));
            if (st != BL_OK || launched) return st;
        }
    }
    if (n_acts > 0) {
        st = from_cuda(bl::launch_quantize_act_jobs(jobs, n_acts, BL_F32, s, true, weights_static));
        if (st != BL_OK) return st;
    }
    // The product kernel streams weights before its dependency wait: chained
    // after this call's own quantisation kernel, or after any work when the
    // caller vouches that nothing in flight writes the weights.
    if (n_fwd > 0) return from_cuda(bl::launch_forward(fwd, n_fwd, s, n_acts > 0 || weights_static));
    return BL_OK;
}

int64_t bitlinear_hadamard_block(int64_t K) {
    if (K < 1) return 0;
    int64_t b = 1;
    while (K % (2 * b) == 0 && 2 * b <= BITLINEAR_MAX_HADAMARD_BLOCK) b *= 2;
    return b;
}

static bitlinear_status check_hadamard(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K, int64_t block) {
    if (!x) return BL_ERR_NULL;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (M < 1 || K < 1 || K > BITLINEAR_MAX_K || M > kMaxRows) return BL_ERR_SHAPE;
    if (block < 1 || (block & (block - 1)) != 0 || block > BITLINEAR_MAX_HADAMARD_BLOCK || K % block != 0)
        return BL_ERR_SHAPE;
    if (block > bl::hadamard_max_block()) return BL_ERR_SHAPE;
    if (misaligned(x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
    return BL_OK;
}

bitlinear_status bitlinear_hadamard(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K, int64_t block,
                                    float scale, float* out, bitlinear_stream_t stream) {
    bitlinear_status st = check_hadamard(x, dtype, M, K, block);
    if (st != BL_OK) return st;
    if (!out) return BL_ERR_NULL;
    if (misaligned(out, 4)) return BL_ERR_ALIGN;
    st = check_device();
    if (st != BL_OK) return st;
    bl::HadJob job{x, out, nullptr, nullptr, M, K, (int)block, scale};
    return from_cuda(bl::launch_hadamard(&job, 1, dtype, reinterpret_cast<cudaStream_t>(stream), false));
}

bitlinear_status bitlinear_quantize_act_hadamard(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                                 int64_t block, int8_t* x_q, float* beta, bitlinear_stream_t stream) {
    bitlinear_status st = check_hadamard(x, dtype, M, K, block);
    if (st != BL_OK) return st;
    if (!x_q || !beta) return BL_ERR_NULL;
    if (misaligned(beta, 4)) return BL_ERR_ALIGN;
    st = check_device();
    if (st != BL_OK) return st;
    bl::HadJob job{x, nullptr, x_q, beta, M, K, (int)block, 1.0f};
    return from_cuda(bl::launch_hadamard(&job, 1, dtype, reinterpret_cast<cudaStream_t>(stream), false));
}

static bool valid_group(int64_t K, int64_t group) { return group >= K || (group > 0 && group % 64 == 0); }

bitlinear_status bitlinear_quantize_weights_scaled(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                                   int64_t group, uint8_t* W_packed, float* alpha,
                                                   bitlinear_stream_t stream) {
    if (!W || !W_packed || !alpha) return BL_ERR_NULL;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (N < 1 || K < 1 || K > BITLINEAR_MAX_K || N > kMaxWeights / K || !valid_group(K, group)) return BL_ERR_SHAPE;
    if (misaligned(W_packed, 16) || misaligned(alpha, 4) || misaligned(W, dtype == BL_F32 ? 4 : 2))
        return BL_ERR_ALIGN;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_quantize_weights_groups(W, dtype, N, K, group >= K ? K : group, W_packed, alpha,
                                                        reinterpret_cast<cudaStream_t>(stream)));
}

bitlinear_status bitlinear_linear_scaled(const bitlinear_scaled_problem* problems, int count, bitlinear_dtype dtype,
                                         uint32_t flags, bitlinear_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (flags & ~(uint32_t)BL_LINEAR_WEIGHTS_STATIC) return BL_ERR_FLAGS;
    bitlinear_act_problem act[BITLINEAR_MAX_GROUP];
    bl::ScaledProblem fwd[BITLINEAR_MAX_GROUP];
    int nact = 0;
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_scaled_problem& q = problems[i];
        bitlinear_forward_problem f{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K};
        bitlinear_status st = check_forward(f);
        if (st != BL_OK) return st;
        if (!valid_group(q.K, q.group) || (q.acc_out && q.group < q.K)) return BL_ERR_SHAPE;
        if (q.x) {
            act[nact] = bitlinear_act_problem{q.x, q.x_q, q.beta, q.M, q.K};
            st = check_act(act[nact]);
            if (st != BL_OK) return st;
            if (misaligned(q.x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
            ++nact;
            rows += q.M;
        }
        fwd[i] = bl::ScaledProblem{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K,
                                   q.group >= q.K ? q.K : q.group};
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool weights_static = (flags & BL_LINEAR_WEIGHTS_STATIC) != 0;
    // One α per row and at most four tokens: the streaming GEMV with the row's
    // α in its epilogue, quantising x in its prologue when it can.
    bool rows_path = true;
    for (int i = 0; i < count && rows_path; ++i) {
        const bitlinear_scaled_problem& q = problems[i];
        rows_path = q.group >= q.K && q.M <= 4 && q.K % 16 == 0 && !misaligned(q.x_q, 16);
    }
    if (rows_path) {
        bitlinear_forward_problem f[BITLINEAR_MAX_GROUP];
        for (int i = 0; i < count; ++i) {
            const bitlinear_scaled_problem& q = problems[i];
            f[i] = bitlinear_forward_problem{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K};
        }
        if (nact == count) {
            bl::FusedInput fin[BITLINEAR_MAX_GROUP];
            for (int i = 0; i < count; ++i) fin[i] = bl::FusedInput{problems[i].x, nullptr, nullptr, true, 0};
            bool launched = false;
            st = from_cuda(bl::launch_linear_fused(f, fin, count, dtype, s, weights_static, &launched, true));
            if (st != BL_OK || launched) return st;
        }
        if (nact > 0) {
            st = from_cuda(bl::launch_quantize_act(act, nact, dtype, s, true, weights_static));
            if (st != BL_OK) return st;
        }
        return from_cuda(bl::launch_forward(f, count, s, nact > 0 || weights_static, true));
    }
    if (nact > 0) {
        st = from_cuda(bl::launch_quantize_act(act, nact, dtype, s, true, weights_static));
        if (st != BL_OK) return st;
    }
    return from_cuda(bl::launch_forward_scaled(fwd, count, s, nact > 0 || weights_static));
}

bitlinear_status bitlinear_quantize_act_a4(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K, uint8_t* x_q4,
                                           float* beta, bitlinear_stream_t stream) {
    bitlinear_act_problem p{x, reinterpret_cast<int8_t*>(x_q4), beta, M, K};
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    bitlinear_status st = check_act(p);
    if (st != BL_OK) return st;
    if (misaligned(x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
    st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_quantize_act_a4(&p, 1, dtype, reinterpret_cast<cudaStream_t>(stream), false));
}

bitlinear_status bitlinear_forward_a4(const uint8_t* x_q4, const float* beta, int64_t M, int64_t K,
                                      const uint8_t* W_packed, const float* alpha, int64_t N, const float* bias,
                                      float* y, int32_t* acc_out, bitlinear_stream_t stream) {
    bitlinear_forward_problem p{reinterpret_cast<const int8_t*>(x_q4), beta, W_packed, alpha, bias, y, acc_out, M, N, K};
    bitlinear_status st = check_forward(p);
    if (st != BL_OK) return st;
    st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_forward_a4(&p, 1, reinterpret_cast<cudaStream_t>(stream), false));
}

bitlinear_status bitlinear_linear_a4(const bitlinear_linear_problem* problems, int count, bitlinear_dtype dtype,
                                     uint32_t flags, bitlinear_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BITLINEAR_MAX_GROUP) return BL_ERR_COUNT;
    if (!valid_dtype(dtype)) return BL_ERR_DTYPE;
    if (flags & ~(uint32_t)BL_LINEAR_WEIGHTS_STATIC) return BL_ERR_FLAGS;
    bitlinear_act_problem act[BITLINEAR_MAX_GROUP];
    bitlinear_forward_problem fwd[BITLINEAR_MAX_GROUP];
    int64_t rows = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_linear_problem& q = problems[i];
        act[i] = bitlinear_act_problem{q.x, q.x_q, q.beta, q.M, q.K};
        fwd[i] = bitlinear_forward_problem{q.x_q, q.beta, q.W_packed, q.alpha, q.bias, q.y, q.acc_out, q.M, q.N, q.K};
        bitlinear_status st = check_act(act[i]);
        if (st == BL_OK) st = check_forward(fwd[i]);
        if (st != BL_OK) return st;
        if (misaligned(q.x, dtype == BL_F32 ? 4 : 2)) return BL_ERR_ALIGN;
        rows += q.M;
    }
    if (rows >= kMaxRows) return BL_ERR_SHAPE;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool weights_static = (flags & BL_LINEAR_WEIGHTS_STATIC) != 0;
    // at most four tokens: one launch of the streaming GEMV that quantises x
    // to 4 bits in its prologue, when the problems fit it
    bool fusable = true;
    for (int i = 0; i < count && fusable; ++i)
        fusable = problems[i].M <= 4 && problems[i].K % 16 == 0 && !misaligned(problems[i].x_q, 4);
    if (fusable) {
        bl::FusedInput fin[BITLINEAR_MAX_GROUP];
        for (int i = 0; i < count; ++i) fin[i] = bl::FusedInput{problems[i].x, nullptr, nullptr, true, 0};
        bool launched = false;
        st = from_cuda(bl::launch_linear_fused(fwd, fin, count, dtype, s, weights_static, &launched, false, true));
        if (st != BL_OK || launched) return st;
    }
    st = from_cuda(bl::launch_quantize_act_a4(act, count, dtype, s, true));
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_forward_a4(fwd, count, s, true));
}

bitlinear_status bitlinear_train_forward(const void* W, bitlinear_dtype w_dtype, int64_t N, int64_t K, const void* x,
                                         bitlinear_dtype x_dtype, int64_t M, uint8_t* W_packed, float* alpha,
                                         int8_t* x_q, float* beta, float* y, void* workspace, size_t workspace_bytes,
                                         bitlinear_stream_t stream) {
    // validate both steps before launching either
    if (!x || !x_q || !beta || !y) return BL_ERR_NULL;
    if (!valid_dtype(x_dtype)) return BL_ERR_DTYPE;
    bitlinear_act_problem a{x, x_q, beta, M, K};
    bitlinear_status st = check_act(a);
    if (st != BL_OK) return st;
    if (misaligned(x, x_dtype == BL_F32 ? 4 : 2) || misaligned(y, 4)) return BL_ERR_ALIGN;
    st = bitlinear_quantize_weights(W, w_dtype, N, K, W_packed, alpha, workspace, workspace_bytes, stream);
    if (st != BL_OK) return st;
    bitlinear_linear_problem p{x, x_q, beta, W_packed, alpha, nullptr, y, nullptr, M, N, K};
    return bitlinear_linear_grouped(&p, 1, x_dtype, 0u, stream);
}

bitlinear_status bitlinear_ste_backward(const float* g, int64_t M, int64_t N, int64_t K, const uint8_t* W_packed,
                                        const float* alpha, const int8_t* x_q, const float* beta, const void* W,
                                        bitlinear_dtype w_dtype, float* grad_x, float* grad_W,
                                        bitlinear_stream_t stream) {
    if (!g || !alpha) return BL_ERR_NULL;
    if (grad_x && !W_packed) return BL_ERR_NULL;
    if (grad_W && (!x_q || !beta || !W)) return BL_ERR_NULL;
    if (grad_W && !valid_dtype(w_dtype)) return BL_ERR_DTYPE;
    if (M < 1 || N < 1 || K < 1 || K > BITLINEAR_MAX_K || M > kMaxRows || N > kMaxRows || N > kMaxWeights / K)
        return BL_ERR_SHAPE;
    if (misaligned(g, 4) || misaligned(alpha, 4) || misaligned(grad_x, 4) || misaligned(grad_W, 4) ||
        misaligned(beta, 4) || (grad_W && misaligned(W, w_dtype == BL_F32 ? 4 : 2)))
        return BL_ERR_ALIGN;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_ste_backward(g, M, N, K, W_packed, alpha, x_q, beta, W, w_dtype, grad_x, grad_W,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

bitlinear_status bitlinear_device_error(int* code) {
    if (!code) return BL_ERR_NULL;
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    int a = 0, b = 0;
    cudaError_t err = bl::read_device_error(&a);
    if (err == cudaSuccess) err = bl::read_gemm_error(&b);
    *code = a ? a : b;
    return from_cuda(err);
}

bitlinear_status bitlinear_selftest_timeout(uint32_t polls, bitlinear_stream_t stream) {
    bitlinear_status st = check_device();
    if (st != BL_OK) return st;
    return from_cuda(bl::launch_wait_timeout_selftest(polls, reinterpret_cast<cudaStream_t>(stream)));
}

const char* bitlinear_status_string(bitlinear_status status) {
    switch (status) {
        case BL_OK: return "ok";
        case BL_ERR_NULL: return "a required pointer is NULL";
        case BL_ERR_SHAPE: return "a size is out of range";
        case BL_ERR_ALIGN: return "a pointer is not aligned as required";
        case BL_ERR_DTYPE: return "unknown dtype";
        case BL_ERR_WORKSPACE: return "workspace missing or too small";
        case BL_ERR_ARCH: return "device is not compute capability 10.0 (B200)";
        case BL_ERR_CUDA: return "CUDA runtime error";
        case BL_ERR_COUNT: return "group count out of range";
        case BL_ERR_TIMEOUT: return "a kernel's bounded wait expired";
        case BL_ERR_FLAGS: return "unknown flag bits";
    }
    return "unknown status";
}

int bitlinear_version(void) { return 102; }

}  // extern "C"
