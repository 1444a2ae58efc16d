// Host-side launchers of the BitLinear kernels; called by the C ABI layer
// (bitlinear_api.cu) after it has validated every argument.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bitlinear.h"

namespace bl {

// Cached per-device properties (thread-safe).
struct DeviceInfo {
    int major = 0, minor = 0, sm_count = 0;
};
cudaError_t device_info(DeviceInfo* out);

// Opts `func` in to `bytes` of dynamic shared memory on the current device,
// once per (kernel, device) for the life of the process (thread-safe).
cudaError_t set_max_dynamic_smem(const void* func, int bytes);

// One activation-quantisation job: x = a, or a + b (float32 only) when b is
// set; x_sum (nullable) receives x.
struct ActJob {
    const void* a;
    const float* b;
    float* x_sum;
    int8_t* x_q;
    float* beta;
    int64_t M, K;
};

// pdl: launch with programmatic dependent launch (the kernel waits for its
// predecessor before reading x); early_trigger: let the next PDL kernel start
// before that wait (only when no work in flight writes the next kernel's
// weights).
cudaError_t launch_quantize_act_jobs(const ActJob* jobs, int count, bitlinear_dtype dtype, cudaStream_t stream,
                                     bool pdl, bool early_trigger);
cudaError_t launch_quantize_act(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                cudaStream_t stream, bool pdl = false, bool early_trigger = false);

// 4-bit activations: x_q of each problem is packed [M][ceil(K/2)] (two per byte).
cudaError_t launch_quantize_act_a4(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                   cudaStream_t stream, bool pdl);

size_t quantize_weights_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_quantize_weights(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K, uint8_t* W_packed,
                                    float* alpha, void* workspace, cudaStream_t stream);

// One α per group of `group` consecutive elements of each row (group a
// multiple of 16, or >= K for one per row): alpha [N][ceil(K/group)].
cudaError_t launch_quantize_weights_groups(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K, int64_t group,
                                           uint8_t* W_packed, float* alpha, cudaStream_t stream);

// Allocation-free weight quantisation: scratch in a static device array.
size_t quantize_weights_static_scratch_bytes();
cudaError_t launch_quantize_weights_static(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                           uint8_t* W_packed, float* alpha, cudaStream_t stream);

// pdl: launch with programmatic dependent launch; only valid right after the
// library's own activation-quantisation kernel on the same stream (the weight
// stream starts before the dependency wait).
// alpha_rows: each problem's alpha is a per-row table [N] ("1.58 位大模型" §3.1:
// one α per output row), applied as y = RN32(RN32(fp32(acc)·α_n)·RN32(RN64(β/127)));
// only for at most four tokens (the streaming GEMV).
cudaError_t launch_forward(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl,
                           bool alpha_rows = false);

// Fused linear for at most four tokens: the streaming GEMV quantises its own
// activations (x, or x + x2 in float32) into shared memory, so the pair of
// kernels becomes one launch.  One entry per problem; x_sum (nullable) and the
// problem's x_q / beta receive x, x̃ and β when write_outputs is set.
struct FusedInput {
    const void* x;
    const float* x2;
    float* x_sum;
    bool write_outputs;
    int32_t had_block;  // > 0: rotate x by the block-diagonal Hadamard of this block first (x2, x_sum NULL)
};
// *launched = false (and nothing enqueued) when the problems do not fit the
// fused kernel; the caller then runs the quantisation and product separately.
// a4: 4-bit activations ("BitNet CPU 实测" §2.1 variant): codes clip(rint(7x/β), ±7),
// x_q written as nibbles [M][K/2], y = fp32(acc)·RN32(RN64(α·β/7)).
cudaError_t launch_linear_fused(const bitlinear_forward_problem* problems, const FusedInput* in, int count,
                                bitlinear_dtype dtype, cudaStream_t stream, bool pdl, bool* launched,
                                bool alpha_rows = false, bool a4 = false);

// Hadamard rotation (out = x·H·scale) or rotation + per-token int8
// quantisation (x_q, beta), one job per problem of a grouped launch; all jobs
// of a launch are of one kind (x_q set on all, or on none) and one dtype.
struct HadJob {
    const void* x;
    float* out;
    int8_t* x_q;
    float* beta;
    int64_t M, K;
    int block;    // power of two dividing K, at most hadamard_max_block()
    float scale;  // rotation only
};
int hadamard_max_block();
cudaError_t launch_hadamard(const HadJob* jobs, int count, bitlinear_dtype dtype, cudaStream_t stream, bool pdl);

// Product with one α per group of `group` input features of a row (group >= K:
// one per row), alpha [N][ceil(K/group)]; any M (four tokens per pass).
struct ScaledProblem {
    const int8_t* x_q;
    const float* beta;
    const uint8_t* W_packed;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;  // one α per row only
    int64_t M, N, K, group;
};
cudaError_t launch_forward_scaled(const ScaledProblem* problems, int count, cudaStream_t stream, bool pdl);
// Product on 4-bit activations (x_q packed [M][ceil(K/2)]), one α for the
// tensor: y = fp32(acc)·RN32(RN64(α·β/7)) (+ bias).
cudaError_t launch_forward_a4(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl);

// Straight-through backward: grad_x [M][K] = α·(g·Ŵ), grad_W [N][K] = clip mask ⊙
// ((g·s)ᵀ·x̃); either output may be NULL.
cudaError_t launch_ste_backward(const float* g, int64_t M, int64_t N, int64_t K, const uint8_t* W_packed,
                                const float* alpha, const int8_t* x_q, const float* beta, const void* W,
                                bitlinear_dtype w_dtype, float* grad_x, float* grad_W, cudaStream_t stream);

// Tensor-core GEMM for many tokens (tcgen05, int8): all problems in one launch.
bool gemm_tc_supported(const bitlinear_forward_problem& p);
cudaError_t launch_gemm_tc(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl);
cudaError_t read_gemm_error(int* code);

// Device-side error word (bounded waits that expired): read and clear.
cudaError_t read_device_error(int* code);
cudaError_t launch_wait_timeout_selftest(uint32_t polls, cudaStream_t stream);

}  // namespace bl
