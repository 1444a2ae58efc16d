// Host-side launchers of the BitLinear kernels; called by the C ABI layer
// (bitlinear_api.cu) after it has validated every argument.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bitlinear.h"

namespace bl {

// Cached per-device properties (thread-safe).
struct DeviceInfo {
    int major = 0, minor = 0, sm_count = 0;
};
cudaError_t device_info(DeviceInfo* out);

cudaError_t launch_quantize_act(const bitlinear_act_problem* problems, int count, bitlinear_dtype dtype,
                                cudaStream_t stream);

size_t quantize_weights_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_quantize_weights(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K, uint8_t* W_packed,
                                    float* alpha, void* workspace, cudaStream_t stream);

// Allocation-free weight quantisation: scratch in a static device array.
size_t quantize_weights_static_scratch_bytes();
cudaError_t launch_quantize_weights_static(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                           uint8_t* W_packed, float* alpha, cudaStream_t stream);

cudaError_t launch_forward(const bitlinear_forward_problem* problems, int count, cudaStream_t stream);

}  // namespace bl
