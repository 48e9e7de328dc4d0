// gdr_launch.h -- host-side launchers of the looped gated-delta-rule kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "gdr_common.cuh"

namespace lt2 {

// One decode token for every head-unit of one loop (in-place state in s.S_out).
cudaError_t launch_decode(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl);

// Token-sequential CUDA-core prefill of one loop (fp32 arithmetic, any supported shape).
cudaError_t launch_prefill_seq(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl);

// Tensor-core chunked prefill of one loop (bf16 inputs, dk = dv = 128).
bool prefill_tc_supports(int dtype_bf16, int dk, int dv, int per_key);
cudaError_t launch_prefill_tc(const LoopSlice& s, cudaStream_t stream, bool pdl);

}  // namespace lt2
