// gdr_launch.h -- host-side launchers of the looped gated-delta-rule kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "gdr_common.cuh"

namespace lt2 {

// One decode token for every head-unit of one loop (in-place state in s.S_out).
cudaError_t launch_decode(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl);

// Token-sequential CUDA-core prefill of one loop (fp32 arithmetic, any supported shape).
cudaError_t launch_prefill_seq(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl);

// Tensor-core chunked prefill (bf16 inputs, dk = dv = 128), all T loops: one launch per loop,
// back to back on `stream`, loops after the first allowed to start early (they share no data).
struct TcCall {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* S0;       // nullable
    void* o;
    float* S_out;          // nullable
    int64_t T;
    int64_t units_per_loop;  // B * H
    int64_t L;               // >= 1
    int out_bf16;
    int decay_first;         // per-key gating as (I - beta k k^T) Diag(alpha)
    unsigned int* err;
    int qk_norm;             // fused prologue and output gate, as in LoopSlice
    int gate_logits;
    float alpha_scale;
    const void* z;
    // packed sequences: device offsets [units_per_loop / H + 1] (null: fixed length L); then L
    // is the packed length Ntot and q/k/v/o/z are [T][H][Ntot][128], alpha/beta [T][H][Ntot]
    const int64_t* cu_seqlens = nullptr;
    int64_t H = 0;
    // scratch for the balanced schedule of the scalar kernel (one flag per unit), or null
    void* workspace = nullptr;
    size_t workspace_bytes = 0;
};
// The fused steps of a call as the template argument of the tensor-core kernels' instances.
enum FuseBits : int { kFuseNorm = 1, kFuseLogits = 2, kFuseGate = 4 };
inline int fuse_bits(const TcCall& c)
{
    return (c.qk_norm ? kFuseNorm : 0) | (c.gate_logits ? kFuseLogits : 0) | (c.z ? kFuseGate : 0);
}

// Scalar gating: 64-token chunks.  Per-key gating: 32-token chunks in the e-form (chunks whose
// per-key decay is out of the tensor-core range run token by token inside the same kernel).
bool prefill_tc_supports(int dtype_bf16, int dk, int dv, int per_key);
// Workspace bytes of the scalar tensor-core prefill's balanced schedule: one flag per unit.
size_t prefill_tc_flag_bytes(int64_t units);
cudaError_t launch_prefill_tc_all(const TcCall& call, cudaStream_t stream);
bool prefill_kda_tc_supports(int dtype_bf16, int dk, int dv);
cudaError_t launch_prefill_kda_tc_all(const TcCall& call, cudaStream_t stream);

// Sliding-window attention prefill, every unit of every loop in one launch.
struct SwaCall {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    int64_t units;     // T * B * H
    int64_t L;         // >= 1
    int64_t d;
    int64_t window;    // >= 1
    float scale;       // > 0 after defaulting
    int dtype_bf16;
    int out_bf16;
    unsigned int* err;
};
// Tensor cores (bf16, d = 128): 128 queries per CTA, keys in blocks of 64, two CTAs per SM.
bool swa_tc_supports(int dtype_bf16, int d);
cudaError_t launch_swa_tc(const SwaCall& c, cudaStream_t stream);
// CUDA cores (fp32 arithmetic, d <= 256): one warp per query.
bool swa_cc_supports(int dtype_bf16, int d);
cudaError_t launch_swa_cc(const SwaCall& c, cudaStream_t stream);

// Backward pass on CUDA cores (fp32 arithmetic; q/k/v/dO fp32 or bf16, gradients fp32), every
// unit of every loop in one launch (units = T * B * H).
struct BwCall {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* S0;       // nullable
    const void* dO;
    const float* dSL;      // nullable
    float* dq;
    float* dk_out;
    float* dv_out;
    float* dalpha;
    float* dbeta;
    float* dS0;            // nullable
    float* ws;
    int64_t units;
    int64_t L;
    int dk;
    int dv;
    int per_key;
    int decay_first;
    int dtype_bf16;
};
size_t backward_workspace_bytes(int64_t units, int64_t L, int dk, int dv);
// The fixed scratch array of the allocation-free backward entry point: its size, and its device
// address on the current device (looked up on the first call on each device).
size_t backward_static_scratch_bytes();
cudaError_t backward_static_scratch(float** out);
cudaError_t launch_backward(const BwCall& c, cudaStream_t stream);

#ifdef LT2_DEBUG
// Fault injection of the debug build: the producer of every later launch stops before `chunk`.
cudaError_t debug_set_skip_chunk_scalar(int chunk);
cudaError_t debug_set_skip_chunk_per_key(int chunk);
#endif

}  // namespace lt2
