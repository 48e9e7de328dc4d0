// gdr_common.cuh -- small device/host helpers shared by the looped gated-delta-rule kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lt2 {

// Device-side status word (bit flags, see lt2_gdr_last_device_error): a bounded wait ran
// out; a tensor-core path produced a non-finite output or state (its fp16 operands out of
// range, or non-finite inputs); a debug build's index check failed.
enum : unsigned int {
    kDevOk = 0u,
    kDevTimeout = 1u,
    kDevRange = 2u,
    kDevCheck = 4u,
    kDevSeqlens = 8u,   // a packed sequence's offsets are out of order or past the packed length
};

// Device-side invariant checks of the debug build (LT2_DEBUG): a failed check records kDevCheck
// in the status word and yields false, so that the caller skips the access; nothing traps.  In
// the product build the check compiles to `true`.
#ifdef LT2_DEBUG
__device__ __forceinline__ bool dbg_ok(bool cond, unsigned int* err)
{
    if (!cond) atomicOr(err, kDevCheck);
    return cond;
}
#else
__device__ __forceinline__ constexpr bool dbg_ok(bool, unsigned int*) { return true; }
#endif

// Per-launch view of one loop's slice: base pointers already offset to loop tau.
struct LoopSlice {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* S0;     // nullable: zero initial state
    void* o;
    float* S_out;        // nullable (prefill) / in-out state (decode)
    int64_t units;       // B * H head-units in this loop
    int64_t L;
    int dk;
    int dv;
    int per_key;
    int decay_first;     // per-key gating applied as (I - beta k k^T) Diag(alpha)
    int out_bf16;        // o stored as bf16 (else fp32)
    unsigned int* err;   // device status word
    // fused prologue and output gate (all zero: none)
    int qk_norm;         // q, k raw: normalise every row to unit L2 norm
    int gate_logits;     // alpha, beta hold logits: alpha = exp(-softplus(a) c), beta = sigmoid(b)
    float alpha_scale;   // c
    const void* z;       // output gate logits (layout and dtype of v), or null
    // packed sequences: unit u = (sequence u / H, head u % H) holds tokens cu[b] .. cu[b+1]-1 of
    // rows [H][L] (L is then the packed length); null: every unit has its own L rows
    const int64_t* cu = nullptr;
    int H = 0;
};

// The fused prologue and output gate, in fp32: the same formulas on every path.
__device__ __forceinline__ float sigmoid_f32(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float softplus_f32(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float alpha_from_logit(float a, float c) { return expf(-softplus_f32(a) * c); }
// 1 / max(sqrt(ss), 1e-12) for a row's sum of squares ss
__device__ __forceinline__ float inv_l2(float ss) { return 1.f / fmaxf(sqrtf(ss), 1e-12f); }
// The same three with the hardware approximations (relative errors 2^-11 to 2^-21), for the
// tensor-core paths, whose operands are fp16 anyway: a short instruction footprint matters
// more there than the last bits.
// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh (relative error ~2^-11, below the
// fp16 operands' own rounding): three instructions
__device__ __forceinline__ float sigmoid_fast(float x)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
__device__ __forceinline__ float alpha_from_logit_fast(float a, float c)
{
    return __expf(-(fmaxf(a, 0.f) + __logf(1.f + __expf(-fabsf(a)))) * c);
}
__device__ __forceinline__ float inv_l2_fast(float ss) { return rsqrtf(fmaxf(ss, 1e-24f)); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Programmatic dependent launch: let the next kernel on the stream start now.  Only the
// library's own launches of later loops carry the attribute that honours this trigger, and
// loops are independent recurrences, so none of them waits on the previous loop's results;
// any other kernel launched after these still waits for their completion.
__device__ __forceinline__ void allow_next_loop_to_start() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float4 ld_stream_f4(const float* p) {
    float4 r;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream_f4(float* p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

}  // namespace lt2
