// swa_prefill_cc.cu -- the looped sliding-window attention mixer on CUDA cores: fp32 arithmetic,
// any head width up to 256, fp32 or bf16 inputs and outputs.
//
// "LT2 transformer looped a tempo lineare", section "Sostituire il motore": sparse attention, every
// token looking at a window of the w most recent positions.  For every unit and token t,
//     o_t = sum_{s = max(0, t-w+1) .. t} softmax_s(scale q_t . k_s) v_s,
// taken here key by key with a running maximum m, running sum l and running output (the online
// form of the softmax: each new key rescales what came before by exp(m_old - m_new)).
//
// One warp per query, lane j holding elements j, j+32, ... of q and of the running output; each key
// costs one coalesced row read of k and of v and a warp reduction of the dot product.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdr_launch.h"
#include "gdr_nvtx.h"

namespace lt2 {
namespace swacc {

constexpr int kWarps = 4;               // queries per block
constexpr int kMaxPerLane = 8;          // d <= 256

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, typename To>
__global__ void __launch_bounds__(32 * kWarps)
swa_prefill_cc_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, To* __restrict__ o,
                      int64_t units, int64_t L, int d, int64_t window, float scale)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);   // unit * L + t
    if (row >= units * L) return;
    const int64_t t = row % L;
    const int64_t base = row - t;                                      // first row of the unit
    float qr[kMaxPerLane], acc[kMaxPerLane];
    #pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
        const int e = lane + 32 * j;
        qr[j] = e < d ? ld(q + row * d + e) * scale : 0.f;
        acc[j] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const int64_t s0 = t - window + 1 > 0 ? t - window + 1 : 0;
    for (int64_t s = s0; s <= t; ++s) {
        const T* kr = k + (base + s) * d;
        float x = 0.f;
        #pragma unroll
        for (int j = 0; j < kMaxPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < d) x = fmaf(qr[j], ld(kr + e), x);
        }
        #pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        const float mn = fmaxf(m, x);
        const float corr = expf(m - mn);                              // 0 for the first key
        const float pw = expf(x - mn);
        l = l * corr + pw;
        const T* vr = v + (base + s) * d;
        #pragma unroll
        for (int j = 0; j < kMaxPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < d) acc[j] = fmaf(pw, ld(vr + e), acc[j] * corr);
        }
        m = mn;
    }
    const float inv_l = 1.f / l;                                       // l >= 1: key t is in the window
    #pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
        const int e = lane + 32 * j;
        if (e < d) st(o + row * d + e, acc[j] * inv_l);
    }
}

template <typename T, typename To>
cudaError_t launch_typed(const SwaCall& c, cudaStream_t stream)
{
    const int64_t rows = c.units * c.L;
    const int64_t blocks = (rows + kWarps - 1) / kWarps;
    if (blocks >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    swa_prefill_cc_kernel<T, To><<<static_cast<unsigned>(blocks), 32 * kWarps, 0, stream>>>(
        static_cast<const T*>(c.q), static_cast<const T*>(c.k), static_cast<const T*>(c.v), static_cast<To*>(c.o),
        c.units, c.L, static_cast<int>(c.d), c.window, c.scale);
    return cudaGetLastError();
}

}  // namespace swacc

bool swa_cc_supports(int dtype_bf16, int d)
{
    (void)dtype_bf16;
    return d >= 1 && d <= 32 * swacc::kMaxPerLane;
}

cudaError_t launch_swa_cc(const SwaCall& c, cudaStream_t stream)
{
    using namespace swacc;
    if (c.units == 0 || c.L == 0) return cudaSuccess;
    NvtxRange range("lt2 sliding-window prefill (CUDA cores)");
    if (c.dtype_bf16)
        return c.out_bf16 ? launch_typed<__nv_bfloat16, __nv_bfloat16>(c, stream) : launch_typed<__nv_bfloat16, float>(c, stream);
    return c.out_bf16 ? launch_typed<float, __nv_bfloat16>(c, stream) : launch_typed<float, float>(c, stream);
}

}  // namespace lt2
