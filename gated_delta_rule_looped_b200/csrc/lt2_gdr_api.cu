// lt2_gdr_api.cu -- the C ABI declared in include/lt2_gdr.h: argument validation, path
// selection and the loop orchestration (T launches back to back on one stream).
#include <cuda_runtime.h>

#include <atomic>
#include <initializer_list>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gdr_common.cuh"
#include "gdr_launch.h"
#include "gdr_nvtx.h"
#include "lt2_gdr.h"

namespace {

// Status word of the kernels on this device (bit flags, see gdr_common.cuh), followed by the
// slot that lt2_gdr_last_device_error() swaps it into; one instance per device that loads the
// library, shared by every call on that device.
__device__ unsigned int g_lt2_device_status[2] = {0u, 0u};

// Reads the status word and clears it in one atomic step, leaving the old value in word 1.
__global__ void take_status_kernel(unsigned int* w) { w[1] = atomicExch(&w[0], 0u); }

using lt2::NvtxRange;

thread_local char t_cuda_error[256] = {0};

lt2_status cuda_fail(cudaError_t e, const char* where)
{
    std::snprintf(t_cuda_error, sizeof(t_cuda_error), "%s: %s (%d)", where,
                  cudaGetErrorString(e), (int)e);
    return LT2_ERR_CUDA;
}

// Device address of the status word for the current device (cached per device).
constexpr int kMaxDevices = 64;
std::atomic<unsigned int*> g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

lt2_status status_word(unsigned int** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return LT2_ERR_UNSUPPORTED;
    unsigned int* p = g_status_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_status_mu);
        p = g_status_ptr[dev].load(std::memory_order_acquire);
        if (!p) {
            e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_lt2_device_status);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
            g_status_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return LT2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte ranges for the aliasing checks.
struct Range {
    uintptr_t lo, hi;
};
Range range_of(const void* p, int64_t bytes)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + static_cast<uintptr_t>(bytes)};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

constexpr int64_t kMaxDim = int64_t(1) << 31;

// Per-key gating in either order of the per-key factors.
bool is_per_key(const lt2_gdr_dims* d)
{
    return d->gate == LT2_GATE_PER_KEY || d->gate == LT2_GATE_PER_KEY_DECAY_FIRST;
}

bool out_is_bf16(const lt2_gdr_dims* d)
{
    return d->out_dtype == LT2_OUT_BF16 || (d->out_dtype == LT2_OUT_SAME && d->dtype == LT2_DTYPE_BF16);
}

struct Sizes {
    int64_t units;        // T*B*H
    int64_t per_loop;     // B*H
    int64_t qk, vo, al, be, st;   // element counts over all loops
    int esz;              // bytes per q/k/v element
    int osz;              // bytes per o element
};

lt2_status validate_dims(const lt2_gdr_dims* d, Sizes* sz)
{
    if (!d) return LT2_ERR_INVALID_ARGUMENT;
    if (d->T < 0 || d->B < 0 || d->H < 0 || d->L < 0 || d->dk <= 0 || d->dv <= 0)
        return LT2_ERR_INVALID_ARGUMENT;
    if (d->T >= kMaxDim || d->B >= kMaxDim || d->H >= kMaxDim || d->L >= kMaxDim ||
        d->dk >= kMaxDim || d->dv >= kMaxDim)
        return LT2_ERR_INVALID_ARGUMENT;
    if (d->dtype != LT2_DTYPE_F32 && d->dtype != LT2_DTYPE_BF16) return LT2_ERR_INVALID_ARGUMENT;
    if (d->gate != LT2_GATE_SCALAR && !is_per_key(d)) return LT2_ERR_INVALID_ARGUMENT;
    if (d->algo < LT2_ALGO_AUTO || d->algo > LT2_ALGO_CUDA_CORE) return LT2_ERR_INVALID_ARGUMENT;
    if (d->out_dtype < LT2_OUT_SAME || d->out_dtype > LT2_OUT_BF16) return LT2_ERR_INVALID_ARGUMENT;
    if (d->dk > 128 || d->dv > 128 || (d->dk % 8) != 0 || (d->dv % 8) != 0)
        return LT2_ERR_UNSUPPORTED;
    // Overflow-safe element counts (each factor < 2^31; check the running products).
    __int128 units = (__int128)d->T * d->B * d->H;
    __int128 tok = units * d->L;
    __int128 big = tok * 128;
    if (big > ((__int128)1 << 62)) return LT2_ERR_INVALID_ARGUMENT;
    sz->units = (int64_t)units;
    sz->per_loop = d->B * d->H;
    sz->qk = (int64_t)(tok * d->dk);
    sz->vo = (int64_t)(tok * d->dv);
    sz->al = (int64_t)(is_per_key(d) ? tok * d->dk : tok);
    sz->be = (int64_t)tok;
    sz->st = (int64_t)(units * d->dk * d->dv);
    sz->esz = d->dtype == LT2_DTYPE_BF16 ? 2 : 4;
    sz->osz = out_is_bf16(d) ? 2 : 4;
    // Head-units are indexed with 32-bit integers inside the kernels (grid size, the first
    // unit of a loop, TMA coordinates).
    if (sz->units >= kMaxDim) return LT2_ERR_UNSUPPORTED;
    return LT2_OK;
}

// Element counts of a packed-sequence call: dims->B sequences whose tokens are packed along
// dims->L = Ntot; q/k/v/o [T][H][Ntot][d], gates [T][H][Ntot](x dk), states [T][B][H][dk][dv].
lt2_status validate_varlen_dims(const lt2_gdr_dims* d, Sizes* sz)
{
    lt2_status st = validate_dims(d, sz);
    if (st != LT2_OK) return st;
    const __int128 rows = (__int128)d->T * d->H * d->L;      // packed token-heads
    if (rows * 128 > ((__int128)1 << 62)) return LT2_ERR_INVALID_ARGUMENT;
    sz->qk = (int64_t)(rows * d->dk);
    sz->vo = (int64_t)(rows * d->dv);
    sz->al = (int64_t)(is_per_key(d) ? rows * d->dk : rows);
    sz->be = (int64_t)rows;
    if (d->T * d->H >= kMaxDim) return LT2_ERR_UNSUPPORTED;   // TMA unit axis, 32-bit
    return LT2_OK;
}

// Every non-null pointer must address device memory of the current device: kernels launch
// on the current device, and the tensor maps of the tensor-core path would otherwise cover
// another GPU's memory.
lt2_status on_current_device(std::initializer_list<const void*> ptrs)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    for (const void* p : ptrs) {
        if (!p) continue;
        cudaPointerAttributes a;
        e = cudaPointerGetAttributes(&a, p);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();      // not a pointer CUDA knows (the error is not sticky)
            return LT2_ERR_INVALID_ARGUMENT;
        }
        const bool device_mem = a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
        if (!device_mem || a.device != dev) return LT2_ERR_INVALID_ARGUMENT;
    }
    return LT2_OK;
}

// Null / alignment checks for a tensor of `count` elements.
bool tensor_ok(const void* p, int64_t count)
{
    if (count == 0) return true;
    return p != nullptr && aligned16(p);
}

bool use_tensor_core(const lt2_gdr_dims* d)
{
    const bool ok = lt2::prefill_tc_supports(d->dtype == LT2_DTYPE_BF16, (int)d->dk, (int)d->dv,
                                             is_per_key(d));
    if (d->algo == LT2_ALGO_CUDA_CORE) return false;
    return ok;
}

// The fused prologue and output gate of a call: a zeroed struct when `f` is null.
lt2_gdr_fused fused_or_none(const lt2_gdr_fused* f)
{
    lt2_gdr_fused none;
    std::memset(&none, 0, sizeof(none));
    return f ? *f : none;
}

lt2_status validate_fused(const lt2_gdr_fused& f, const Sizes& sz, const void* o, const float* S_out)
{
    if (f.reserved != 0) return LT2_ERR_INVALID_ARGUMENT;
    if ((f.qk_l2norm != 0 && f.qk_l2norm != 1) || (f.gate_logits != 0 && f.gate_logits != 1))
        return LT2_ERR_INVALID_ARGUMENT;
    if (f.gate_logits && !(f.alpha_scale >= 0.f && f.alpha_scale <= 3.4e38f)) return LT2_ERR_INVALID_ARGUMENT;
    if (f.z) {
        if (!aligned16(f.z)) return LT2_ERR_INVALID_ARGUMENT;
        const Range rz = range_of(f.z, sz.vo * sz.esz);
        if (overlap(rz, range_of(o, sz.vo * sz.osz))) return LT2_ERR_INVALID_ARGUMENT;
        if (S_out && overlap(rz, range_of(S_out, sz.st * 4))) return LT2_ERR_INVALID_ARGUMENT;
    }
    return LT2_OK;
}

lt2::LoopSlice loop_slice(const lt2_gdr_dims* d, const Sizes& sz, int64_t tau,
                          const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* S0, void* o, float* S_out,
                          unsigned int* err, const lt2_gdr_fused& f)
{
    const int64_t U = sz.per_loop, L = d->L, dk = d->dk, dv = d->dv;
    const int64_t na = is_per_key(d) ? dk : 1;
    lt2::LoopSlice s;
    s.q = static_cast<const char*>(q) + tau * U * L * dk * sz.esz;
    s.k = static_cast<const char*>(k) + tau * U * L * dk * sz.esz;
    s.v = static_cast<const char*>(v) + tau * U * L * dv * sz.esz;
    s.alpha = alpha + tau * U * L * na;
    s.beta = beta + tau * U * L;
    s.S0 = S0 ? S0 + tau * U * dk * dv : nullptr;
    s.o = static_cast<char*>(o) + tau * U * L * dv * sz.osz;
    s.S_out = S_out ? S_out + tau * U * dk * dv : nullptr;
    s.units = U;
    s.L = L;
    s.dk = (int)dk;
    s.dv = (int)dv;
    s.per_key = is_per_key(d) ? 1 : 0;
    s.decay_first = d->gate == LT2_GATE_PER_KEY_DECAY_FIRST ? 1 : 0;
    s.out_bf16 = out_is_bf16(d) ? 1 : 0;
    s.err = err;
    s.qk_norm = f.qk_l2norm;
    s.gate_logits = f.gate_logits;
    s.alpha_scale = f.alpha_scale;
    s.z = f.z ? static_cast<const char*>(f.z) + tau * U * L * dv * sz.esz : nullptr;
    return s;
}

}  // namespace

extern "C" {

size_t lt2_gdr_prefill_workspace_bytes(const lt2_gdr_dims* dims)
{
    Sizes sz;
    if (validate_dims(dims, &sz) != LT2_OK) return 0;
    // the scalar tensor-core prefill's balanced schedule: one flag per unit
    if (dims->gate == LT2_GATE_SCALAR && dims->algo != LT2_ALGO_CUDA_CORE && sz.units > 0 &&
        lt2::prefill_tc_supports(dims->dtype == LT2_DTYPE_BF16, (int)dims->dk, (int)dims->dv, 0))
        return lt2::prefill_tc_flag_bytes(sz.units);
    return 0;
}

lt2_status lt2_gdr_prefill(const lt2_gdr_dims* dims, const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta, const float* S0, void* o,
                           float* S_out, void* workspace, size_t workspace_bytes, void* stream)
{
    return lt2_gdr_prefill_fused(dims, nullptr, q, k, v, alpha, beta, S0, o, S_out, workspace,
                                 workspace_bytes, stream);
}

lt2_status lt2_gdr_prefill_fused(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused, const void* q,
                                 const void* k, const void* v, const float* alpha, const float* beta,
                                 const float* S0, void* o, float* S_out, void* workspace,
                                 size_t workspace_bytes, void* stream)
{
    Sizes sz;
    lt2_status st = validate_dims(dims, &sz);
    if (st != LT2_OK) return st;
    const lt2_gdr_fused f = fused_or_none(fused);
    if (dims->algo == LT2_ALGO_TENSOR_CORE &&
        !lt2::prefill_tc_supports(dims->dtype == LT2_DTYPE_BF16, (int)dims->dk, (int)dims->dv,
                                  is_per_key(dims)))
        return LT2_ERR_UNSUPPORTED;
    if (!tensor_ok(q, sz.qk) || !tensor_ok(k, sz.qk) || !tensor_ok(v, sz.vo) ||
        !tensor_ok(alpha, sz.al) || !tensor_ok(beta, sz.be) || !tensor_ok(o, sz.vo))
        return LT2_ERR_INVALID_ARGUMENT;
    if ((S0 && !aligned16(S0)) || (S_out && !aligned16(S_out))) return LT2_ERR_INVALID_ARGUMENT;
    // The workspace is optional: without it the scalar tensor-core prefill runs one unit per CTA.
    const size_t need = lt2_gdr_prefill_workspace_bytes(dims);
    if (workspace != nullptr && need > 0 && (workspace_bytes < need || !aligned16(workspace)))
        return LT2_ERR_WORKSPACE;
    if (need == 0) workspace = nullptr;
    // Aliasing: o and S_out are written; neither may overlap an input or each other
    // (S_out == S0 exactly is the documented in-place resume); nor may the workspace.
    const Range ro = range_of(o, sz.vo * sz.osz);
    const Range rin[5] = {range_of(q, sz.qk * sz.esz), range_of(k, sz.qk * sz.esz),
                          range_of(v, sz.vo * sz.esz), range_of(alpha, sz.al * 4),
                          range_of(beta, sz.be * 4)};
    for (const Range& r : rin)
        if (overlap(ro, r)) return LT2_ERR_INVALID_ARGUMENT;
    if (S0 && overlap(ro, range_of(S0, sz.st * 4))) return LT2_ERR_INVALID_ARGUMENT;
    if (S_out) {
        const Range rs = range_of(S_out, sz.st * 4);
        if (overlap(rs, ro)) return LT2_ERR_INVALID_ARGUMENT;
        for (const Range& r : rin)
            if (overlap(rs, r)) return LT2_ERR_INVALID_ARGUMENT;
        if (S0 && S0 != S_out && overlap(rs, range_of(S0, sz.st * 4)))
            return LT2_ERR_INVALID_ARGUMENT;
    }
    if (workspace) {
        const Range rw = range_of(workspace, static_cast<int64_t>(need));
        if (overlap(rw, ro) || (S_out && overlap(rw, range_of(S_out, sz.st * 4))) ||
            (S0 && overlap(rw, range_of(S0, sz.st * 4))))
            return LT2_ERR_INVALID_ARGUMENT;
        for (const Range& r : rin)
            if (overlap(rw, r)) return LT2_ERR_INVALID_ARGUMENT;
    }
    st = validate_fused(f, sz, o, S_out);
    if (st != LT2_OK) return st;
    if (sz.units == 0) return LT2_OK;
    st = on_current_device({q, k, v, alpha, beta, S0, o, S_out, workspace, f.z});
    if (st != LT2_OK) return st;

    NvtxRange range("lt2_gdr_prefill");
    unsigned int* err = nullptr;
    st = status_word(&err);
    if (st != LT2_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc = use_tensor_core(dims) && dims->L > 0;
    if (tc) {
        lt2::TcCall call;
        call.q = q;
        call.k = k;
        call.v = v;
        call.alpha = alpha;
        call.beta = beta;
        call.S0 = S0;
        call.o = o;
        call.S_out = S_out;
        call.T = dims->T;
        call.units_per_loop = sz.per_loop;
        call.L = dims->L;
        call.out_bf16 = out_is_bf16(dims) ? 1 : 0;
        call.decay_first = dims->gate == LT2_GATE_PER_KEY_DECAY_FIRST ? 1 : 0;
        call.err = err;
        call.qk_norm = f.qk_l2norm;
        call.gate_logits = f.gate_logits;
        call.alpha_scale = f.alpha_scale;
        call.z = f.z;
        call.workspace = workspace;
        call.workspace_bytes = workspace_bytes;
        cudaError_t e = is_per_key(dims) ? lt2::launch_prefill_kda_tc_all(call, s)
                                         : lt2::launch_prefill_tc_all(call, s);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "prefill (tensor core)");
        return LT2_OK;
    }
    for (int64_t tau = 0; tau < dims->T; ++tau) {
        const lt2::LoopSlice ls = loop_slice(dims, sz, tau, q, k, v, alpha, beta, S0, o, S_out, err, f);
        // Loop 0 waits for all earlier work on the stream; later loops may start as soon as
        // the previous loop's grid is running (the loops share no data).
        const bool pdl = tau > 0;
        NvtxRange loop_range("lt2 prefill loop (cuda core)");
        cudaError_t e = lt2::launch_prefill_seq(ls, dims->dtype == LT2_DTYPE_BF16, s, pdl);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "prefill (cuda core)");
    }
    return LT2_OK;
}

lt2_status lt2_gdr_prefill_varlen(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused, const int64_t* cu_seqlens,
                                  const void* q, const void* k, const void* v, const float* alpha,
                                  const float* beta, const float* S0, void* o, float* S_out, void* workspace,
                                  size_t workspace_bytes, void* stream)
{
    (void)workspace;
    (void)workspace_bytes;
    Sizes sz;
    lt2_status st = validate_varlen_dims(dims, &sz);
    if (st != LT2_OK) return st;
    const lt2_gdr_fused f = fused_or_none(fused);
    const bool tc_ok = lt2::prefill_tc_supports(dims->dtype == LT2_DTYPE_BF16, (int)dims->dk, (int)dims->dv,
                                                is_per_key(dims));
    if (dims->algo == LT2_ALGO_TENSOR_CORE && !tc_ok) return LT2_ERR_UNSUPPORTED;
    if (sz.units == 0) return LT2_OK;
    if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 7u) != 0) return LT2_ERR_INVALID_ARGUMENT;
    if (!tensor_ok(q, sz.qk) || !tensor_ok(k, sz.qk) || !tensor_ok(v, sz.vo) || !tensor_ok(alpha, sz.al) ||
        !tensor_ok(beta, sz.be) || !tensor_ok(o, sz.vo))
        return LT2_ERR_INVALID_ARGUMENT;
    if ((S0 && !aligned16(S0)) || (S_out && !aligned16(S_out))) return LT2_ERR_INVALID_ARGUMENT;
    const Range ro = range_of(o, sz.vo * sz.osz);
    const Range rin[6] = {range_of(q, sz.qk * sz.esz), range_of(k, sz.qk * sz.esz), range_of(v, sz.vo * sz.esz),
                          range_of(alpha, sz.al * 4), range_of(beta, sz.be * 4),
                          range_of(cu_seqlens, (dims->B + 1) * 8)};
    for (const Range& r : rin)
        if (overlap(ro, r)) return LT2_ERR_INVALID_ARGUMENT;
    if (S0 && overlap(ro, range_of(S0, sz.st * 4))) return LT2_ERR_INVALID_ARGUMENT;
    if (S_out) {
        const Range rs = range_of(S_out, sz.st * 4);
        if (overlap(rs, ro)) return LT2_ERR_INVALID_ARGUMENT;
        for (const Range& r : rin)
            if (overlap(rs, r)) return LT2_ERR_INVALID_ARGUMENT;
        if (S0 && S0 != S_out && overlap(rs, range_of(S0, sz.st * 4))) return LT2_ERR_INVALID_ARGUMENT;
    }
    st = validate_fused(f, sz, o, S_out);
    if (st != LT2_OK) return st;
    st = on_current_device({q, k, v, alpha, beta, S0, o, S_out, f.z, cu_seqlens});
    if (st != LT2_OK) return st;

    NvtxRange range("lt2_gdr_prefill_varlen");
    unsigned int* err = nullptr;
    st = status_word(&err);
    if (st != LT2_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tc_ok && dims->algo != LT2_ALGO_CUDA_CORE && dims->L > 0) {
        lt2::TcCall call;
        call.q = q;
        call.k = k;
        call.v = v;
        call.alpha = alpha;
        call.beta = beta;
        call.S0 = S0;
        call.o = o;
        call.S_out = S_out;
        call.T = dims->T;
        call.units_per_loop = sz.per_loop;
        call.L = dims->L;
        call.out_bf16 = out_is_bf16(dims) ? 1 : 0;
        call.decay_first = dims->gate == LT2_GATE_PER_KEY_DECAY_FIRST ? 1 : 0;
        call.err = err;
        call.qk_norm = f.qk_l2norm;
        call.gate_logits = f.gate_logits;
        call.alpha_scale = f.alpha_scale;
        call.z = f.z;
        call.cu_seqlens = cu_seqlens;
        call.H = dims->H;
        cudaError_t e = is_per_key(dims) ? lt2::launch_prefill_kda_tc_all(call, s)
                                         : lt2::launch_prefill_tc_all(call, s);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "prefill varlen (tensor core)");
        return LT2_OK;
    }
    const int64_t rows = dims->H * dims->L;                  // packed token-heads of one loop
    const int64_t na = is_per_key(dims) ? dims->dk : 1;
    for (int64_t tau = 0; tau < dims->T; ++tau) {
        lt2::LoopSlice ls = loop_slice(dims, sz, tau, q, k, v, alpha, beta, S0, o, S_out, err, f);
        ls.q = static_cast<const char*>(q) + tau * rows * dims->dk * sz.esz;
        ls.k = static_cast<const char*>(k) + tau * rows * dims->dk * sz.esz;
        ls.v = static_cast<const char*>(v) + tau * rows * dims->dv * sz.esz;
        ls.alpha = alpha + tau * rows * na;
        ls.beta = beta + tau * rows;
        ls.o = static_cast<char*>(o) + tau * rows * dims->dv * sz.osz;
        ls.z = f.z ? static_cast<const char*>(f.z) + tau * rows * dims->dv * sz.esz : nullptr;
        ls.cu = cu_seqlens;
        ls.H = static_cast<int>(dims->H);
        NvtxRange loop_range("lt2 prefill varlen loop (cuda core)");
        cudaError_t e = lt2::launch_prefill_seq(ls, dims->dtype == LT2_DTYPE_BF16, s, tau > 0);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "prefill varlen (cuda core)");
    }
    return LT2_OK;
}

size_t lt2_gdr_backward_workspace_bytes(const lt2_gdr_dims* dims)
{
    Sizes sz;
    if (validate_dims(dims, &sz) != LT2_OK) return 0;
    return lt2::backward_workspace_bytes(sz.units, dims->L, (int)dims->dk, (int)dims->dv);
}

lt2_status lt2_gdr_backward(const lt2_gdr_dims* dims, const void* q, const void* k, const void* v,
                            const float* alpha, const float* beta, const float* S0, const void* dO,
                            const float* dS_L, float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                            float* dS0, void* workspace, size_t workspace_bytes, void* stream)
{
    Sizes sz;
    lt2_status st = validate_dims(dims, &sz);
    if (st != LT2_OK) return st;
    if (dims->algo == LT2_ALGO_TENSOR_CORE) return LT2_ERR_UNSUPPORTED;
    if (sz.units == 0) return LT2_OK;
    if (!tensor_ok(q, sz.qk) || !tensor_ok(k, sz.qk) || !tensor_ok(v, sz.vo) || !tensor_ok(alpha, sz.al) ||
        !tensor_ok(beta, sz.be) || !tensor_ok(dO, sz.vo) || !tensor_ok(dq, sz.qk) || !tensor_ok(dk, sz.qk) ||
        !tensor_ok(dv, sz.vo) || !tensor_ok(dalpha, sz.al) || !tensor_ok(dbeta, sz.be))
        return LT2_ERR_INVALID_ARGUMENT;
    if ((S0 && !aligned16(S0)) || (dS_L && !aligned16(dS_L)) || (dS0 && !aligned16(dS0)))
        return LT2_ERR_INVALID_ARGUMENT;
    const size_t need = lt2_gdr_backward_workspace_bytes(dims);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return LT2_ERR_WORKSPACE;
    // the gradients are written: none may overlap an input, another gradient or the workspace
    const Range rin[8] = {range_of(q, sz.qk * sz.esz), range_of(k, sz.qk * sz.esz), range_of(v, sz.vo * sz.esz),
                          range_of(alpha, sz.al * 4), range_of(beta, sz.be * 4), range_of(dO, sz.vo * sz.esz),
                          range_of(S0, S0 ? sz.st * 4 : 0), range_of(dS_L, dS_L ? sz.st * 4 : 0)};
    const Range rout[7] = {range_of(dq, sz.qk * 4), range_of(dk, sz.qk * 4), range_of(dv, sz.vo * 4),
                           range_of(dalpha, sz.al * 4), range_of(dbeta, sz.be * 4),
                           range_of(dS0, dS0 ? sz.st * 4 : 0), range_of(workspace, (int64_t)need)};
    for (int a = 0; a < 7; ++a) {
        for (const Range& r : rin)
            if (overlap(rout[a], r)) return LT2_ERR_INVALID_ARGUMENT;
        for (int b = a + 1; b < 7; ++b)
            if (overlap(rout[a], rout[b])) return LT2_ERR_INVALID_ARGUMENT;
    }
    st = on_current_device({q, k, v, alpha, beta, S0, dO, dS_L, dq, dk, dv, dalpha, dbeta, dS0, workspace});
    if (st != LT2_OK) return st;

    NvtxRange range("lt2_gdr_backward");
    lt2::BwCall c;
    c.q = q;
    c.k = k;
    c.v = v;
    c.alpha = alpha;
    c.beta = beta;
    c.S0 = S0;
    c.dO = dO;
    c.dSL = dS_L;
    c.dq = dq;
    c.dk_out = dk;
    c.dv_out = dv;
    c.dalpha = dalpha;
    c.dbeta = dbeta;
    c.dS0 = dS0;
    c.ws = static_cast<float*>(workspace);
    c.units = sz.units;
    c.L = dims->L;
    c.dk = (int)dims->dk;
    c.dv = (int)dims->dv;
    c.per_key = is_per_key(dims) ? 1 : 0;
    c.decay_first = dims->gate == LT2_GATE_PER_KEY_DECAY_FIRST ? 1 : 0;
    c.dtype_bf16 = dims->dtype == LT2_DTYPE_BF16 ? 1 : 0;
    cudaError_t e = lt2::launch_backward(c, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "backward (cuda core)");
    return LT2_OK;
}

lt2_status lt2_gdr_backward_static(const lt2_gdr_dims* dims, const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const float* S0, const void* dO,
                                   const float* dS_L, float* dq, float* dk, float* dv, float* dalpha,
                                   float* dbeta, float* dS0, void* stream)
{
    Sizes sz;
    lt2_status st = validate_dims(dims, &sz);
    if (st != LT2_OK) return st;
    if (sz.units == 0) return lt2_gdr_backward(dims, q, k, v, alpha, beta, S0, dO, dS_L, dq, dk, dv, dalpha,
                                               dbeta, dS0, nullptr, 0, stream);
    const size_t need = lt2_gdr_backward_workspace_bytes(dims);
    if (need > lt2::backward_static_scratch_bytes()) return LT2_ERR_WORKSPACE;
    float* scratch = nullptr;
    const cudaError_t e = lt2::backward_static_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static backward scratch)");
    return lt2_gdr_backward(dims, q, k, v, alpha, beta, S0, dO, dS_L, dq, dk, dv, dalpha, dbeta, dS0, scratch,
                            lt2::backward_static_scratch_bytes(), stream);
}

lt2_status lt2_gdr_decode(const lt2_gdr_dims* dims, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, float* S, void* o, void* stream)
{
    return lt2_gdr_decode_fused(dims, nullptr, q, k, v, alpha, beta, S, o, stream);
}

lt2_status lt2_gdr_decode_fused(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused, const void* q,
                                const void* k, const void* v, const float* alpha, const float* beta,
                                float* S, void* o, void* stream)
{
    Sizes sz;
    lt2_status st = validate_dims(dims, &sz);
    if (st != LT2_OK) return st;
    const lt2_gdr_fused f = fused_or_none(fused);
    if (dims->L != 1) return LT2_ERR_INVALID_ARGUMENT;
    if (!tensor_ok(q, sz.qk) || !tensor_ok(k, sz.qk) || !tensor_ok(v, sz.vo) ||
        !tensor_ok(alpha, sz.al) || !tensor_ok(beta, sz.be) || !tensor_ok(o, sz.vo) ||
        !tensor_ok(S, sz.st))
        return LT2_ERR_INVALID_ARGUMENT;
    const Range ro = range_of(o, sz.vo * sz.osz), rs = range_of(S, sz.st * 4);
    const Range rin[5] = {range_of(q, sz.qk * sz.esz), range_of(k, sz.qk * sz.esz),
                          range_of(v, sz.vo * sz.esz), range_of(alpha, sz.al * 4),
                          range_of(beta, sz.be * 4)};
    if (overlap(ro, rs)) return LT2_ERR_INVALID_ARGUMENT;
    for (const Range& r : rin)
        if (overlap(ro, r) || overlap(rs, r)) return LT2_ERR_INVALID_ARGUMENT;
    st = validate_fused(f, sz, o, S);
    if (st != LT2_OK) return st;
    if (sz.units == 0) return LT2_OK;
    st = on_current_device({q, k, v, alpha, beta, S, o, f.z});
    if (st != LT2_OK) return st;

    NvtxRange range("lt2_gdr_decode");
    unsigned int* err = nullptr;
    st = status_word(&err);
    if (st != LT2_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int64_t tau = 0; tau < dims->T; ++tau) {
        NvtxRange loop_range("lt2 decode loop");
        lt2::LoopSlice ls = loop_slice(dims, sz, tau, q, k, v, alpha, beta, nullptr, o, S, err, f);
        cudaError_t e = lt2::launch_decode(ls, dims->dtype == LT2_DTYPE_BF16, s, tau > 0);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "decode");
    }
    return LT2_OK;
}

lt2_status lt2_swa_prefill(const lt2_swa_dims* d, const void* q, const void* k, const void* v, void* o,
                           void* stream)
{
    if (!d) return LT2_ERR_INVALID_ARGUMENT;
    if (d->T < 0 || d->B < 0 || d->H < 0 || d->L < 0 || d->d < 1 || d->window < 1) return LT2_ERR_INVALID_ARGUMENT;
    if (d->T >= kMaxDim || d->B >= kMaxDim || d->H >= kMaxDim || d->L >= kMaxDim) return LT2_ERR_INVALID_ARGUMENT;
    if (d->dtype != LT2_DTYPE_F32 && d->dtype != LT2_DTYPE_BF16) return LT2_ERR_INVALID_ARGUMENT;
    if (d->algo < LT2_ALGO_AUTO || d->algo > LT2_ALGO_CUDA_CORE) return LT2_ERR_INVALID_ARGUMENT;
    if (d->out_dtype < LT2_OUT_SAME || d->out_dtype > LT2_OUT_BF16) return LT2_ERR_INVALID_ARGUMENT;
    if (!(d->scale >= 0.f && d->scale <= 3.4e38f)) return LT2_ERR_INVALID_ARGUMENT;
    const int bf16 = d->dtype == LT2_DTYPE_BF16 ? 1 : 0;
    const int out_bf16 = d->out_dtype == LT2_OUT_BF16 || (d->out_dtype == LT2_OUT_SAME && bf16) ? 1 : 0;
    if (d->d > 256) return LT2_ERR_UNSUPPORTED;
    const __int128 units = (__int128)d->T * d->B * d->H;
    const __int128 elems = units * d->L * d->d;
    if (elems > ((__int128)1 << 62)) return LT2_ERR_INVALID_ARGUMENT;
    const bool tc_ok = lt2::swa_tc_supports(bf16, (int)d->d);
    if (d->algo == LT2_ALGO_TENSOR_CORE && !tc_ok) return LT2_ERR_UNSUPPORTED;
    const bool tc = tc_ok && d->algo != LT2_ALGO_CUDA_CORE;
    // grid sizes: units x query blocks of 128 (tensor cores) or queries / 4 (CUDA cores) < 2^31
    if (tc ? units * ((d->L + 127) / 128) >= kMaxDim : units * d->L / 4 >= kMaxDim) return LT2_ERR_UNSUPPORTED;
    const int64_t n = (int64_t)elems;
    const int esz = bf16 ? 2 : 4, osz = out_bf16 ? 2 : 4;
    if (!tensor_ok(q, n) || !tensor_ok(k, n) || !tensor_ok(v, n) || !tensor_ok(o, n)) return LT2_ERR_INVALID_ARGUMENT;
    const Range ro = range_of(o, n * osz);
    for (const void* in : {q, k, v})
        if (overlap(ro, range_of(in, n * esz))) return LT2_ERR_INVALID_ARGUMENT;
    if (n == 0) return LT2_OK;
    lt2_status st = on_current_device({q, k, v, o});
    if (st != LT2_OK) return st;

    NvtxRange range("lt2_swa_prefill");
    unsigned int* err = nullptr;
    st = status_word(&err);
    if (st != LT2_OK) return st;
    lt2::SwaCall c;
    c.q = q;
    c.k = k;
    c.v = v;
    c.o = o;
    c.units = (int64_t)units;
    c.L = d->L;
    c.d = d->d;
    c.window = d->window < d->L ? d->window : d->L;
    c.scale = d->scale > 0.f ? d->scale : 1.f / std::sqrt((float)d->d);
    c.dtype_bf16 = bf16;
    c.out_bf16 = out_bf16;
    c.err = err;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = tc ? lt2::launch_swa_tc(c, s) : lt2::launch_swa_cc(c, s);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, tc ? "sliding-window prefill (tensor core)" : "sliding-window prefill (cuda core)");
    return LT2_OK;
}

lt2_status lt2_gdr_last_device_error(void)
{
    unsigned int* p = nullptr;
    lt2_status st = status_word(&p);
    if (st != LT2_OK) return st;
    // Every stream of the device, blocking or not, has finished its work before the word is
    // read; the read and the clear are one atomic exchange on the device, so a flag that a
    // kernel raises concurrently (another thread's work) is never lost, only left for the
    // next call.
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    take_status_kernel<<<1, 1, 0, 0>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "take device status");
    unsigned int h = 0;
    e = cudaMemcpy(&h, p + 1, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read device status");
    if (h & lt2::kDevTimeout) return LT2_ERR_DEVICE_TIMEOUT;
    if (h & lt2::kDevSeqlens) return LT2_ERR_SEQLENS;
    if (h & lt2::kDevRange) return LT2_ERR_RANGE;
    if (h & lt2::kDevCheck) return LT2_ERR_DEVICE_CHECK;
    return LT2_OK;
}

const char* lt2_status_string(lt2_status s)
{
    switch (s) {
        case LT2_OK: return "LT2_OK";
        case LT2_ERR_INVALID_ARGUMENT: return "LT2_ERR_INVALID_ARGUMENT";
        case LT2_ERR_UNSUPPORTED: return "LT2_ERR_UNSUPPORTED";
        case LT2_ERR_WORKSPACE: return "LT2_ERR_WORKSPACE";
        case LT2_ERR_CUDA: return "LT2_ERR_CUDA";
        case LT2_ERR_DEVICE_TIMEOUT: return "LT2_ERR_DEVICE_TIMEOUT";
        case LT2_ERR_RANGE: return "LT2_ERR_RANGE";
        case LT2_ERR_DEVICE_CHECK: return "LT2_ERR_DEVICE_CHECK";
        case LT2_ERR_SEQLENS: return "LT2_ERR_SEQLENS";
    }
    return "LT2_STATUS_UNKNOWN";
}

const char* lt2_last_cuda_error_string(void) { return t_cuda_error; }

int lt2_gdr_version(void) { return 220; }

}  // extern "C"

#ifdef LT2_DEBUG
#include "lt2_gdr_debug.h"
#include "gdr_tc_common.cuh"

extern "C" {

lt2_status lt2_debug_set_skip_chunk(int kernel, int chunk)
{
    if (chunk < -1) return LT2_ERR_INVALID_ARGUMENT;
    cudaError_t e;
    if (kernel == LT2_DEBUG_SCALAR_TC)
        e = lt2::debug_set_skip_chunk_scalar(chunk);
    else if (kernel == LT2_DEBUG_PER_KEY_TC)
        e = lt2::debug_set_skip_chunk_per_key(chunk);
    else
        return LT2_ERR_INVALID_ARGUMENT;
    return e == cudaSuccess ? LT2_OK : cuda_fail(e, "lt2_debug_set_skip_chunk");
}

uint64_t lt2_debug_wait_timeout_ns(void) { return lt2::tcc::kWaitTimeoutNs; }

}  // extern "C"
#endif
