// gdr_decode.cu -- one decode token of the gated delta rule per (loop, batch, head).
//
// "LT2 transformer looped a tempo lineare", section "Sostituire il motore", displayed
// equation, applied to a single token with the state read from and written back to HBM:
//
//   e   = k^T S                                   (d_v row vector)
//   S'  = Diag(alpha) (S - beta k e) + beta k v^T
//   o   = S'^T q = S^T (alpha . q) - beta ((alpha . q) . k) e + beta (q . k) v
//
// The last line is the same readout rearranged so that both column reductions (k^T S and
// (alpha.q)^T S) come from ONE read of S: each state is streamed through HBM exactly once
// (64 KiB read + 64 KiB written for d = 128), which is the whole cost of the step.
//
// Per-key gating in the decay-first order, A = (I - beta k k^T) Diag(alpha):
//
//   e   = (alpha . k)^T S,   S' = Diag(alpha) S - beta k e + beta k v^T
//   o   = S^T (alpha . q) - beta (q . k) e + beta (q . k) v
//
// Mapping: one CTA of 256 threads per head-unit.  Warp w owns the contiguous rows
// [w*dk/8, (w+1)*dk/8); lane c owns columns 4c..4c+3 (one 16-byte access per row), so
// every warp-wide access touches whole 128-byte lines; a thread issues its state loads before it
// reads the token's vectors, so the two latencies overlap.  The per-column partial sums are
// combined across the 8 warps through shared memory; the update is applied in registers
// and written back with streaming stores.  The fused prologue (q, k normalised to unit L2
// norm; alpha, beta from logits) and output gate (o <- sigmoid(z) o) have their own instances.
#include "gdr_common.cuh"
#include "gdr_launch.h"

namespace lt2 {

// kFused: the instance with the fused prologue and output gate (lt2_gdr_fused); the plain
// instances compile exactly as without them.
template <typename T, typename To, bool kDecayFirst, bool kFused>
__global__ void __launch_bounds__(256, 2) gdr_decode_kernel(LoopSlice p, int use_pdl)
{
    (void)use_pdl;
    allow_next_loop_to_start();

    __shared__ __align__(16) float sk[128];
    __shared__ __align__(16) float saq[128];
    __shared__ __align__(16) float sa[128];
    __shared__ __align__(16) float sv[128];
    __shared__ __align__(16) float red_e[8][128];
    __shared__ __align__(16) float red_f[8][128];
    __shared__ float s_qk, s_aqk;

    const int64_t u = blockIdx.x;
    const int dk = p.dk, dv = p.dv;
    const int rpw = dk >> 3;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // The state first: its loads (16 per thread) are in flight while the token's vectors are read
    // and reduced, instead of after them.
    float* S = p.S_out + u * (int64_t)dk * dv;
    const bool active = lane * 4 < dv;
    const int col = lane * 4;
    const int r0 = w * rpw;
    float4 s[16];
    #pragma unroll
    for (int m = 0; m < 16; ++m)
        if (m < rpw && active) s[m] = ld_stream_f4(S + (int64_t)(r0 + m) * dv + col);

    const T* q = static_cast<const T*>(p.q) + u * dk;
    const T* k = static_cast<const T*>(p.k) + u * dk;
    const T* v = static_cast<const T*>(p.v) + u * dv;
    float beta = p.beta[u];
    float a_scalar = p.per_key ? 0.f : p.alpha[u];
    float iq = 1.f, ik = 1.f;          // inverse L2 norms of q and k (fused prologue)
    if (kFused) {
        if (p.gate_logits) {
            beta = sigmoid_f32(beta);
            if (!p.per_key) a_scalar = alpha_from_logit(a_scalar, p.alpha_scale);
        }
        if (p.qk_norm) {
            float nq = 0.f, nk = 0.f;
            for (int i = threadIdx.x; i < dk; i += blockDim.x) {
                const float qi = to_f32(q[i]), ki = to_f32(k[i]);
                nq += qi * qi;
                nk += ki * ki;
            }
            #pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
            }
            if (lane == 0) {
                red_e[1][w] = nq;
                red_f[1][w] = nk;
            }
            __syncthreads();
            nq = 0.f;
            nk = 0.f;
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                nq += red_e[1][i];
                nk += red_f[1][i];
            }
            iq = inv_l2(nq);
            ik = inv_l2(nk);
        }
    }

    float qk_part = 0.f, aqk_part = 0.f;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        float a = p.per_key ? p.alpha[u * dk + i] : a_scalar;
        if (kFused && p.per_key && p.gate_logits) a = alpha_from_logit(a, p.alpha_scale);
        const float qi = kFused ? to_f32(q[i]) * iq : to_f32(q[i]);
        const float ki = kFused ? to_f32(k[i]) * ik : to_f32(k[i]);
        sk[i] = ki;
        sa[i] = a;
        saq[i] = a * qi;
        qk_part += qi * ki;
        aqk_part += a * qi * ki;
    }
    for (int j = threadIdx.x; j < dv; j += blockDim.x) sv[j] = to_f32(v[j]);
    // q.k and (alpha.q).k: dk <= 128 < blockDim, so every thread holds at most one term;
    // reduce within each warp, then across the 8 warps (red_e/red_f rows reused as scratch).
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        qk_part += __shfl_xor_sync(0xffffffffu, qk_part, off);
        aqk_part += __shfl_xor_sync(0xffffffffu, aqk_part, off);
    }
    if (lane == 0) {
        red_e[0][w] = qk_part;
        red_f[0][w] = aqk_part;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.f, b = 0.f;
        for (int i = 0; i < 8; ++i) { a += red_e[0][i]; b += red_f[0][i]; }
        s_qk = a;
        s_aqk = b;
    }
    __syncthreads();

    float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    #pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < rpw && active) {
            const int r = r0 + m;
            const float kr = kDecayFirst ? sk[r] * sa[r] : sk[r], ar = saq[r];
            e.x += kr * s[m].x; e.y += kr * s[m].y; e.z += kr * s[m].z; e.w += kr * s[m].w;
            f.x += ar * s[m].x; f.y += ar * s[m].y; f.z += ar * s[m].z; f.w += ar * s[m].w;
        }
    }
    if (active) {
        *reinterpret_cast<float4*>(&red_e[w][col]) = e;
        *reinterpret_cast<float4*>(&red_f[w][col]) = f;
    }
    __syncthreads();
    if (!active) return;

    float4 E = make_float4(0.f, 0.f, 0.f, 0.f), F = E;
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 a = *reinterpret_cast<const float4*>(&red_e[i][col]);
        const float4 b = *reinterpret_cast<const float4*>(&red_f[i][col]);
        E.x += a.x; E.y += a.y; E.z += a.z; E.w += a.w;
        F.x += b.x; F.y += b.y; F.z += b.z; F.w += b.w;
    }
    const float4 vv = *reinterpret_cast<const float4*>(&sv[col]);

    #pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < rpw) {
            const int r = r0 + m;
            const float bk = beta * sk[r];
            const float ar = sa[r];
            float4 n;
            if (kDecayFirst) {
                n.x = ar * s[m].x + bk * (vv.x - E.x);
                n.y = ar * s[m].y + bk * (vv.y - E.y);
                n.z = ar * s[m].z + bk * (vv.z - E.z);
                n.w = ar * s[m].w + bk * (vv.w - E.w);
            } else {
                n.x = ar * (s[m].x - bk * E.x) + bk * vv.x;
                n.y = ar * (s[m].y - bk * E.y) + bk * vv.y;
                n.z = ar * (s[m].z - bk * E.z) + bk * vv.z;
                n.w = ar * (s[m].w - bk * E.w) + bk * vv.w;
            }
            st_stream_f4(S + (int64_t)r * dv + col, n);
        }
    }

    if (w == 0) {
        const float c1 = beta * (kDecayFirst ? s_qk : s_aqk), c2 = beta * s_qk;
        To* o = static_cast<To*>(p.o) + u * dv + col;
        float4 ov = make_float4(F.x - c1 * E.x + c2 * vv.x, F.y - c1 * E.y + c2 * vv.y,
                                F.z - c1 * E.z + c2 * vv.z, F.w - c1 * E.w + c2 * vv.w);
        if (kFused && p.z) {            // the fused output gate
            const T* z = static_cast<const T*>(p.z) + u * dv + col;
            ov.x *= sigmoid_f32(to_f32(z[0]));
            ov.y *= sigmoid_f32(to_f32(z[1]));
            ov.z *= sigmoid_f32(to_f32(z[2]));
            ov.w *= sigmoid_f32(to_f32(z[3]));
        }
        o[0] = from_f32<To>(ov.x);
        o[1] = from_f32<To>(ov.y);
        o[2] = from_f32<To>(ov.z);
        o[3] = from_f32<To>(ov.w);
    }
}

template <bool kDecayFirst, bool kFused>
static cudaError_t launch_decode_typed(const cudaLaunchConfig_t& cfg, const LoopSlice& s, int dtype_bf16,
                                       int use_pdl)
{
    using bf = __nv_bfloat16;
    if (dtype_bf16) {
        if (s.out_bf16) return cudaLaunchKernelEx(&cfg, gdr_decode_kernel<bf, bf, kDecayFirst, kFused>, s, use_pdl);
        return cudaLaunchKernelEx(&cfg, gdr_decode_kernel<bf, float, kDecayFirst, kFused>, s, use_pdl);
    }
    if (s.out_bf16) return cudaLaunchKernelEx(&cfg, gdr_decode_kernel<float, bf, kDecayFirst, kFused>, s, use_pdl);
    return cudaLaunchKernelEx(&cfg, gdr_decode_kernel<float, float, kDecayFirst, kFused>, s, use_pdl);
}

cudaError_t launch_decode(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl)
{
    if (s.units == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)s.units, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int use_pdl = pdl ? 1 : 0;
    // one instance per input type, output type, order of the per-key factors and fusion
    const bool fused = s.qk_norm || s.gate_logits || s.z;
    if (s.decay_first)
        return fused ? launch_decode_typed<true, true>(cfg, s, dtype_bf16, use_pdl)
                     : launch_decode_typed<true, false>(cfg, s, dtype_bf16, use_pdl);
    return fused ? launch_decode_typed<false, true>(cfg, s, dtype_bf16, use_pdl)
                 : launch_decode_typed<false, false>(cfg, s, dtype_bf16, use_pdl);
}

}  // namespace lt2
