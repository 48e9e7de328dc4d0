// gdr_prefill_seq.cu -- token-sequential prefill on CUDA cores, fp32 arithmetic.
//
// The displayed equation of "LT2 transformer looped a tempo lineare" (section "Sostituire
// il motore") applied token after token, exactly as written, with the state held in
// registers:
//
//   e_t = k_t^T S,  f_t = (alpha_t . q_t)^T S                  (one pass over S)
//   S  <- Diag(alpha_t) (S - beta_t k_t e_t) + beta_t k_t v_t^T
//   o_t = f_t - beta_t ((alpha_t . q_t) . k_t) e_t + beta_t (q_t . k_t) v_t   (= S_t^T q_t)
//
// With per-key gating in the decay-first order, A_t = (I - beta_t k_t k_t^T) Diag(alpha_t):
//
//   e_t = (alpha_t . k_t)^T S,  f_t = (alpha_t . q_t)^T S
//   S  <- Diag(alpha_t) S - beta_t k_t e_t + beta_t k_t v_t^T
//   o_t = f_t - beta_t (q_t . k_t) e_t + beta_t (q_t . k_t) v_t
//
// The fused prologue and output gate (lt2_gdr_fused) run here too: q and k rows normalised to
// unit L2 norm, alpha = exp(-softplus(a) c) and beta = sigmoid(b) from logits when the tile is
// staged, and o_t <- sigmoid(z_t) o_t when it is written.
//
// This path serves fp32 inputs (where bf16 tensor cores cannot meet a 1e-4 tolerance) and
// every shape the tensor-core kernel does not cover.  Columns of S evolve independently
// (A_t acts from the left), so the grid is (head-unit, 32-column slice of d_v).  Inside a
// CTA, warp w owns dk/8 contiguous rows and lane c one column; per token, the two column
// sums are combined across warps through a double-buffered shared array, so one barrier
// per token suffices.  Inputs are staged in shared memory 16 tokens at a time.
#include "gdr_common.cuh"
#include "gdr_launch.h"

namespace lt2 {

namespace {
constexpr int kTile = 16;    // tokens staged per round
constexpr int kCols = 32;    // d_v columns per CTA
}

template <typename T, typename To>
__global__ void __launch_bounds__(256) gdr_prefill_seq_kernel(LoopSlice p, int use_pdl)
{
    (void)use_pdl;
    allow_next_loop_to_start();

    extern __shared__ __align__(16) float smem[];
    const int dk = p.dk, dv = p.dv;
    const int rpw = dk >> 3;
    const int w = threadIdx.x >> 5, c = threadIdx.x & 31;
    const int j0 = blockIdx.y * kCols;
    const int ncol = min(kCols, dv - j0);
    const bool active = c < ncol;
    const int64_t u = blockIdx.x;
    const int na = p.per_key ? dk : 1;

    float* sk = smem;                              // [kTile][dk]
    float* saq = sk + kTile * dk;                  // [kTile][dk]   alpha . q
    float* sa = saq + kTile * dk;                  // [kTile][na]
    float* sv = sa + kTile * na;                   // [kTile][kCols]
    float* sb = sv + kTile * kCols;                // [kTile]  beta
    float* sqk = sb + kTile;                       // [kTile]  q.k
    float* saqk = sqk + kTile;                     // [kTile]  (alpha.q).k
    float* red = saqk + kTile;                     // [2][2][8][kCols]

    // the unit's first row and length: its own L rows, or a packed sequence's tokens
    int64_t row0 = u * p.L, Lu = p.L;
    if (p.cu) {
        const int64_t b = u / p.H, h = u - b * p.H;
        const int64_t c0 = p.cu[b], c1 = p.cu[b + 1];
        if (!(0 <= c0 && c0 <= c1 && c1 <= p.L)) {
            if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(p.err, kDevSeqlens);
            return;
        }
        row0 = h * p.L + c0;
        Lu = c1 - c0;
    }
    const T* q = static_cast<const T*>(p.q) + row0 * dk;
    const T* k = static_cast<const T*>(p.k) + row0 * dk;
    const T* v = static_cast<const T*>(p.v) + row0 * dv;
    const float* al = p.alpha + row0 * na;
    const float* be = p.beta + row0;
    To* o = static_cast<To*>(p.o) + row0 * dv;

    const int r0 = w * rpw;
    float s[16];
    const float* S0 = p.S0 ? p.S0 + u * (int64_t)dk * dv : nullptr;
    #pragma unroll
    for (int m = 0; m < 16; ++m)
        s[m] = (m < rpw && active && S0) ? S0[(int64_t)(r0 + m) * dv + j0 + c] : 0.f;

    int buf = 0;
    for (int64_t t0 = 0; t0 < Lu; t0 += kTile) {
        const int nt = (Lu - t0 < kTile) ? (int)(Lu - t0) : kTile;
        __syncthreads();   // previous tile fully consumed
        // k, q (raw), alpha and beta of the tile; with gate logits, alpha = exp(-softplus(a) c)
        // and beta = sigmoid(b) (the fused prologue)
        for (int idx = threadIdx.x; idx < nt * dk; idx += blockDim.x) {
            const int tt = idx / dk, i = idx - tt * dk;
            const int64_t g = (t0 + tt) * dk + i;
            sk[tt * dk + i] = to_f32(k[g]);
            saq[tt * dk + i] = to_f32(q[g]);
            if (p.per_key) sa[tt * dk + i] = p.gate_logits ? alpha_from_logit(al[g], p.alpha_scale) : al[g];
        }
        for (int idx = threadIdx.x; idx < nt * kCols; idx += blockDim.x) {
            const int tt = idx / kCols, j = idx - tt * kCols;
            sv[idx] = (j < ncol) ? to_f32(v[(t0 + tt) * dv + j0 + j]) : 0.f;
        }
        if (threadIdx.x < nt) {
            const float b = be[t0 + threadIdx.x];
            sb[threadIdx.x] = p.gate_logits ? sigmoid_f32(b) : b;
            if (!p.per_key) {
                const float a = al[t0 + threadIdx.x];
                sa[threadIdx.x] = p.gate_logits ? alpha_from_logit(a, p.alpha_scale) : a;
            }
        }
        __syncthreads();
        // per token, one warp over the channels: the fused L2 normalisation of q and k, then
        // q.k, alpha . q and (alpha.q).k
        for (int tt = w; tt < nt; tt += 8) {
            float* kt = sk + tt * dk;
            float* qt = saq + tt * dk;
            if (p.qk_norm) {
                float nq = 0.f, nk = 0.f;
                for (int i = c; i < dk; i += 32) {
                    nq += qt[i] * qt[i];
                    nk += kt[i] * kt[i];
                }
                #pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    nq += __shfl_xor_sync(0xffffffffu, nq, off);
                    nk += __shfl_xor_sync(0xffffffffu, nk, off);
                }
                const float iq = inv_l2(nq), ik = inv_l2(nk);
                for (int i = c; i < dk; i += 32) {
                    qt[i] *= iq;
                    kt[i] *= ik;
                }
            }
            float a = 0.f, b = 0.f;
            for (int i = c; i < dk; i += 32) {
                const float al_i = p.per_key ? sa[tt * dk + i] : sa[tt];
                const float kq = qt[i] * kt[i];
                qt[i] *= al_i;
                a += kq;
                b += qt[i] * kt[i];
            }
            #pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, off);
                b += __shfl_xor_sync(0xffffffffu, b, off);
            }
            if (c == 0) { sqk[tt] = a; saqk[tt] = b; }
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            const float* kr = sk + tt * dk + r0;
            const float* qr = saq + tt * dk + r0;
            float e = 0.f, f = 0.f;
            #pragma unroll
            for (int m = 0; m < 16; ++m) {
                if (m < rpw) {
                    const float ke = p.decay_first ? kr[m] * sa[tt * dk + r0 + m] : kr[m];
                    e += ke * s[m];
                    f += qr[m] * s[m];
                }
            }
            float* rb = red + buf * (2 * 8 * kCols);
            rb[w * kCols + c] = e;
            rb[8 * kCols + w * kCols + c] = f;
            __syncthreads();
            float E = 0.f, F = 0.f;
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                E += rb[i * kCols + c];
                F += rb[8 * kCols + i * kCols + c];
            }
            buf ^= 1;
            const float bt = sb[tt];
            const float vc = sv[tt * kCols + c];
            #pragma unroll
            for (int m = 0; m < 16; ++m) {
                if (m < rpw) {
                    const float a = p.per_key ? sa[tt * dk + r0 + m] : sa[tt];
                    const float bk = bt * kr[m];
                    s[m] = p.decay_first ? a * s[m] - bk * E + bk * vc : a * (s[m] - bk * E) + bk * vc;
                }
            }
            const float qke = p.decay_first ? sqk[tt] : saqk[tt];
            if (w == 0 && active) {
                float ov = F - bt * qke * E + bt * sqk[tt] * vc;
                if (p.z)        // the fused output gate
                    ov *= sigmoid_f32(to_f32(static_cast<const T*>(p.z)[(row0 + t0 + tt) * dv + j0 + c]));
                o[(t0 + tt) * dv + j0 + c] = from_f32<To>(ov);
            }
        }
    }

    if (p.S_out && active) {
        float* So = p.S_out + u * (int64_t)dk * dv;
        #pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m < rpw) So[(int64_t)(r0 + m) * dv + j0 + c] = s[m];
    }
}

static size_t seq_smem_bytes(int dk, int per_key)
{
    const int na = per_key ? dk : 1;
    return sizeof(float) * (size_t)(2 * kTile * dk + kTile * na + kTile * kCols + 3 * kTile +
                                    2 * 2 * 8 * kCols);
}

template <typename T, typename To>
static cudaError_t launch_typed(const cudaLaunchConfig_t& cfg, const LoopSlice& s, int use_pdl)
{
    cudaError_t e = cudaFuncSetAttribute(gdr_prefill_seq_kernel<T, To>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, gdr_prefill_seq_kernel<T, To>, s, use_pdl);
}

cudaError_t launch_prefill_seq(const LoopSlice& s, int dtype_bf16, cudaStream_t stream, bool pdl)
{
    if (s.units == 0) return cudaSuccess;
    const size_t smem = seq_smem_bytes(s.dk, s.per_key);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)s.units, (unsigned)((s.dv + kCols - 1) / kCols), 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int use_pdl = pdl ? 1 : 0;
    using bf = __nv_bfloat16;
    if (dtype_bf16) {
        if (s.out_bf16) return launch_typed<bf, bf>(cfg, s, use_pdl);
        return launch_typed<bf, float>(cfg, s, use_pdl);
    }
    if (s.out_bf16) return launch_typed<float, bf>(cfg, s, use_pdl);
    return launch_typed<float, float>(cfg, s, use_pdl);
}

}  // namespace lt2
