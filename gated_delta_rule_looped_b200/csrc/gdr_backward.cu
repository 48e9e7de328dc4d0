// gdr_backward.cu -- backward pass of the looped gated delta rule on CUDA cores (fp32).
//
// The forward recurrence ("LT2 transformer looped a tempo lineare", section "Sostituire il
// motore", displayed equation), per (loop, batch, head) unit and token t:
//     printed order:      e = S_{t-1}^T k,  P = S_{t-1} - beta k e^T,  S_t = Diag(alpha) P + beta k v^T
//     decay-first order:  R = Diag(alpha) S_{t-1},  e = R^T k,  S_t = R - beta k e^T + beta k v^T
//     o_t = S_t^T q_t
// The pages train looped models but give no training kernel; this is the plain reverse-mode
// derivative of the recurrence.  For upstream gradients dO_t and dS_L, a sweep from t = L down to
// 1 carries G = dLoss/dS_t:
//     G += q_t dO_t^T;  dq_t = S_t dO_t
//     printed:      dP = Diag(alpha) G;  dv = beta G^T k;  dbeta = (G^T k).v - (dP^T k).e
//                   dk = beta G v - beta (S_{t-1} (dP^T k) + dP e);  dalpha = rowsum(G * P)
//                   G <- dP - beta k (dP^T k)^T
//     decay-first:  kG = G^T k;  dR = G - beta k kG^T;  dv = beta kG;  dbeta = kG.(v - e)
//                   dk = beta G (v - e) - beta R kG;  dalpha = rowsum(dR * S_{t-1});  G <- Diag(alpha) dR
// and dS_0 = G at the end (scalar alpha: dalpha sums over the rows too).
//
// The columns of S evolve independently given the token's k, alpha, beta (e_j only reads column
// j), so a block takes one unit and a slice of 32 columns of d_v, and each warp four whole columns
// of it: lane 4 g + c holds rows g*dk/8 .. (g+1)*dk/8 - 1 of column j0 + 4 w + c.  Every column sum
// a step needs (k^T S_{t-1} or k^T R, k^T G, k^T Diag(alpha) G) is then a sum over the 8 row groups
// of one warp -- three shuffles, no block barrier -- and the warps run their columns' recurrences
// independently.  The reverse sweep needs S_{t-1} and S_t at every t, newest first:
//   phase A  runs the forward over the whole sequence and keeps the state at the start of every
//            32-token chunk (a checkpoint) in the workspace;
//   phase B  takes the chunks from the last: it recomputes the chunk's states from its checkpoint
//            into the workspace, then sweeps the chunk backwards.
// The workspace is thread-major (element m of thread i of a state at [m / 4][i][m % 4] when the
// rows move as float4, else at [m][i]): each thread reads back only what it wrote, in coalesced
// rows.  A chunk's inputs are staged in shared memory once
// per phase; the sweep reuses S_{t-1} of token t+1 as S_t of token t and loads the next S_{t-1}
// one token ahead.  The row sums (dq, dk and the per-key dalpha: sums over the slice's 32
// columns) are summed over a warp's 4 columns with shuffles, parked per warp in shared memory, and
// every few tokens added over the 8 warps and into the fp32 outputs with atomics (zeroed first by
// this library), as are the dbeta and scalar dalpha terms.  dv and dS_0 belong to one block each
// and are stored directly.  The kernel is instantiated per input type, order and gating, with
// d_k = 128 fixed at compile time (the rows of a thread then move as float4; any other d_k is read
// at run time), so no per-element branch stays in the token loops.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "gdr_common.cuh"
#include "gdr_launch.h"
#include "gdr_nvtx.h"

namespace lt2 {
namespace bw {

constexpr int kCols = 32;          // columns of d_v per block
constexpr int kThreads = 256;      // 8 warps, 4 columns each
constexpr int kChunk = 32;         // tokens between checkpoints, staged in shared memory at once
constexpr int kMaxRows = 16;       // dk / 8 rows per thread, dk <= 128

// Tokens whose row-sum partials wait in shared memory before they are added up and written
// (fewer with a per-key alpha, which adds a third row sum).
__host__ __device__ constexpr int flush_tokens(bool per_key) { return per_key ? 4 : 8; }
// Floats per warp row of the row-sum partials: d_k plus one pad per 32 rows (no bank conflicts)
__host__ __device__ constexpr int part_stride(int dk) { return dk + 4; }

__device__ __forceinline__ float warp_sum(float x)
{
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// A column sum over all d_k rows: the 8 row groups of a column are lanes c, c + 4, ..., c + 28.
__device__ __forceinline__ float sum_row_groups(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 16);
    return x;
}

// Row sums over a warp's 4 columns (lanes 4 g .. 4 g + 3) of 16 values per lane at once, by
// recursive halving (12 shuffles instead of 16 x 2).  On return v[i], i < 4, holds the sum of row
// (c & 1) * 8 + (c & 2) * 2 + i of the thread's rows, c = lane & 3.
__device__ __forceinline__ void sum_cols4(float (&v)[kMaxRows], int c)
{
    #pragma unroll
    for (int half = 8, off = 1; half >= 4; half >>= 1, off <<= 1) {
        const bool upper = (c & off) != 0;
        #pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
}

struct Params {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
    const float* S0;       // nullable
    const void* dO;
    const float* dSL;      // nullable
    float* dq;             // [units][L][dk], accumulated (zeroed first)
    float* gdk;            // dk, accumulated
    float* gdv;            // dv [units][L][dv], stored
    float* dalpha;         // [units][L] or [units][L][dk], accumulated
    float* dbeta;          // [units][L], accumulated
    float* dS0;            // nullable, stored
    float* ws;             // per block: checkpoints, then the states of one chunk
    int64_t units;
    int64_t L;
    int dk;
    int dv;
    int per_key;
    int decay_first;
};

// Workspace floats per block: ceil(L / 32) checkpoints and the 33 states of one chunk, dk x 32 each.
__host__ __device__ inline int64_t ws_floats_per_block(int64_t L, int dk)
{
    return ((L + kChunk - 1) / kChunk + kChunk + 1) * static_cast<int64_t>(dk) * kCols;
}

// Shared memory of a block: one chunk's inputs in fp32 (k, q, alpha rows, beta, and the slice's v
// and dO columns), the row-sum partials [dq, dk(, dalpha)][token][warp][row], the per-warp
// dbeta and scalar dalpha terms [token][warp], and the column sums e of the chunk's tokens
// [token][column] (about 111 KB with d_k = 128: two blocks per SM).
__host__ __device__ inline size_t smem_bytes(int dk, int per_key)
{
    const size_t na = per_key ? dk : 1;
    const size_t f = flush_tokens(per_key != 0), ng = per_key ? 3 : 2;
    return (static_cast<size_t>(kChunk) * (2 * dk + na + 1 + 3 * kCols) + ng * f * 8 * part_stride(dk) + 2 * f * 8) *
           sizeof(float);
}

// 8 consecutive elements of a row (16-byte aligned) into shared memory as fp32, in two halves:
// a thread issues all its loads before it stores any of them.
template <typename T> struct Raw8;
template <> struct Raw8<float> { float4 a, b; };
template <> struct Raw8<__nv_bfloat16> { uint4 a; };
__device__ __forceinline__ Raw8<float> raw8_load(const float* src)
{
    return Raw8<float>{__ldg(reinterpret_cast<const float4*>(src)), __ldg(reinterpret_cast<const float4*>(src) + 1)};
}
__device__ __forceinline__ Raw8<__nv_bfloat16> raw8_load(const __nv_bfloat16* src)
{
    return Raw8<__nv_bfloat16>{__ldg(reinterpret_cast<const uint4*>(src))};
}
__device__ __forceinline__ void raw8_store(const Raw8<float>& r, float* dst)
{
    reinterpret_cast<float4*>(dst)[0] = r.a;
    reinterpret_cast<float4*>(dst)[1] = r.b;
}
__device__ __forceinline__ void raw8_store(const Raw8<__nv_bfloat16>& r, float* dst)
{
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.a);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
    reinterpret_cast<float4*>(dst)[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
    reinterpret_cast<float4*>(dst)[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
}
__device__ __forceinline__ void zero8(float* dst)
{
    reinterpret_cast<float4*>(dst)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(dst)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// This thread's rows of one shared-memory row vector: with kRpw a multiple of 4 (d_k = 32, 64,
// 96, 128) the rows r0 .. r0 + kRpw - 1 are 16-byte aligned and move as float4; otherwise one by one.
template <int kRpw>
__device__ __forceinline__ void lds_rows(const float* src, float (&dst)[kMaxRows], int rpw)
{
    if constexpr (kRpw > 0 && kRpw % 4 == 0) {
        #pragma unroll
        for (int m = 0; m < kRpw; m += 4) {
            const float4 x = *reinterpret_cast<const float4*>(src + m);
            dst[m] = x.x;
            dst[m + 1] = x.y;
            dst[m + 2] = x.z;
            dst[m + 3] = x.w;
        }
        #pragma unroll
        for (int m = kRpw; m < kMaxRows; ++m) dst[m] = 0.f;
    } else {
        #pragma unroll
        for (int m = 0; m < kMaxRows; ++m) dst[m] = m < rpw ? src[m] : 0.f;
    }
}

// One block = one unit and one 32-column slice of d_v.  kRpw = d_k / 8 when the launch knows it
// (16: d_k = 128), 0 for any d_k (a multiple of 8, <= 128) read at run time; kDF: decay-first
// order; kPK: per-key alpha.
template <typename T, int kRpw, bool kDF, bool kPK>
__global__ void __launch_bounds__(kThreads, 2) gdr_backward_kernel(Params p)
{
    constexpr int kF = flush_tokens(kPK);
    constexpr int kNg = kPK ? 3 : 2;               // row sums: dq, dk (and the per-key dalpha)
    extern __shared__ __align__(16) float smem[];
    const int dk = kRpw > 0 ? 8 * kRpw : p.dk, dv = p.dv, rpw = kRpw > 0 ? kRpw : dk >> 3;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, cg = lane & 3;
    const int j0 = blockIdx.y * kCols;
    const int jl = 4 * w + cg, j = j0 + jl;        // this thread's column (in the slice, in d_v)
    const bool active = j < dv;
    const int64_t u = blockIdx.x, L = p.L;
    const int r0 = g * rpw;                        // first of this thread's rows
    const int na = kPK ? dk : 1;
    const int ps = part_stride(dk);
    float* sk = smem;                              // [32][dk]
    float* sq = sk + kChunk * dk;                  // [32][dk]
    float* sa = sq + kChunk * dk;                  // [32][na]
    float* sbe = sa + kChunk * na;                 // [32]
    float* sv = sbe + kChunk;                      // [32][32]
    float* sdo = sv + kChunk * kCols;              // [32][32]
    float* part = sdo + kChunk * kCols;            // [kNg][kF][8][ps]
    float* pbe = part + kNg * kF * 8 * ps;         // [kF][8]
    float* pal = pbe + kF * 8;                     // [kF][8] (scalar alpha)
    float* se = pal + kF * 8;                      // [32][32] e of the chunk's tokens, from the recompute

    const T* q = static_cast<const T*>(p.q) + u * L * dk;
    const T* k = static_cast<const T*>(p.k) + u * L * dk;
    const T* v = static_cast<const T*>(p.v) + u * L * dv;
    const T* dO = static_cast<const T*>(p.dO) + u * L * dv;
    const float* al = p.alpha + u * L * na;
    const float* be = p.beta + u * L;
    const int nck = static_cast<int>((L + kChunk - 1) / kChunk);
    // A state in the workspace takes rpw * 256 floats.  Element m of thread i sits at [m][i], or,
    // when the rows move as float4 (kRpw a multiple of 4), at [m / 4][i][m % 4]; either way at
    // base + m * 256 from the thread's own base, for m a multiple of 4 in the second layout.
    constexpr bool kVec = kRpw > 0 && kRpw % 4 == 0;
    const int64_t sst = static_cast<int64_t>(rpw) * kThreads;
    float* ck = p.ws + (u * gridDim.y + blockIdx.y) * ws_floats_per_block(L, dk) + (kVec ? 4 * tid : tid);
    float* st = ck + nck * sst;                    // [33] states of the chunk being swept
    auto ws_store = [&](float* dst, const float (&x)[kMaxRows]) {
        if constexpr (kVec) {
            #pragma unroll
            for (int m = 0; m < kRpw; m += 4)
                *reinterpret_cast<float4*>(dst + m * kThreads) = make_float4(x[m], x[m + 1], x[m + 2], x[m + 3]);
        } else {
            #pragma unroll
            for (int m = 0; m < kMaxRows; ++m)
                if (m < rpw) dst[m * kThreads] = x[m];
        }
    };
    auto ws_load = [&](float (&x)[kMaxRows], const float* src) {
        if constexpr (kVec) {
            #pragma unroll
            for (int m = 0; m < kRpw; m += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(src + m * kThreads);
                x[m] = v4.x;
                x[m + 1] = v4.y;
                x[m + 2] = v4.z;
                x[m + 3] = v4.w;
            }
            #pragma unroll
            for (int m = kRpw; m < kMaxRows; ++m) x[m] = 0.f;
        } else {
            #pragma unroll
            for (int m = 0; m < kMaxRows; ++m) x[m] = m < rpw ? src[m * kThreads] : 0.f;
        }
    };

    // the inputs of tokens t0 .. t0+n-1 into shared memory (q and dO only for the reverse sweep);
    // every tensor is 16-byte aligned and d_k, d_v are multiples of 8, so rows move 8 elements at a time
    // A thread's pieces: rows of k, q (and per-key alpha) at most 2 (i0, i1), one v / dO piece,
    // one beta and one scalar alpha.  All are loaded before the barrier that frees the previous
    // chunk's buffers, so their latency overlaps the wait for the other warps.
    static_assert(kChunk * 128 / 8 <= 2 * kThreads && kChunk * (kCols / 8) <= kThreads, "chunk pieces per thread");
    auto load_chunk = [&](int64_t t0, int n, bool with_q) {
        const int pieces = n * dk / 8;
        const int i0 = tid, i1 = tid + kThreads;
        Raw8<T> k0{}, k1{}, q0{}, q1{}, v0{}, o0{};
        Raw8<float> a0{}, a1{};
        float as = 1.f, bs = 0.f;
        if (i0 < pieces) {
            k0 = raw8_load(k + t0 * dk + 8 * i0);
            if (with_q) q0 = raw8_load(q + t0 * dk + 8 * i0);
            if constexpr (kPK) a0 = raw8_load(al + t0 * dk + 8 * i0);
        }
        if (i1 < pieces) {
            k1 = raw8_load(k + t0 * dk + 8 * i1);
            if (with_q) q1 = raw8_load(q + t0 * dk + 8 * i1);
            if constexpr (kPK) a1 = raw8_load(al + t0 * dk + 8 * i1);
        }
        if (tid < n) {
            if constexpr (!kPK) as = al[t0 + tid];
            bs = be[t0 + tid];
        }
        const int tt = tid / (kCols / 8), cc = (tid % (kCols / 8)) * 8;
        const bool vpiece = tid < n * (kCols / 8), vin = vpiece && j0 + cc < dv;   // wholly inside d_v or outside
        if (vin) {
            v0 = raw8_load(v + (t0 + tt) * dv + j0 + cc);
            if (with_q) o0 = raw8_load(dO + (t0 + tt) * dv + j0 + cc);
        }
        __syncthreads();                                        // the previous chunk is consumed
        if (i0 < pieces) {
            raw8_store(k0, sk + 8 * i0);
            if (with_q) raw8_store(q0, sq + 8 * i0);
            if constexpr (kPK) raw8_store(a0, sa + 8 * i0);
        }
        if (i1 < pieces) {
            raw8_store(k1, sk + 8 * i1);
            if (with_q) raw8_store(q1, sq + 8 * i1);
            if constexpr (kPK) raw8_store(a1, sa + 8 * i1);
        }
        if (tid < n) {
            if constexpr (!kPK) sa[tid] = as;
            sbe[tid] = bs;
        }
        if (vpiece) {
            if (vin) {
                raw8_store(v0, sv + tt * kCols + cc);
                if (with_q) raw8_store(o0, sdo + tt * kCols + cc);
            } else {
                zero8(sv + tt * kCols + cc);
                if (with_q) zero8(sdo + tt * kCols + cc);
            }
        }
        __syncthreads();
    };

    // one forward step of the recurrence (token tau of the loaded chunk) on this thread's state
    // (keep_e: the column sum e of the token goes to se for the reverse sweep, which needs the same
    // value, computed from the same S_{t-1} in the same order)
    auto step = [&](float (&s)[kMaxRows], int tau, bool keep_e) {
        const float b = sbe[tau];
        float kr[kMaxRows], ar[kMaxRows];
        lds_rows<kRpw>(sk + tau * dk + r0, kr, rpw);
        if constexpr (kPK) lds_rows<kRpw>(sa + tau * dk + r0, ar, rpw);
        const float a0 = kPK ? 0.f : sa[tau];
        float pe = 0.f;
        #pragma unroll
        for (int m = 0; m < kMaxRows; ++m)
            if (m < rpw) pe += kr[m] * ((kDF && kPK) ? ar[m] * s[m] : s[m]);
        if (kDF && !kPK) pe *= a0;
        const float e = sum_row_groups(pe);
        if (keep_e && g == 0) se[tau * kCols + jl] = e;
        const float vj = sv[tau * kCols + jl];
        const float bd = b * (vj - e), bv = b * vj, be_ = b * e;
        const float cs = bv - a0 * be_;        // scalar alpha, printed order: a s + (b v - a b e) k
        #pragma unroll
        for (int m = 0; m < kMaxRows; ++m) {
            if (m >= rpw) break;
            const float ar_ = kPK ? ar[m] : a0;
            if (kDF) s[m] = ar_ * s[m] + kr[m] * bd;
            else if (kPK) s[m] = ar_ * (s[m] - kr[m] * be_) + kr[m] * bv;
            else s[m] = kr[m] * cs + a0 * s[m];
        }
    };

    // a warp's row sums over its 4 columns (16 per thread) into the partials of gradient gi, token slot sl
    auto park_rows = [&](float (&x)[kMaxRows], int gi, int sl) {
        sum_cols4(x, cg);
        float* dst = part + ((gi * kF + sl) * 8 + w) * ps;
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = (cg & 1) * 8 + (cg & 2) * 2 + i;
            const int r = r0 + m;
            if (m < rpw) dst[r + (r >> 5)] = x[i];
        }
    };

    // tokens tg0 .. tg0 + cnt - 1 (slots 0 .. cnt - 1): partials summed over the 8 warps, added to the outputs
    auto flush = [&](int64_t tg0, int cnt) {
        __syncthreads();                                        // every warp has parked its partials
        const int half = tid >> 7, r = tid & 127;
        if (r < dk) {
            for (int gs = half; gs < kNg * cnt; gs += 2) {
                const int gi = gs / cnt, sl = gs - gi * cnt;
                const float* src = part + ((gi * kF + sl) * 8) * ps + r + (r >> 5);
                float x = 0.f;
                #pragma unroll
                for (int ww = 0; ww < 8; ++ww) x += src[ww * ps];
                float* out = gi == 0 ? p.dq : (gi == 1 ? p.gdk : p.dalpha);
                atomicAdd(out + (u * L + tg0 + sl) * dk + r, x);
            }
        }
        if (tid < cnt) {
            float xb = 0.f, xa = 0.f;
            #pragma unroll
            for (int ww = 0; ww < 8; ++ww) {
                xb += pbe[tid * 8 + ww];
                if (!kPK) xa += pal[tid * 8 + ww];
            }
            atomicAdd(p.dbeta + u * L + tg0 + tid, xb);
            if (!kPK) atomicAdd(p.dalpha + u * L + tg0 + tid, xa);
        }
        __syncthreads();                                        // the partials are free again
    };

    // ---- phase A: forward, checkpoints at the chunk starts ----
    float s[kMaxRows];
    const float* S0 = p.S0 ? p.S0 + u * static_cast<int64_t>(dk) * dv : nullptr;
    #pragma unroll
    for (int m = 0; m < kMaxRows; ++m) s[m] = (m < rpw && active && S0) ? S0[static_cast<int64_t>(r0 + m) * dv + j] : 0.f;
    for (int ci = 0; ci < nck; ++ci) {
        const int64_t t0 = static_cast<int64_t>(ci) * kChunk;
        const int n = static_cast<int>(L - t0 < kChunk ? L - t0 : kChunk);
        ws_store(ck + ci * sst, s);
        load_chunk(t0, n, false);
        for (int tau = 0; tau < n; ++tau) step(s, tau, false);
    }

    // ---- phase B: chunks from the last, each recomputed, then swept backwards ----
    float G[kMaxRows];
    const float* dSL = p.dSL ? p.dSL + u * static_cast<int64_t>(dk) * dv : nullptr;
    #pragma unroll
    for (int m = 0; m < kMaxRows; ++m) G[m] = (m < rpw && active && dSL) ? dSL[static_cast<int64_t>(r0 + m) * dv + j] : 0.f;
    for (int ci = nck - 1; ci >= 0; --ci) {
        const int64_t t0 = static_cast<int64_t>(ci) * kChunk;
        const int n = static_cast<int>(L - t0 < kChunk ? L - t0 : kChunk);
        ws_load(s, ck + ci * sst);                              // (in flight while the inputs load)
        load_chunk(t0, n, true);
        ws_store(st, s);
        for (int tau = 0; tau < n; ++tau) {
            step(s, tau, true);
            if (tau + 1 < n) ws_store(st + (tau + 1) * sst, s); // S_t of the last token stays in s
        }
        __syncwarp();                                           // se is read by the warp's other lanes
        // S_t arrives from the previous step (S_{t-1} of token t+1); S_{t-1} is loaded one token ahead
        float sc[kMaxRows], sp[kMaxRows];
        #pragma unroll
        for (int m = 0; m < kMaxRows; ++m) sc[m] = s[m];
        ws_load(sp, st + (n - 1) * sst);
        for (int tau = n - 1; tau >= 0; --tau) {
            const int sl = tau % kF;                            // this token's slot among the parked partials
            // S_{t-2}, for the next token (at tau = 0 the chunk's first state again, never used)
            float spn[kMaxRows];
            ws_load(spn, st + (tau > 0 ? tau - 1 : 0) * sst);
            const float b = sbe[tau];
            const float vj = sv[tau * kCols + jl];
            const float oj = sdo[tau * kCols + jl];
            float kr[kMaxRows], ar[kMaxRows];
            lds_rows<kRpw>(sk + tau * dk + r0, kr, rpw);
            if constexpr (kPK) lds_rows<kRpw>(sa + tau * dk + r0, ar, rpw);
            const float a0 = kPK ? 0.f : sa[tau];
            {
                float qr[kMaxRows];
                lds_rows<kRpw>(sq + tau * dk + r0, qr, rpw);
                #pragma unroll
                for (int m = 0; m < kMaxRows; ++m)
                    if (m < rpw) G[m] += qr[m] * oj;           // from o_t = S_t^T q_t
            }
            // dq_t = S_t dO_t: row sums over the slice's columns
            {
                float x[kMaxRows];
                #pragma unroll
                for (int m = 0; m < kMaxRows; ++m) x[m] = m < rpw ? sc[m] * oj : 0.f;
                park_rows(x, 0, sl);
            }
            // the column sums of this step: e, k^T G, k^T Diag(alpha) G
            // (with a scalar alpha the third is alpha k^T G, and e of the decay-first order alpha k^T S)
            // (scalar alpha: gs = G . S_{t-1} over the thread's rows gives its dalpha term without a
            // per-element product: sum G P = gs - b e pg, sum dR S_{t-1} = gs - b kG ks)
            // e comes from the recompute, except with a scalar alpha in the decay-first order, whose
            // dalpha term needs this thread's share ks of k^T S_{t-1}
            constexpr bool kOwnE = kDF && !kPK;
            float pe = 0.f, pg = 0.f, pd = 0.f, gs = 0.f;
            #pragma unroll
            for (int m = 0; m < kMaxRows; ++m) {
                if (m >= rpw) break;
                if (kOwnE) pe += kr[m] * sp[m];
                pg += kr[m] * G[m];
                if (kPK) pd += kr[m] * ar[m] * G[m];
                if (!kPK) gs += G[m] * sp[m];
            }
            const float ks = pe;                        // k^T S_{t-1} over the thread's rows (kOwnE)
            const float e = kOwnE ? sum_row_groups(pe * a0) : se[tau * kCols + jl];
            const float kG = sum_row_groups(pg);
            const float kdP = kPK ? sum_row_groups(pd) : a0 * kG;
            if (active && g == 0) p.gdv[(u * L + t0 + tau) * dv + j] = b * kG;
            // dbeta: column terms summed over the warp's columns, parked per warp
            {
                float tb = active ? (kDF ? kG * (vj - e) : kG * vj - kdP * e) : 0.f;
                tb += __shfl_xor_sync(0xffffffffu, tb, 1);
                tb += __shfl_xor_sync(0xffffffffu, tb, 2);
                if (lane == 0) pbe[sl * 8 + w] = tb;
            }
            // (a column past d_v has S = 0, G = 0 and v = dO = 0 throughout, so its terms are 0)
            float dkx[kMaxRows], dax[kMaxRows];
            {
                const float bkG = b * kG, bkdP = b * kdP, bd = b * (vj - e), bv = b * vj, bE = b * e;
                // scalar alpha: R bkG = (a bkG) S_{t-1}, and G bv - dP bE = (bv - a bE) G
                const float abkG = a0 * bkG, cv = bv - a0 * bE;
                #pragma unroll
                for (int m = 0; m < kMaxRows; ++m) {
                    dkx[m] = dax[m] = 0.f;
                    if (m >= rpw) continue;
                    const float ar_ = kPK ? ar[m] : a0;
                    if (kDF) {
                        const float dR = G[m] - kr[m] * bkG;
                        if (kPK) {
                            dkx[m] = G[m] * bd - ar_ * sp[m] * bkG;
                            dax[m] = dR * sp[m];
                        } else {
                            dkx[m] = G[m] * bd - sp[m] * abkG;
                        }
                        G[m] = ar_ * dR;
                    } else if (kPK) {
                        const float dP = ar_ * G[m];
                        dkx[m] = G[m] * bv - (sp[m] * bkdP + dP * bE);
                        dax[m] = G[m] * (sp[m] - kr[m] * bE);
                        G[m] = dP - kr[m] * bkdP;
                    } else {
                        dkx[m] = G[m] * cv - sp[m] * bkdP;
                        G[m] = a0 * G[m] - kr[m] * bkdP;
                    }
                }
            }
            park_rows(dkx, 1, sl);
            if constexpr (kPK) {
                park_rows(dax, 2, sl);
            } else {
                const float dal_sum = kDF ? gs - b * kG * ks : gs - b * e * pg;
                const float x = warp_sum(dal_sum);
                if (lane == 0) pal[sl * 8 + w] = x;
            }
            if (sl == 0) flush(t0 + tau, min(kF, n - tau));
            #pragma unroll
            for (int m = 0; m < kMaxRows; ++m) {
                sc[m] = sp[m];
                sp[m] = spn[m];
            }
        }
    }
    if (p.dS0 && active) {
        float* o = p.dS0 + u * static_cast<int64_t>(dk) * dv;
        #pragma unroll
        for (int m = 0; m < kMaxRows; ++m)
            if (m < rpw) o[static_cast<int64_t>(r0 + m) * dv + j] = G[m];
    }
}

// Scratch of the allocation-free entry point (lt2_gdr_backward_static): a fixed 64 MiB array in
// device memory, reserved on every GPU that loads this library until the process exits.  For
// callers that may not allocate device memory themselves: a host program whose device memory is
// all handed out by someone else's allocator, or a service that must not call cudaMalloc once it
// is serving (the call can block the device).  Every call of that entry point on a device uses
// this one array, so calls that overlap on the GPU -- from two streams or two host threads --
// overwrite each other's scratch and must be serialised by the caller.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

__global__ void zero_kernel(float* x, int64_t n)
{
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        x[i] = 0.f;
}

}  // namespace bw

size_t backward_static_scratch_bytes() { return bw::kStaticScratchBytes; }

// The device address of the static scratch on the current device.  In host code the array's name
// is only a host-side stand-in, so the address comes from cudaGetSymbolAddress, once per device
// with that device current, and is cached.
cudaError_t backward_static_scratch(float** out)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<float*> cache[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    float* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(mu);
        p = cache[dev].load(std::memory_order_acquire);
        if (!p) {
            void* addr = nullptr;
            e = cudaGetSymbolAddress(&addr, bw::g_static_scratch);
            if (e != cudaSuccess) return e;
            p = static_cast<float*>(addr);
            cache[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

size_t backward_workspace_bytes(int64_t units, int64_t L, int dk, int dv)
{
    const int64_t slices = (dv + bw::kCols - 1) / bw::kCols;
    return static_cast<size_t>(units * slices * bw::ws_floats_per_block(L, dk) * 4);
}

cudaError_t launch_backward(const BwCall& c, cudaStream_t stream)
{
    using namespace bw;
    if (c.units == 0) return cudaSuccess;
    NvtxRange range("lt2 backward (cuda core)");
    const int64_t na = c.per_key ? c.dk : 1;
    const int64_t zn[4] = {c.units * c.L * c.dk, c.units * c.L * c.dk, c.units * c.L * na, c.units * c.L};
    float* zp[4] = {c.dq, c.dk_out, c.dalpha, c.dbeta};
    for (int i = 0; i < 4; ++i) {
        if (zn[i] == 0) continue;
        const int64_t blocks = (zn[i] + 255) / 256 < 4096 ? (zn[i] + 255) / 256 : 4096;
        zero_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(zp[i], zn[i]);
    }
    Params p;
    p.q = c.q;
    p.k = c.k;
    p.v = c.v;
    p.alpha = c.alpha;
    p.beta = c.beta;
    p.S0 = c.S0;
    p.dO = c.dO;
    p.dSL = c.dSL;
    p.dq = c.dq;
    p.gdk = c.dk_out;
    p.gdv = c.dv_out;
    p.dalpha = c.dalpha;
    p.dbeta = c.dbeta;
    p.dS0 = c.dS0;
    p.ws = c.ws;
    p.units = c.units;
    p.L = c.L;
    p.dk = c.dk;
    p.dv = c.dv;
    p.per_key = c.per_key;
    p.decay_first = c.decay_first;
    const dim3 grid(static_cast<unsigned>(c.units), static_cast<unsigned>((c.dv + kCols - 1) / kCols), 1);
    const size_t smem = smem_bytes(c.dk, c.per_key);
    // [bf16][d_k == 128][decay-first][per-key]
    using Kernel = void (*)(Params);
    static const Kernel kernels[2][2][2][2] = {
        {{{gdr_backward_kernel<float, 0, false, false>, gdr_backward_kernel<float, 0, false, true>},
          {gdr_backward_kernel<float, 0, true, false>, gdr_backward_kernel<float, 0, true, true>}},
         {{gdr_backward_kernel<float, 16, false, false>, gdr_backward_kernel<float, 16, false, true>},
          {gdr_backward_kernel<float, 16, true, false>, gdr_backward_kernel<float, 16, true, true>}}},
        {{{gdr_backward_kernel<__nv_bfloat16, 0, false, false>, gdr_backward_kernel<__nv_bfloat16, 0, false, true>},
          {gdr_backward_kernel<__nv_bfloat16, 0, true, false>, gdr_backward_kernel<__nv_bfloat16, 0, true, true>}},
         {{gdr_backward_kernel<__nv_bfloat16, 16, false, false>, gdr_backward_kernel<__nv_bfloat16, 16, false, true>},
          {gdr_backward_kernel<__nv_bfloat16, 16, true, false>, gdr_backward_kernel<__nv_bfloat16, 16, true, true>}}}};
    const Kernel kernel = kernels[c.dtype_bf16 ? 1 : 0][c.dk == 128 ? 1 : 0][c.decay_first ? 1 : 0][c.per_key ? 1 : 0];
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace lt2
