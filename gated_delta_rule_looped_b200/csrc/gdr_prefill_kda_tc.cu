// gdr_prefill_kda_tc.cu -- chunked prefill of the gated delta rule with per-key gating
// (alpha_t a d_k vector) on Blackwell tensor cores, d_k = d_v = 128, bf16 q/k/v.
//
// The recurrence ("LT2 transformer looped a tempo lineare", section "Sostituire il motore",
// displayed equation)  S_t = Diag(alpha_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
// read out as o_t = S_t^T q_t, is taken 32 tokens ("a chunk") at a time in its e-form: with the
// chunk's incoming state S, G_r = sum_{s<=r} log alpha_s (a d_k vector, G_{-1} = 0),
// Gamma_r = Diag(e^{G_r}) and e_r = k_r^T S_{r-1},
//
//   (I + M_ke) E = K^ S + M_kv V                                    (E: rows e_r)
//   O  = Q^ S + N_qv V - N_qe E
//   S' = Gamma_31 S + Kv^T V - Ke^T E
//
//   K^_r = Gamma_{r-1} k_r,  Q^_r = Gamma_r q_r,  Kv_s = beta_s Gamma_31 Gamma_s^{-1} k_s,
//   Ke_s = beta_s Gamma_31 Gamma_{s-1}^{-1} k_s,
//   M_ke[r,s] = beta_s k_r^T Gamma_{r-1} Gamma_{s-1}^{-1} k_s  (s < r),  M_kv: Gamma_s^{-1} (s < r),
//   N_qe[r,s] = beta_s q_r^T Gamma_r Gamma_{s-1}^{-1} k_s  (s <= r),     N_qv: Gamma_s^{-1} (s <= r).
//
// (Checked in fp64 against the sequential definition by the test suite's chunked oracle.)
// K^ and Q^ carry factors of at most 1.  The four chunk Gram matrices are products of fp16
// tiles Kt, Qt and Be, Bv that carry e^{G - R} and e^{R - G} around a per-key reference
// R = G_31 / 2; Be and Bv also serve the state update (Kv = sq Bv, Ke = sq Be, sq = e^{G_31/2}).
// The tiles stay in range while a key decays by at most e^-19 over the chunk.  A chunk beyond
// that (or with any alpha <= 0, a reset) is instead run token by token, exactly, on the fp32
// state in TMEM.  A growing alpha > 1 stays on the tensor cores while the state and the tiles
// remain inside fp16.
//
// With the solve X = [T; N_qe T], T = (I + M_ke)^{-1}, and Z = X M_kv - [0; N_qv]:
//   [E; -(O - Q^ S)] = X (K^ S) + Z V,
// so one MMA (MMA_B) gives both E and the non-state part of O.  Per chunk, on transposed
// quantities (one d_v column per TMEM lane):
//   MMA_A  (K^ S, Q^ S)^T    = S^T [K^; Q^]^T          A = S^T (TMEM, fp16)   N = 64
//   MMA_B  ([E; -O'])^T      = V^T Z^T + (K^ S)^T X^T  A = V^T (smem), then (K^ S)^T (TMEM)
//   MMA_C  (sq S)^T += V^T Bv - E^T Be, giving (S' / sq)^T
// where sq = sqrt(P_31) per key and Bv, Be are the Gram tiles below: Kv = sq Bv, Ke = sq Be, so
// the fp32 state in TMEM is kept scaled by sq (per key, i.e. per TMEM column) around MMA_C.
//
// Decay-first order (A_t = (I - beta_t k_t k_t^T) Diag(alpha_t), the other reading of the
// per-key equation): e_r = k_r^T Diag(alpha_r) S_{r-1}, and token s's delta term decays like its
// write term, so the same system holds with Gamma_r in place of Gamma_{r-1} on the k_r side
// (K^, and M_ke, M_kv) and Gamma_s^{-1} in place of Gamma_{s-1}^{-1} on the e side (M_ke, N_qe,
// Ke): M_ke = M_kv, N_qe = N_qv, Ke = Kv.  In the tiles below that is K^_t = P_t k_t,
// Kt_t = F_t k_t and Be_t = Bv_t; everything else is unchanged.
//
// CTA = one (loop, batch, head) unit, 16 warps:
//   warp 0       TMA producer (and TMEM allocation)
//   warps 1-3    conversion of tokens 0-10 / 11-21 / 22-31: per-key decay factors, the six
//                fp16 tiles of K and Q, and V to fp16
//   warps 4-7    prep: Gram epilogue, diagonal-block inverses, back substitution, Z; warp 4
//                then issues the next chunk's Gram MMA
//   warps 8-15   the S-dependent chain (warp 8 issues MMA_A, MMA_B, MMA_C) and the output
//                epilogue, which runs while MMA_C does.  Warps w and w + 4 share TMEM lanes
//                32 (w & 3) .. + 31 (d_v columns) and split every epilogue by TMEM column: keys
//                0-63 / 64-127 of the state, tokens 0-15 / 16-31 of the chunk
// Every mbarrier wait is bounded (see mbar_wait); a timeout is recorded in the device status
// word and the CTA drains its copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "gdr_common.cuh"
#include "gdr_launch.h"
#include "gdr_nvtx.h"
#include "gdr_tc_common.cuh"
#include "gdr_tma_host.h"
#include "sm100_primitives.cuh"

namespace lt2 {
namespace kda {

using namespace sm100;
using namespace tcc;

constexpr int kC = 32;                 // tokens per chunk
constexpr int kThreads = 512;
constexpr int kConv = 3;               // conversion warps
constexpr int kStages = 3;
constexpr uint64_t kTimeoutNs = kWaitTimeoutNs;
// Gram tiles carry factors e^{+-(G - G_31/2)}: in range while they stay within [2^-14, 2^14].
constexpr float kFactorMax = 16384.f;
constexpr float kFactorMin = 1.f / 16384.f;

// Shared memory map (offsets from a 1024-byte aligned base).  Tiles are fp16, 128-byte rows
// (64 elements) under the 128-byte swizzle; a 128-wide operand is two panels.
// Chunk stage (3): [K^ | Q^] x 2 panels (rows 0-31 K^, 32-63 Q^), [Be | Bv] x 2 panels, V x 2.
constexpr uint32_t ST_KQ = 0;          // + panel * 8192
constexpr uint32_t ST_KVE = 16384;     // + panel * 8192
constexpr uint32_t ST_V = 32768;       // + panel * 4096
constexpr uint32_t STAGE_BYTES = 40960;
constexpr uint32_t STAGE_TX = 6 * 4096;   // K, Q, V boxes of 64 columns x 32 tokens (bf16)
constexpr uint32_t OFF_STG = 0;
// Gram tiles, two buffers: buffer b holds [Kt (rows 64b + 0-31) | Qt (64b + 32-63)] of each panel.
// The Gram reads 128 rows from its buffer's first row; the 64 rows past the buffer (the other
// buffer, or the next region) reach only TMEM lanes that are never read.
constexpr uint32_t OFF_GRAM = OFF_STG + kStages * STAGE_BYTES;
constexpr uint32_t GRAM_PANEL = 16384;
constexpr uint32_t GRAM_BUF = 8192;
// [X | Z] stages (2): 64 rows; X = [T; N_qe T] in columns 0-31, Z in columns 32-63.
constexpr uint32_t OFF_TP = OFF_GRAM + 2 * GRAM_PANEL;
constexpr uint32_t TP_STAGE = 8192;
constexpr int TP_ZCOL = 32;
// Gram blocks for the solve (32 rows each): [-M_ke | N_qe] and [M_kv | N_qv].
constexpr uint32_t OFF_MA = OFF_TP + 2 * TP_STAGE;
constexpr uint32_t OFF_MB = OFF_MA + 4096;
// alpha of a chunk, [32 tokens][128] fp32, landed by TMA (2 stages).
constexpr uint32_t OFF_ALPHA = OFF_MB + 4096;
constexpr uint32_t ALPHA_STAGE = 16384;
constexpr uint32_t OFF_ADIAG = OFF_ALPHA + 2 * ALPHA_STAGE;   // fp32 diagonal blocks of -M_ke
constexpr uint32_t ADIAG_BLOCK = 16 * kAdiagRow;
constexpr uint32_t OFF_OST = OFF_ADIAG + 2304;   // o staging: 2 x [32 tokens][64] bf16
constexpr uint32_t OFF_GATES = OFF_OST + 8192;
constexpr uint32_t GATE_STAGE = 640;
constexpr uint32_t OFF_BAR = OFF_GATES + kStages * GATE_STAGE;
constexpr uint32_t BAR_BYTES = 512;
constexpr uint32_t SMEM_USED = OFF_BAR + BAR_BYTES;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

struct Gates {
    float sq[kD];      // sqrt(e^{G_31}): square root of the chunk's decay per key
    int in_range[8];   // per conversion warp: Gram factors within range for its tokens
};
static_assert(sizeof(Gates) <= GATE_STAGE, "gate stage too small");

__device__ __forceinline__ bool gates_in_range(const Gates* g)
{
    int all = 1;
    #pragma unroll
    for (int w = 0; w < kConv; ++w) all &= g->in_range[w];
    return all != 0;
}

enum Bar : uint32_t {
    B_FULL = 0,        // [3] TMA of a stage landed
    B_CONV = 3,        // [3] stage and Gram tiles converted (the conversion warps)
    B_EMPTY = 6,       // [3] chain done with a stage
    B_GATE_FULL = 9,   // [3] decay factors written (the conversion warps)
    B_GATE_EMPTY = 12, // [3] chain done with a gate stage
    B_TP_FULL = 15,    // [2]
    B_TP_EMPTY = 17,   // [2]
    B_G_FULL = 19,     // Gram in TMEM
    B_GFREE = 21,      // [2] Gram MMA done reading a Gram tile buffer
    B_A_FULL = 23,
    B_B_FULL = 24,
    B_S_FULL = 25,
    B_DRAIN = 26,      // [2]
    B_AL_FULL = 28,    // [2] TMA of a chunk's alpha landed
    B_AL_EMPTY = 30,   // [2] conversion warps done with it
    B_COUNT = 32
};
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + B_COUNT * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 16;
static_assert(OFF_ABORT + 16 <= OFF_BAR + BAR_BYTES, "barrier area too small");

constexpr int NB_PREP = 1, NB_CHAIN = 2, NB_CONV = 3;

// TMEM columns (lane j = d_v index in the chain's regions).
constexpr uint32_t TM_G = 0;           // Gram (64 columns; lanes 0-31 Kt rows, 32-63 Qt rows)
constexpr uint32_t TM_S = 64;          // S^T fp32, scaled per key by sq around MMA_C (128)
constexpr uint32_t TM_SH = 192;        // S^T fp16 pairs (64): A operand of MMA_A
constexpr uint32_t TM_AB = 256;        // (K^ S)^T 256..287, (Q^ S)^T 288..319
constexpr uint32_t TM_Y = 384;         // (K^ S)^T as fp16 pairs (16), A operand of MMA_B
constexpr uint32_t TM_E = 400;         // -E^T as fp16 pairs (16), A operand of MMA_C
constexpr uint32_t TM_B = 320;         // E^T 320..351, -(O - Q^ S)^T 352..383
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_GRAM = idesc_f16_f32(128, 64, 0, 0);
constexpr uint32_t ID_T64 = idesc_f16_f32(128, 64, 0, 0);     // A in TMEM, B K-major, N = 64
constexpr uint32_t ID_M64 = idesc_f16_f32(128, 64, 1, 0);     // A MN-major (smem), B K-major
constexpr uint32_t ID_MM = idesc_f16_f32(128, 128, 1, 1);     // A MN-major (smem), B MN-major
constexpr uint32_t ID_TM = idesc_f16_f32(128, 128, 0, 1);     // A in TMEM, B MN-major

struct Params {
    const __nv_bfloat16* q;    // [units_total][L][128] (the exact path of out-of-range chunks)
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* alpha;        // [units_total][L][128]
    const float* beta;         // [units_total][L]
    const float* S0;           // [units_total][128][128] or null
    void* o;
    float* S_out;              // nullable
    int64_t L;
    int unit0;
    int units_total;           // T*B*H (the extent of the tensor maps' unit axis)
    int out_bf16;
    unsigned int* err;
    // fused prologue and output gate (used by the instances that compile the step in)
    int qk_norm;
    int gate_logits;
    float alpha_scale;
    const __nv_bfloat16* z;    // [units_total][L][128] output gate logits, or null
};
// The packed-sequence instances' parameters: q/k/v/o/z/alpha [T][H][L][128], beta [T][H][L] with L
// the packed length; CTA = (sequence b, head h) of loop `loop`, tokens cu[b] .. cu[b+1]-1.  (A
// separate type, so that the fixed-length instances keep their parameter block as it was.)
struct ParamsVar : Params {
    const int64_t* cu;
    int H;
    int loop;
};
template <bool kVar> using KdaParams = typename std::conditional<kVar, ParamsVar, Params>::type;

#ifdef LT2_DEBUG
// Fault injection of the debug build: the producer stops before this chunk (-1: never), so its
// copies never arrive and the waits for them run out.
__device__ int g_debug_skip_chunk = -1;
#endif

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, uint32_t i) { return base + OFF_BAR + 8u * i; }

// ---- conversion: per-key decay factors and the six fp16 tiles of one chunk ----------------
// Conversion warp w (0 .. 2) converts tokens [conv_begin(w), conv_begin(w + 1)) of the chunk for
// all 128 keys; lane l owns keys 4l .. 4l+3 (8 bytes of a row of panel l >> 4 of every 128-wide
// tile).  With P_t = e^{G_t} (P_-1 = 1), sq = sqrt(P_31), F_t = P_t / sq and R_t = 1 / F_t:
//   K^_t = P_{t-1} k_t,  Q^_t = P_t q_t,  Kt_t = F_{t-1} k_t,  Qt_t = F_t q_t,
//   Bv_t = b_t R_t k_t,  Be_t = b_t R_{t-1} k_t
// (the state products need Kv = sq Bv and Ke = sq Be: sq R_t = P_31 / P_t), and V_t to fp16.
// P_t comes in two steps: each warp first overwrites the alpha rows of its own tokens with the
// running product over them (local_products); after a barrier of the conversion warps, row
// conv_begin(v + 1) - 1 holds the product over warp v's tokens, from which a warp takes the
// product over the tokens before its own and over the whole chunk (chunk_products).  The loops
// stay rolled: this code runs once per chunk per warp and would otherwise be fetched afresh
// every time.
__device__ __forceinline__ int conv_begin(int w) { return w < kConv ? 11 * w : kC; }

__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 scale4(float4 a, float s) { return make_float4(a.x * s, a.y * s, a.z * s, a.w * s); }
__device__ __forceinline__ float4 rcp4(float4 a)
{
    return make_float4(rcp_approx(a.x), rcp_approx(a.y), rcp_approx(a.z), rcp_approx(a.w));
}
__device__ __forceinline__ float4 unpack4_bf16(uint2 w)
{
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}
__device__ __forceinline__ uint2 pack4_scaled(float4 x, float4 f)
{
    return make_uint2(pack_half2(x.x * f.x, x.y * f.y), pack_half2(x.z * f.z, x.w * f.w));
}
__device__ __forceinline__ bool in_factor_range(float4 f)
{
    return fminf(fminf(f.x, f.y), fminf(f.z, f.w)) >= kFactorMin && fmaxf(fmaxf(f.x, f.y), fmaxf(f.z, f.w)) <= kFactorMax;
}

// Row t of the chunk's alpha (t in [t_begin, t_end)) becomes prod_{t_begin <= u <= t} alpha_u,
// alpha taken as 1 past the chunk's last token n - 1.
// With kLogits (the fused prologue) the rows hold logits a, and alpha = exp(-softplus(a) c).
template <bool kLogits>
__device__ __forceinline__ void local_products(float* alpha_c, int n, int t_begin, int t_end, int lane, float c)
{
    float4 p = make_float4(1.f, 1.f, 1.f, 1.f);
    #pragma unroll 1
    for (int t4 = t_begin; t4 < t_end; t4 += 4) {
        float4* row = reinterpret_cast<float4*>(alpha_c + t4 * kD + 4 * lane);
        float4 a[4];
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] = t4 + i < n && t4 + i < t_end ? row[i * (kD / 4)] : make_float4(1.f, 1.f, 1.f, 1.f);
            if (kLogits && t4 + i < n)
                a[i] = make_float4(alpha_from_logit_fast(a[i].x, c), alpha_from_logit_fast(a[i].y, c),
                                   alpha_from_logit_fast(a[i].z, c), alpha_from_logit_fast(a[i].w, c));
        }
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            p = mul4(p, a[i]);
            if (t4 + i < t_end) row[i * (kD / 4)] = p;
        }
    }
}

// After local_products of every conversion warp: the product over the tokens before warp w's
// (Ph) and over the whole chunk (returned).
__device__ __forceinline__ float4 chunk_products(const float* alpha_c, int w, int lane, float4& Ph)
{
    float4 Pt = make_float4(1.f, 1.f, 1.f, 1.f);
    Ph = Pt;
    #pragma unroll
    for (int v = 0; v < kConv; ++v) {
        const float4 tot = *reinterpret_cast<const float4*>(alpha_c + (conv_begin(v + 1) - 1) * kD + 4 * lane);
        if (v == w) Ph = Pt;
        Pt = mul4(Pt, tot);
    }
    return Pt;
}

// The tiles of tokens [t_begin, t_end), given Ph and the chunk's product Pt; alpha_c holds the
// running products of local_products.  The warp starting at token 0 writes sq of every key to
// `sq_out`; the return value says whether every F_t of the warp's tokens lies in
// [kFactorMin, kFactorMax].
// kNorm (the fused prologue): every k and q row is divided by its L2 norm first (the warp holds
// the whole row, four keys a lane).
template <bool decay_first, bool kNorm>
__device__ __forceinline__ bool convert_kqv(uint32_t st, uint32_t gram, const float* alpha_c, float bl, float4 Ph,
                                            float4 Pt, int t_begin, int t_end, int lane, uint8_t* sbase, uint32_t sb,
                                            float* sq_out)
{
    const float4 isq = make_float4(rsqrt_approx(Pt.x), rsqrt_approx(Pt.y), rsqrt_approx(Pt.z), rsqrt_approx(Pt.w));
    if (t_begin == 0) *reinterpret_cast<float4*>(sq_out + 4 * lane) = mul4(Pt, isq);
    float4 P = Ph;                               // P_{t-1}
    float4 F = mul4(P, isq);                     // F_{t-1}
    float4 R = rcp4(F);                          // 1 / F_{t-1}
    bool ok = in_factor_range(F);
    // the eight bytes of row t this lane owns, in every tile (rows 32 + t: +4096 bytes)
    const int panel = lane >> 4;
    const uint32_t chunk = static_cast<uint32_t>((lane & 15) >> 1), within = static_cast<uint32_t>(lane & 1) * 8u;
    uint8_t* kq = sbase + (st + ST_KQ + panel * 8192 - sb);
    uint8_t* bve = sbase + (st + ST_KVE + panel * 8192 - sb);
    uint8_t* vt = sbase + (st + ST_V + panel * 4096 - sb);
    uint8_t* gp = sbase + (gram + panel * GRAM_PANEL - sb);
    const float* arow = alpha_c + 4 * lane;
    #pragma unroll 1
    for (int t = t_begin; t < t_end; ++t) {
        const float4 lp = *reinterpret_cast<const float4*>(arow + t * kD);
        const float b = __shfl_sync(0xffffffffu, bl, t);
        const uint32_t off = sw128(0u, t, chunk) + within;
        uint2* kp = reinterpret_cast<uint2*>(kq + off);
        uint2* qp = reinterpret_cast<uint2*>(kq + off + 4096);
        uint2* vp = reinterpret_cast<uint2*>(vt + off);
        float4 k = unpack4_bf16(*kp), q = unpack4_bf16(*qp);
        if (kNorm) {
            float nk = k.x * k.x + k.y * k.y + k.z * k.z + k.w * k.w;
            float nq = q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
            #pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
            }
            k = scale4(k, inv_l2_fast(nk));
            q = scale4(q, inv_l2_fast(nq));
        }
        const uint2 vb = *vp;
        const float4 Pn = mul4(Ph, lp), Fn = mul4(Pn, isq), Rn = rcp4(Fn);
        ok = ok && in_factor_range(Fn);
        *kp = pack4_scaled(k, decay_first ? Pn : P);                            // K^ (in place)
        *qp = pack4_scaled(q, Pn);                                              // Q^ (in place)
        *vp = make_uint2(pack_half2(bf16_lo(vb.x), bf16_hi(vb.x)), pack_half2(bf16_lo(vb.y), bf16_hi(vb.y)));
        *reinterpret_cast<uint2*>(gp + off) = pack4_scaled(k, decay_first ? Fn : F);               // Kt
        *reinterpret_cast<uint2*>(gp + off + 4096) = pack4_scaled(q, Fn);       // Qt
        *reinterpret_cast<uint2*>(bve + off) = pack4_scaled(k, scale4(decay_first ? Rn : R, b));   // Be
        *reinterpret_cast<uint2*>(bve + off + 4096) = pack4_scaled(k, scale4(Rn, b));   // Bv
        P = Pn;
        F = Fn;
        R = Rn;
    }
    return __all_sync(0xffffffffu, ok);
}

// ---- prep helpers (32-token chunk: two 16-token blocks) -----------------------------------

// Gram epilogue, row r of the Kt rows (warp 4) or Qt rows (warp 5): the two 32-column halves
// of the Gram row (against Be, against Bv), masked to s < r (Kt rows) or s <= r (Qt rows),
// as fp16 rows of -M_ke / M_kv (columns 0-31 of the MA / MB tiles) or N_qe / N_qv (columns
// 32-63); the Kt rows also keep fp32 copies of the diagonal 16x16 blocks of -M_ke.
__device__ __forceinline__ void gram_epilogue_row(const float (&v)[64], int r, bool kt_rows, uint8_t* sbase,
                                                  uint32_t sb, float* adiag)
{
    const int lim = kt_rows ? r : r + 1;
    const float sg = kt_rows ? -1.f : 1.f;
    const uint32_t t_e = sb + OFF_MA, t_v = sb + OFF_MB;
    const int c0 = kt_rows ? 0 : 4;             // Kt rows in columns 0-31, Qt rows in 32-63
    float e[32], w[32];
    #pragma unroll
    for (int s = 0; s < 32; ++s) {
        e[s] = s < lim ? sg * v[s] : 0.f;
        w[s] = s < lim ? v[32 + s] : 0.f;
    }
    #pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        *reinterpret_cast<uint4*>(sbase + (sw128(t_e, r, c0 + ch) - sb)) = pack8_half(e + 8 * ch);
        *reinterpret_cast<uint4*>(sbase + (sw128(t_v, r, c0 + ch) - sb)) = pack8_half(w + 8 * ch);
    }
    if (kt_rows) {
        const bool upper = (r & 16) != 0;
        float* ad = adiag + (r >> 4) * ADIAG_BLOCK + (r & 15) * kAdiagRow;
        #pragma unroll
        for (int j = 0; j < 16; ++j) ad[j] = upper ? e[16 + j] : e[j];
    }
}

// Row block rb of Z = X M_kv - [0; N_qv] (X in columns 0-31 of TP, Z to columns 32-63; M_kv
// and N_qv in columns 0-31 and 32-63 of MB; M_kv strictly lower).
__device__ __noinline__ void z_row_block(uint32_t tp, uint32_t mb, int rb, int lane)
{
    const bool is_t = rb < 2;
    const uint32_t g = lane >> 2, tq = lane & 3;
    #pragma unroll 1
    for (int j = 0; j < 2; ++j) {
        float acc[2][4];
        zero_c(acc);
        if (!is_t) {
            // -N_qv block (rb - 2, j) in the accumulator layout: rows g, g+8; columns 2tq, 2tq+1
            const int row0 = 16 * (rb - 2);
            #pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const uint32_t c0 = lds32(sw128(mb, row0 + g, 4 + 2 * j + nb) + tq * 4);
                const uint32_t c1 = lds32(sw128(mb, row0 + g + 8, 4 + 2 * j + nb) + tq * 4);
                acc[nb][0] = -half_lo(c0);
                acc[nb][1] = -half_hi(c0);
                acc[nb][2] = -half_lo(c1);
                acc[nb][3] = -half_hi(c1);
            }
        }
        const int kmax = is_t ? rb : 1;
        #pragma unroll 1
        for (int k = j; k <= kmax; ++k) {
            uint32_t a[4], b[4];
            frag_a(tp, 16 * rb, 16 * k, lane, a);
            frag_b(mb, 16 * k, 16 * j, lane, b);
            mma_block(acc, a, b);
        }
        store_block(tp, 16 * rb, TP_ZCOL + 16 * j, lane, acc, 1.f);
    }
}

// ---- chain helpers --------------------------------------------------------------------------

// Chain thread (d_v column j, key half piece0 / 2): keys 32 piece0 .. + 63 of S0^T row j into
// TMEM, as fp16 pairs (unscaled) and as fp32 scaled per column i (= key) by f[i] (nullptr:
// unscaled).
__device__ __noinline__ void load_initial_state(uint32_t tm_s, uint32_t tm_sh, const float* s0, const float* f,
                                                int piece0)
{
    #pragma unroll 1
    for (int piece = piece0; piece < piece0 + 2; ++piece) {
        float v[32];
        #pragma unroll
        for (int d = 0; d < 32; ++d) v[d] = s0 ? s0[(32 * piece + d) * kD] : 0.f;
        uint32_t hpk[16];
        #pragma unroll
        for (int e = 0; e < 16; ++e) hpk[e] = pack_half2(v[2 * e], v[2 * e + 1]);
        tmem_st16(tm_sh + 16 * piece, hpk);
        if (f) {
            #pragma unroll
            for (int d = 0; d < 32; ++d) v[d] *= f[32 * piece + d];
        }
        tmem_st32(tm_s + 32 * piece, v);
    }
    tmem_wait_st();
}

// Chain thread (d_v column j, keys 32 piece .. + 63), after a chunk: the state
// S' = f_sh (.) TM_S (per column i = key; nullptr: 1) as fp16 pairs for MMA_A, and
// TM_S <- f_s (.) S' (nullptr: 1), the pre-scaled state the next chunk's MMA_C accumulates into.
__device__ __forceinline__ void state_update(uint32_t tm_s, uint32_t tm_sh, const float* f_sh, const float* f_s,
                                             int piece)
{
    {
        float v[64];
        tmem_load_2x32(tm_s + 32 * piece, tm_s + 32 * piece + 32, v);
        if (f_sh) {
            #pragma unroll
            for (int d4 = 0; d4 < 64; d4 += 4) {
                const float4 f = *reinterpret_cast<const float4*>(f_sh + 32 * piece + d4);
                v[d4 + 0] *= f.x;
                v[d4 + 1] *= f.y;
                v[d4 + 2] *= f.z;
                v[d4 + 3] *= f.w;
            }
        }
        uint32_t hpk[32];
        #pragma unroll
        for (int e = 0; e < 32; ++e) hpk[e] = pack_half2(v[2 * e], v[2 * e + 1]);
        tmem_st16(tm_sh + 16 * piece, *reinterpret_cast<uint32_t(*)[16]>(hpk));
        tmem_st16(tm_sh + 16 * piece + 16, *reinterpret_cast<uint32_t(*)[16]>(hpk + 16));
        if (f_s) {
            #pragma unroll
            for (int d4 = 0; d4 < 64; d4 += 4) {
                const float4 f = *reinterpret_cast<const float4*>(f_s + 32 * piece + d4);
                v[d4 + 0] *= f.x;
                v[d4 + 1] *= f.y;
                v[d4 + 2] *= f.z;
                v[d4 + 3] *= f.w;
            }
        }
        if (f_sh || f_s) {
            tmem_st32(tm_s + 32 * piece, *reinterpret_cast<float(*)[32]>(v));
            tmem_st32(tm_s + 32 * piece + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        }
    }
    tmem_wait_st();
}

// Chain thread (d_v column j, keys 32 piece .. + 63): that part of column j of the final state,
// f (.) TM_S (nullptr: 1), to S_out.  Returns false if any entry is not finite.
__device__ __noinline__ bool store_final_state_scaled(uint32_t tm_s, float* so, const float* f, int piece)
{
    bool fin = true;
    float v[64];
    tmem_load_2x32(tm_s + 32 * piece, tm_s + 32 * piece + 32, v);
    #pragma unroll
    for (int d = 0; d < 64; ++d) {
        const float x = f ? v[d] * f[32 * piece + d] : v[d];
        fin &= is_finite(x);
        so[(32 * piece + d) * kD] = x;
    }
    return fin;
}

// Chain thread j: the chunk's n tokens run one at a time on column j of the fp32 state in
// TMEM (the definition, in fp32): e = k^T S, S <- Diag(alpha) (S - beta k e) + beta k v^T,
// o = S^T q.  Inputs are read from global memory (the same 256-byte rows for every thread).
struct ExactIn {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* alpha;
    const float* beta;
    void* o;
    int out_bf16;
    unsigned int* err;      // status word: a non-finite output is flagged there
    int qk_norm;            // the fused prologue and output gate (instances with kF != 0)
    int gate_logits;
    float alpha_scale;
    const __nv_bfloat16* z;
};
// decay_first: (I - beta k k^T) Diag(alpha), e = (alpha . k)^T S, S <- Diag(alpha) S + beta k (v - e)
// kF (FuseBits): alpha and beta from logits, k and q divided by their L2 norms, o times sigmoid(z).
template <bool decay_first, int kF>
__device__ __forceinline__ void exact_body(uint32_t tm_s, const ExactIn& p, int64_t row0, int n, int j)
{
    #pragma unroll 1
    for (int t = 0; t < n; ++t) {
        const int64_t row = row0 + t;
        const __nv_bfloat16* kr = p.k + row * kD;
        const __nv_bfloat16* qr = p.q + row * kD;
        const float* ar = p.alpha + row * kD;
        float b = p.beta[row];
        float ik = 1.f, iq = 1.f;           // inverse L2 norms of k and q (fused prologue)
        {
            if (kF & kFuseLogits) b = sigmoid_fast(b);
            if (kF & kFuseNorm) {
                float nk = 0.f, nq = 0.f;
                #pragma unroll 1
                for (int d8 = 0; d8 < kD; d8 += 8) {
                    const uint4 kw = *reinterpret_cast<const uint4*>(kr + d8);
                    const uint4 qw = *reinterpret_cast<const uint4*>(qr + d8);
                    const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        nk = fmaf(bf16_lo(kk[u]), bf16_lo(kk[u]), fmaf(bf16_hi(kk[u]), bf16_hi(kk[u]), nk));
                        nq = fmaf(bf16_lo(qq[u]), bf16_lo(qq[u]), fmaf(bf16_hi(qq[u]), bf16_hi(qq[u]), nq));
                    }
                }
                ik = inv_l2_fast(nk);
                iq = inv_l2_fast(nq);
            }
        }
        auto alpha_at = [&](float a) { return (kF & kFuseLogits) ? alpha_from_logit_fast(a, p.alpha_scale) : a; };
        const float vj = __bfloat162float(p.v[row * kD + j]);
        float e = 0.f;
        #pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float sv[64];
            tmem_load_2x32(tm_s + 64 * h, tm_s + 64 * h + 32, sv);
            #pragma unroll
            for (int d8 = 0; d8 < 64; d8 += 8) {
                const uint4 kw = *reinterpret_cast<const uint4*>(kr + 64 * h + d8);
                const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
                float4 a0 = make_float4(1.f, 1.f, 1.f, 1.f), a1 = a0;
                if (decay_first) {   // e = (alpha . k)^T S
                    a0 = *reinterpret_cast<const float4*>(ar + 64 * h + d8);
                    a1 = *reinterpret_cast<const float4*>(ar + 64 * h + d8 + 4);
                }
                if ((kF & kFuseLogits) && decay_first) {
                    a0 = make_float4(alpha_at(a0.x), alpha_at(a0.y), alpha_at(a0.z), alpha_at(a0.w));
                    a1 = make_float4(alpha_at(a1.x), alpha_at(a1.y), alpha_at(a1.z), alpha_at(a1.w));
                }
                const float aa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    e = fmaf(bf16_lo(kk[u]) * ik * aa[2 * u], sv[d8 + 2 * u], e);
                    e = fmaf(bf16_hi(kk[u]) * ik * aa[2 * u + 1], sv[d8 + 2 * u + 1], e);
                }
            }
        }
        float o = 0.f;
        #pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float sv[64];
            tmem_load_2x32(tm_s + 64 * h, tm_s + 64 * h + 32, sv);
            #pragma unroll
            for (int d8 = 0; d8 < 64; d8 += 8) {
                const uint4 kw = *reinterpret_cast<const uint4*>(kr + 64 * h + d8);
                const uint4 qw = *reinterpret_cast<const uint4*>(qr + 64 * h + d8);
                float4 a0 = *reinterpret_cast<const float4*>(ar + 64 * h + d8);
                float4 a1 = *reinterpret_cast<const float4*>(ar + 64 * h + d8 + 4);
                if (kF & kFuseLogits) {
                    a0 = make_float4(alpha_at(a0.x), alpha_at(a0.y), alpha_at(a0.z), alpha_at(a0.w));
                    a1 = make_float4(alpha_at(a1.x), alpha_at(a1.y), alpha_at(a1.z), alpha_at(a1.w));
                }
                const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
                const uint32_t qq[4] = {qw.x, qw.y, qw.z, qw.w};
                const float aa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float k0 = bf16_lo(kk[u]) * ik, k1 = bf16_hi(kk[u]) * ik;
                    float& s0 = sv[d8 + 2 * u];
                    float& s1 = sv[d8 + 2 * u + 1];
                    if (decay_first) {
                        s0 = aa[2 * u] * s0 + b * k0 * (vj - e);
                        s1 = aa[2 * u + 1] * s1 + b * k1 * (vj - e);
                    } else {
                        s0 = aa[2 * u] * (s0 - b * k0 * e) + b * k0 * vj;
                        s1 = aa[2 * u + 1] * (s1 - b * k1 * e) + b * k1 * vj;
                    }
                    o = fmaf(bf16_lo(qq[u]) * iq, s0, o);
                    o = fmaf(bf16_hi(qq[u]) * iq, s1, o);
                }
            }
            tmem_st32(tm_s + 64 * h, *reinterpret_cast<float(*)[32]>(sv));
            tmem_st32(tm_s + 64 * h + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
            tmem_wait_st();
        }
        if (kF & kFuseGate) o *= sigmoid_fast(__bfloat162float(p.z[row * kD + j]));
        if (p.out_bf16)
            static_cast<__nv_bfloat16*>(p.o)[row * kD + j] = __float2bfloat16_rn(o);
        else
            static_cast<float*>(p.o)[row * kD + j] = o;
    }
}

// Two entry points with the same body.  The fixed-length kernels pass the inputs as one struct by
// value: measured the lightest call for their register allocation.  The packed-sequence kernels,
// whose parameter block is longer, pass them one by one: with that block, the struct passed by
// value arrived wrong in a measured build.
template <bool decay_first, int kF>
__device__ __noinline__ void exact_chunk(uint32_t tm_s, ExactIn p, int64_t row0, int n, int j)
{
    exact_body<decay_first, kF>(tm_s, p, row0, n, j);
}
template <bool decay_first, int kF>
__device__ __noinline__ void exact_chunk_args(uint32_t tm_s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                             const __nv_bfloat16* v, const float* alpha, const float* beta, void* o,
                                             int out_bf16, int qk_norm, int gate_logits, float alpha_scale,
                                             const __nv_bfloat16* z, int64_t row0, int n, int j)
{
    const ExactIn p{q, k, v, alpha, beta, o, out_bf16, nullptr, qk_norm, gate_logits, alpha_scale, z};
    exact_body<decay_first, kF>(tm_s, p, row0, n, j);
}

// Chain thread j, fp32 output: o[r][j] = (Q^ S)_rj - B_rj for tokens r = r0 .. r0 + 15 below n
// (tm_qs and tm_b address token r0), times sigmoid(z[r][j]) when z (column j of the chunk's
// output gate logits) is given.
__device__ __noinline__ void store_o_f32(uint32_t tm_qs, uint32_t tm_b, float* o, int r0, int n,
                                         const __nv_bfloat16* z)
{
    float qp[32];
    tmem_load_2x16(tm_qs, tm_b, qp);
    #pragma unroll
    for (int r = 0; r < 16; ++r) {
        float ov = qp[r] - qp[16 + r];
        if (z && r0 + r < n) ov *= sigmoid_fast(__bfloat162float(z[(r0 + r) * kD]));
        if (r0 + r < n) o[(r0 + r) * kD] = ov;
    }
}

// Gram [Kt; Qt; -] [Be; Bv]^T (M = 128, N = 64, K = 128) into TMEM, Be and Bv from the chunk
// stage `st`; only lanes 0-63 are read.  Commits the Gram barrier and the release of the Gram
// tiles.
__device__ __forceinline__ void issue_gram(uint32_t sb, uint32_t tmem, uint32_t st, int gbuf)
{
    const uint32_t g = sb + OFF_GRAM + gbuf * GRAM_BUF;
    for (int k = 0; k < 8; ++k) {
        umma_f16(tmem + TM_G, smem_desc_sw128(g + (k >> 2) * GRAM_PANEL + (k & 3) * 32, 16, 1024),
                 smem_desc_sw128(st + ST_KVE + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024), ID_GRAM, k > 0);
    }
    umma_commit(bar_addr(sb, B_G_FULL));
    umma_commit(bar_addr(sb, B_GFREE + gbuf));
}

// Prep warp 4: the Gram of chunk k once its tiles are converted (prep has read the previous
// Gram out of TMEM before it gets here).  Returns 1 if issued; `issuer` is the issuing lane.
__device__ __noinline__ int issue_gram_of(int k, uint32_t sb, uint32_t tmem, int lane, volatile int* abort_flag,
                                          unsigned int* err, uint32_t& issuer)
{
    const bool gok = mbar_wait(bar_addr(sb, B_CONV + k % kStages), (k / kStages) & 1, abort_flag, err, kTimeoutNs);
    if (!__all_sync(0xffffffffu, gok)) return 0;
    tc_fence_after();
    if (elect_one(issuer)) issue_gram(sb, tmem, sb + OFF_STG + (k % kStages) * STAGE_BYTES, k & 1);
    __syncwarp();
    return 1;
}

// kF (FuseBits): the fused steps this instance compiles in -- alpha, beta from logits; k, q rows
// normalised to unit L2 norm while they are converted; the output gate (o <- sigmoid(z) o, z read
// from L1, where the chain prefetches it at the top of the chunk).  One instance per combination,
// so that a call carries the code of the steps it uses only; kF = 0 compiles exactly as without.
template <bool kDecayFirst, int kF, bool kVar>
__global__ void __launch_bounds__(kThreads, 1)
gdr_prefill_kda_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                          const __grid_constant__ CUtensorMap tm_a, KdaParams<kVar> p)
{
    allow_next_loop_to_start();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sbase = smem_raw + (sb - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + OFF_ABORT);
    auto gate = [&](int s) -> Gates* { return reinterpret_cast<Gates*>(sbase + OFF_GATES + s * GATE_STAGE); };
    auto sts = [&](uint32_t addr, uint4 v) { *reinterpret_cast<uint4*>(sbase + (addr - sb)) = v; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ug = p.unit0 + blockIdx.x;             // global head-unit index (states)
    unsigned int* err = p.err;
    // Where the unit's tokens live.  Fixed lengths: unit ug of the tensor maps, rows ug * L + t.
    // Packed sequences: the TMA unit coordinate zv of (loop, head), the sequence's first row y0 and
    // length, and the row index gbase of its first token in the gate, o and z arrays; a bad pair
    // of offsets is reported and the CTA does nothing.
    struct Where { int32_t zv; int64_t y0, len, gbase; bool ok; };
    const Where wh = [&]() -> Where {
        if constexpr (kVar) {
            const int b = blockIdx.x / p.H, hd = blockIdx.x - b * p.H;
            const int64_t c0 = p.cu[b], c1 = p.cu[b + 1];
            const bool ok = 0 <= c0 && c0 <= c1 && c1 <= p.L;
            if (!ok && threadIdx.x == 0) atomicOr(p.err, kDevSeqlens);
            const int32_t zv = p.loop * p.H + hd;
            return Where{zv, ok ? c0 : 0, ok ? c1 - c0 : 0, static_cast<int64_t>(zv) * p.L + (ok ? c0 : 0), ok};
        } else {
            return Where{ug, 0, p.L, 0, true};
        }
    }();
    const int64_t L = wh.len;
    const int32_t zc = kVar ? wh.zv : ug;
    const bool seq_ok = wh.ok;
    // row index of token t0 of the unit in the gate, o and z arrays; its TMA row coordinate
    auto row_of = [&](int64_t t0) -> int64_t { return kVar ? wh.gbase + t0 : static_cast<int64_t>(ug) * L + t0; };
    auto tma_row = [&](int64_t t0) -> int32_t { return static_cast<int32_t>(kVar ? wh.y0 + t0 : t0); };
    const int nchunks = static_cast<int>((L + kC - 1) / kC);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_addr(sb, B_FULL + s), 1);
            mbar_init(bar_addr(sb, B_CONV + s), kConv);
            mbar_init(bar_addr(sb, B_EMPTY + s), 1);
            mbar_init(bar_addr(sb, B_GATE_FULL + s), kConv);
            mbar_init(bar_addr(sb, B_GATE_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_addr(sb, B_TP_FULL + s), 1);
            mbar_init(bar_addr(sb, B_TP_EMPTY + s), 1);
            mbar_init(bar_addr(sb, B_DRAIN + s), 1);
            mbar_init(bar_addr(sb, B_AL_FULL + s), 1);
            mbar_init(bar_addr(sb, B_AL_EMPTY + s), kConv);
        }
        mbar_init(bar_addr(sb, B_G_FULL), 1);
        mbar_init(bar_addr(sb, B_GFREE + 0), 1);
        mbar_init(bar_addr(sb, B_GFREE + 1), 1);
        mbar_init(bar_addr(sb, B_A_FULL), 1);
        mbar_init(bar_addr(sb, B_B_FULL), 1);
        mbar_init(bar_addr(sb, B_S_FULL), 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_TMEM_SLOT, TM_COLS);
        tmem_relinquish();
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_o);
            prefetch_tmap(&tm_a);
        }
    }
    if (warp >= 4 && warp < 8) {
        // zero both [X | Z] stages once: the blocks of X right of its diagonal are never written
        const int t = threadIdx.x - 128;
        for (uint32_t off = t * 16; off < 2 * TP_STAGE; off += 128 * 16) sts(sb + OFF_TP + off, make_uint4(0, 0, 0, 0));
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + OFF_TMEM_SLOT);
    // every TMEM column this CTA addresses lies inside its allocation
    if (threadIdx.x == 0) dbg_ok((tmem & 0xFFFFu) + TM_COLS <= 512u && (tmem >> 16) == 0u, err);

    if (warp == 0) {
        // ================= TMA producer =================
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
#ifdef LT2_DEBUG
            if (c == g_debug_skip_chunk) break;
#endif
            const int s = c % kStages;
            const uint32_t ph = ((c / kStages) & 1) ^ 1;
            int free_ok = 0;
            if (lane == 0)
                free_ok = mbar_wait(bar_addr(sb, B_EMPTY + s), ph, abort_flag, err, kTimeoutNs) &&
                          mbar_wait(bar_addr(sb, B_AL_EMPTY + (c & 1)), ((c >> 1) & 1) ^ 1, abort_flag, err, kTimeoutNs);
            if (!__shfl_sync(0xffffffffu, free_ok, 0)) break;
            uint32_t leader;
            if (elect_one(leader) && dbg_ok(c * kC < L && zc < p.units_total, err)) {
                const uint32_t fb = bar_addr(sb, B_FULL + s);
                mbar_arrive_expect_tx(fb, STAGE_TX);
                const uint32_t st = sb + OFF_STG + s * STAGE_BYTES;
                const int32_t y = tma_row(static_cast<int64_t>(c) * kC);
                tma_load_3d(st + ST_KQ, &tm_k, 0, y, zc, fb);
                tma_load_3d(st + ST_KQ + 8192, &tm_k, 64, y, zc, fb);
                tma_load_3d(st + ST_KQ + 4096, &tm_q, 0, y, zc, fb);
                tma_load_3d(st + ST_KQ + 8192 + 4096, &tm_q, 64, y, zc, fb);
                tma_load_3d(st + ST_V, &tm_v, 0, y, zc, fb);
                tma_load_3d(st + ST_V + 4096, &tm_v, 64, y, zc, fb);
                const uint32_t ab = bar_addr(sb, B_AL_FULL + (c & 1));
                mbar_arrive_expect_tx(ab, ALPHA_STAGE);
                tma_load_3d(sb + OFF_ALPHA + (c & 1) * ALPHA_STAGE, &tm_a, 0, y, zc, ab);
            }
            __syncwarp();
            issued = c + 1;
        }
        if (lane == 0 && *abort_flag) {
            for (int c = issued - kStages < 0 ? 0 : issued - kStages; c < issued; ++c)
                mbar_wait(bar_addr(sb, B_FULL + c % kStages), (c / kStages) & 1, abort_flag, err, kTimeoutNs / 4);
            for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
                mbar_wait(bar_addr(sb, B_AL_FULL + (c & 1)), (c >> 1) & 1, abort_flag, err, kTimeoutNs / 4);
        }
    } else if (warp < 4) {
        // ================= conversion (warps 1-3): decay factors, K/Q/V tiles =================
        const int w = warp - 1;
        const int t_begin = conv_begin(w), t_end = conv_begin(w + 1);
        // the conversion warps wait for the chunk's inputs together and leave the loop together
        Group grp{NB_CONV, 32 * kConv, warp == 1 && lane == 0, abort_flag, err};
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const uint32_t ph = (c / kStages) & 1;
            const uint32_t st = sb + OFF_STG + s * STAGE_BYTES;
            const int64_t t0 = static_cast<int64_t>(c) * kC;
            const int n = static_cast<int>(L - t0 < kC ? L - t0 : kC);
            // beta of token `lane` of this chunk: the load is issued before the waits below, which
            // hide its latency
            float bl = lane < n ? p.beta[row_of(t0) + lane] : 0.f;
            if ((kF & kFuseLogits) && lane < n) bl = sigmoid_fast(bl);
            if (!grp.wait(bar_addr(sb, B_FULL + s), ph, bar_addr(sb, B_GATE_EMPTY + s), ph ^ 1,
                          bar_addr(sb, B_AL_FULL + (c & 1)), (c >> 1) & 1))
                break;
            if (!grp.wait(bar_addr(sb, B_GFREE + (c & 1)), ((c >> 1) & 1) ^ 1)) break;
            float* alpha_c = reinterpret_cast<float*>(sbase + OFF_ALPHA + (c & 1) * ALPHA_STAGE);
            if (kF & kFuseLogits)
                local_products<true>(alpha_c, n, t_begin, t_end, lane, p.alpha_scale);
            else
                local_products<false>(alpha_c, n, t_begin, t_end, lane, 0.f);
            grp.sync();
            float4 Ph;
            const float4 Pt = chunk_products(alpha_c, w, lane, Ph);
            Gates* gs = gate(s);
            // (written as a select between the two instances: the plain kernel's register
            // allocation, measured, is better this way)
            // (packed sequences: the rows of a last, partial chunk past n hold the next sequence's
            // tokens; with beta = 0 and alpha = 1 there they reach only their own rows of E and o,
            // never the state or the rows below n, exactly as the zero rows of fixed lengths do)
            const bool in_range = ((kF & kFuseNorm) && p.qk_norm ? convert_kqv<kDecayFirst, true> : convert_kqv<kDecayFirst, false>)(
                                                           st, sb + OFF_GRAM + (c & 1) * GRAM_BUF, alpha_c, bl, Ph, Pt,
                                                           t_begin, t_end, lane, sbase, sb, gs->sq);
            if (lane == 0) gs->in_range[w] = in_range ? 1 : 0;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar_addr(sb, B_CONV + s));
                mbar_arrive(bar_addr(sb, B_GATE_FULL + s));
                mbar_arrive(bar_addr(sb, B_AL_EMPTY + (c & 1)));
            }
        }
    } else if (warp < 8) {
        // ======= prep: Gram epilogue, diagonal inverses, back substitution, Z; the next Gram =======
        const int t = threadIdx.x - 128;
        const int q = warp - 4;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        Group grp{NB_PREP, 128, t == 0, abort_flag, err};
        float* adiag = reinterpret_cast<float*>(sbase + OFF_ADIAG);
        uint32_t gram_issuer = 0;
        int gram_issued = 0;
        if (warp == 4 && nchunks > 0) gram_issued |= issue_gram_of(0, sb, tmem, lane, abort_flag, err, gram_issuer);
        for (int c = 0; c < nchunks; ++c) {
            const int tps = c & 1;
            if (!grp.wait(bar_addr(sb, B_G_FULL), c & 1, bar_addr(sb, B_TP_EMPTY + tps), ((c >> 1) & 1) ^ 1)) break;
            tc_fence_after();
            if (q < 2) {
                float v[64];
                tmem_load_2x32(tmem + TM_G + lane_addr, tmem + TM_G + lane_addr + 32, v);
                gram_epilogue_row(v, lane, q == 0, sbase, sb, adiag);
            }
            tc_fence_before();
            grp.sync();
            const uint32_t tp = sb + OFF_TP + tps * TP_STAGE;
            if (q == 0) diag_block_inverse_row(tp, lane, adiag + (lane >> 4) * ADIAG_BLOCK);
            grp.sync();
            // warp q: row block q of X = [T; N_qe T] (T rows 0..31, then 32..63), then of Z
            solve_row_block(tp, sb + OFF_MA, 0, sb + OFF_MA, 32, q, 2, lane);
            z_row_block(tp, sb + OFF_MB, q, lane);
            fence_proxy_async_smem();
            grp.sync();
            if (t == 0) mbar_arrive(bar_addr(sb, B_TP_FULL + tps));
            if (warp == 4 && c + 1 < nchunks) gram_issued |= issue_gram_of(c + 1, sb, tmem, lane, abort_flag, err, gram_issuer);
        }
        if (warp == 4 && lane == gram_issuer && gram_issued && *abort_flag) {
            umma_commit(bar_addr(sb, B_DRAIN + 1));
            mbar_wait(bar_addr(sb, B_DRAIN + 1), 0, abort_flag, err, kTimeoutNs / 4);
        }
    } else {
        // ======= the S-dependent chain (lane j = d_v column j of S; half h of the TMEM columns) =======
        const int j = 32 * (warp & 3) + lane;
        const int h = (warp - 8) >> 2;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const bool leader = warp == 8 && lane == 0;
        Group grp{NB_CHAIN, 256, leader, abort_flag, err};
        bool ok = nchunks > 0;
        if constexpr (kVar) {
            // an empty packed sequence: the state passes through unchanged (keys 64 h .. + 63)
            if (nchunks == 0 && seq_ok && p.S_out) {
                const int64_t base = static_cast<int64_t>(ug) * kD * kD + j;
                for (int i = 64 * h; i < 64 * h + 64; ++i) p.S_out[base + i * kD] = p.S0 ? p.S0[base + i * kD] : 0.f;
            }
        }
        uint32_t ph_a = 0, ph_b = 0, ph_s = 0;
        if (ok) ok = grp.wait(bar_addr(sb, B_GATE_FULL + 0), 0);
        if (ok) {
            const Gates* g0 = gate(0);
            const bool exact0 = !gates_in_range(g0);
            load_initial_state(tmem + TM_S + lane_addr, tmem + TM_SH + lane_addr,
                               p.S0 ? p.S0 + static_cast<int64_t>(ug) * kD * kD + j : nullptr,
                               exact0 ? nullptr : g0->sq, 2 * h);
            tc_fence_before();
        }
        uint32_t drain_needed = 0;
        uint32_t mma_issuer = 0;
        // the previous chunk's gate stage, released after the next group barrier (-1: none)
        int pend_gate = -1;
        for (int c = 0; ok && c < nchunks; ++c) {
            const int s = c % kStages;
            const uint32_t ph = (c / kStages) & 1;
            const int tps = c & 1;
            const uint32_t st = sb + OFF_STG + s * STAGE_BYTES;
            const uint32_t tp = sb + OFF_TP + tps * TP_STAGE;
            const int64_t t0 = static_cast<int64_t>(c) * kC;
            const int n = static_cast<int>(L - t0 < kC ? L - t0 : kC);
            const Gates* gs = gate(s);
            const bool exact = !gates_in_range(gs);
            const bool last = c + 1 == nchunks;
            const int s1 = (c + 1) % kStages;
            if ((kF & kFuseGate) && j < 2 * n) {
                // the chunk's output gate logits (n rows of 256 bytes, two lines a row) into L1,
                // for the output epilogue that runs under MMA_C
                const __nv_bfloat16* zl = p.z + (row_of(t0) + (j >> 1)) * kD + (j & 1) * 64;
                asm volatile("prefetch.global.L1 [%0];" ::"l"(zl));
            }
            if (!exact) {
                // --- MMA_A: (K^ S, Q^ S)^T = S^T [K^; Q^]^T ---
                grp.sync();
                if (leader && pend_gate >= 0) mbar_arrive(bar_addr(sb, B_GATE_EMPTY + pend_gate));
                pend_gate = -1;
                if (warp == 8) {
                    const bool lok = mbar_wait(bar_addr(sb, B_CONV + s), ph, abort_flag, err, kTimeoutNs);
                    if (__all_sync(0xffffffffu, lok)) {
                        tc_fence_after();
                        if (elect_one(mma_issuer)) {
                            for (int k = 0; k < 8; ++k) {
                                const uint32_t boff = ST_KQ + (k >> 2) * 8192 + (k & 3) * 32;
                                umma_f16_tmem_a(tmem + TM_AB, tmem + TM_SH + 8 * k,
                                                smem_desc_sw128(st + boff, 16, 1024), ID_T64, k > 0);
                            }
                            umma_commit(bar_addr(sb, B_A_FULL));
                        }
                        __syncwarp();
                        drain_needed = 1;
                    }
                }
                ok = grp.wait(bar_addr(sb, B_A_FULL), ph_a);
                ph_a ^= 1u;
                if (!ok) break;
                tc_fence_after();
                // --- (K^ S)^T as fp16 pairs: the second A operand of MMA_B (tokens 16h .. + 15) ---
                {
                    float ks[16];
                    tmem_load16(tmem + TM_AB + lane_addr + 16 * h, ks);
                    uint32_t hpk[8];
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) hpk[e] = pack_half2(ks[2 * e], ks[2 * e + 1]);
                    tmem_st8(tmem + TM_Y + lane_addr + 8 * h, hpk);
                    tmem_wait_st();
                }
                tc_fence_before();
                grp.sync();
                // --- MMA_B: ([E; -O'])^T = V^T Z^T + (K^ S)^T X^T ---
                if (warp == 8) {
                    const bool tok = mbar_wait(bar_addr(sb, B_TP_FULL + tps), (c >> 1) & 1, abort_flag, err, kTimeoutNs);
                    if (__all_sync(0xffffffffu, tok)) {
                        tc_fence_after();
                        if (elect_one(mma_issuer)) {
                            for (int k = 0; k < 2; ++k)
                                umma_f16(tmem + TM_B, smem_desc_sw128(st + ST_V + k * 2048, 4096, 1024),
                                         smem_desc_sw128(tp + 2 * TP_ZCOL + k * 32, 16, 1024), ID_M64, k > 0);
                            for (int k = 0; k < 2; ++k)
                                umma_f16_tmem_a(tmem + TM_B, tmem + TM_Y + 8 * k, smem_desc_sw128(tp + k * 32, 16, 1024),
                                                ID_T64, 1);
                            umma_commit(bar_addr(sb, B_B_FULL));
                            umma_commit(bar_addr(sb, B_TP_EMPTY + tps));
                        }
                        __syncwarp();
                    }
                }
                ok = grp.wait(bar_addr(sb, B_B_FULL), ph_b);
                ph_b ^= 1u;
                if (!ok) break;
                tc_fence_after();
                // --- -E^T as fp16 pairs: the A operand of the E half of MMA_C (tokens 16h .. + 15) ---
                {
                    float ev[16];
                    tmem_load16(tmem + TM_B + lane_addr + 16 * h, ev);
                    uint32_t hpk[8];
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) hpk[e] = pack_half2(-ev[2 * e], -ev[2 * e + 1]);
                    tmem_st8(tmem + TM_E + lane_addr + 8 * h, hpk);
                    tmem_wait_st();
                }
                if (leader) bulk_wait_read_all();      // the previous chunk's o store has left the staging
                tc_fence_before();
                grp.sync();
                // --- MMA_C: (sq S)^T += V^T Bv - E^T Be ---
                if (warp == 8) {
                    tc_fence_after();
                    if (elect_one(mma_issuer)) {
                        for (int k = 0; k < 2; ++k)
                            umma_f16(tmem + TM_S, smem_desc_sw128(st + ST_V + k * 2048, 4096, 1024),
                                     smem_desc_sw128(st + ST_KVE + 4096 + k * 2048, 8192, 1024), ID_MM, 1);
                        for (int k = 0; k < 2; ++k)
                            umma_f16_tmem_a(tmem + TM_S, tmem + TM_E + 8 * k,
                                            smem_desc_sw128(st + ST_KVE + k * 2048, 8192, 1024), ID_TM, 1);
                        umma_commit(bar_addr(sb, B_S_FULL));
                        umma_commit(bar_addr(sb, B_EMPTY + s));
                    }
                    __syncwarp();
                }
                // --- while MMA_C runs: o = Q^ S - (the -O' half of MMA_B), tokens 16h .. + 15 ---
                // (out-of-range operands are flagged through the final state: a state that left
                // the fp16 range carries infinities or NaNs to the end of the sequence)
                if (!p.out_bf16) {
                    store_o_f32(tmem + TM_AB + lane_addr + 32 + 16 * h, tmem + TM_B + lane_addr + 32 + 16 * h,
                                     static_cast<float*>(p.o) + row_of(t0) * kD + j, 16 * h, n,
                                     (kF & kFuseGate) ? p.z + row_of(t0) * kD + j : nullptr);
                } else {
                    float qp[32];
                    tmem_load_2x16(tmem + TM_AB + lane_addr + 32 + 16 * h, tmem + TM_B + lane_addr + 32 + 16 * h, qp);
                    uint8_t* ost = sbase + OFF_OST + (j >> 6) * 4096 + (j & 63) * 2 + 16 * h * 128;
                    // the fused output gate: column j of the chunk's logits, prefetched to L1
                    const __nv_bfloat16* zr = (kF & kFuseGate) ? p.z + (row_of(t0) + 16 * h) * kD + j : nullptr;
                    #pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float ov = qp[r] - qp[16 + r];
                        if ((kF & kFuseGate) && 16 * h + r < n) ov *= sigmoid_fast(__bfloat162float(zr[r * kD]));
                        *reinterpret_cast<__nv_bfloat16*>(ost + r * 128) = __float2bfloat16_rn(ov);
                    }
                    fence_proxy_async_smem();
                }
                // MMA_C done, and the next chunk's gates written
                ok = grp.wait(bar_addr(sb, B_S_FULL), ph_s, last ? 0u : bar_addr(sb, B_GATE_FULL + s1),
                              ((c + 1) / kStages) & 1);
                ph_s ^= 1u;
                if (!ok) break;
                tc_fence_after();
                if (kVar && t0 + kC > L) {
                    // a packed sequence's last, partial chunk: the rows past its end belong to the
                    // next sequence, so its n rows leave by plain 16-byte stores (both 64-column
                    // halves of a row: 16 pieces), not by the two box stores
                    if (p.out_bf16) {
                        __nv_bfloat16* orow0 = static_cast<__nv_bfloat16*>(p.o) + row_of(t0) * kD;
                        for (int i = threadIdx.x - 256; i < n * 16; i += 256) {
                            const int r = i >> 4, part = i & 15;
                            const uint4 w = *reinterpret_cast<const uint4*>(sbase + OFF_OST + (part >> 3) * 4096 +
                                                                            r * 128 + (part & 7) * 16);
                            *reinterpret_cast<uint4*>(orow0 + static_cast<int64_t>(r) * kD + (part >> 3) * 64 +
                                                      (part & 7) * 8) = w;
                        }
                    }
                } else if (leader && p.out_bf16 && dbg_ok(t0 < L && zc < p.units_total, err)) {
                    tma_store_3d(&tm_o, sb + OFF_OST, 0, tma_row(t0), zc);
                    tma_store_3d(&tm_o, sb + OFF_OST + 4096, 64, tma_row(t0), zc);
                    bulk_commit_group();
                }
            } else {
                // --- out-of-range chunk: the definition, token by token, on the fp32 state (the
                // first half of the chain's warps; every key of a column takes part in k^T S) ---
                // The state's keys 64-127 were written by the second half (the initial state or the
                // last update): the group barrier orders those TMEM stores before these loads.
                grp.sync();
                tc_fence_after();
                if (h == 0) {
                    if constexpr (kVar)
                        exact_chunk_args<kDecayFirst, kF>(tmem + TM_S + lane_addr, p.q, p.k, p.v, p.alpha, p.beta,
                                                          p.o, p.out_bf16, p.qk_norm, p.gate_logits, p.alpha_scale,
                                                          p.z, row_of(t0), n, j);
                    else
                        exact_chunk<kDecayFirst, kF>(tmem + TM_S + lane_addr,
                                                     ExactIn{p.q, p.k, p.v, p.alpha, p.beta, p.o, p.out_bf16, err,
                                                             p.qk_norm, p.gate_logits, p.alpha_scale, p.z},
                                                     row_of(t0), n, j);
                }
                tc_fence_before();
                // keep every hand-off in step: the stage and the [X; Z] stage are released
                // once their producers are done with them, the output epilogue is released
                ok = grp.wait(bar_addr(sb, B_CONV + s), ph, bar_addr(sb, B_TP_FULL + tps), (c >> 1) & 1,
                              last ? 0u : bar_addr(sb, B_GATE_FULL + s1), ((c + 1) / kStages) & 1);
                if (!ok) break;
                tc_fence_after();                       // the first half's TMEM stores, for the update
                if (leader) {
                    mbar_arrive(bar_addr(sb, B_EMPTY + s));
                    mbar_arrive(bar_addr(sb, B_TP_EMPTY + tps));
                    if (pend_gate >= 0) mbar_arrive(bar_addr(sb, B_GATE_EMPTY + pend_gate));
                }
                pend_gate = -1;
            }
            // --- the new state ---
            // TM_S holds S' / sq after a tensor-core chunk, S' itself after an exact one
            const float* f_sh = exact ? nullptr : gs->sq;
            if (last) {
                if (p.S_out && !store_final_state_scaled(tmem + TM_S + lane_addr,
                                                         p.S_out + static_cast<int64_t>(ug) * kD * kD + j, f_sh, 2 * h))
                    atomicOr(err, kDevRange);
                drain_needed = 0;
            } else {
                const Gates* g1 = gate(s1);
                const bool exact1 = !gates_in_range(g1);
                state_update(tmem + TM_S + lane_addr, tmem + TM_SH + lane_addr, f_sh, exact1 ? nullptr : g1->sq, 2 * h);
                tc_fence_before();
                pend_gate = s;
            }
        }
        if (warp == 8 && lane == mma_issuer && drain_needed && !ok) {
            umma_commit(bar_addr(sb, B_DRAIN + 0));
            mbar_wait(bar_addr(sb, B_DRAIN + 0), 0, abort_flag, err, kTimeoutNs / 4);
        }
        if (leader) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace kda

bool prefill_kda_tc_supports(int dtype_bf16, int dk, int dv)
{
    return dtype_bf16 && dk == kda::kD && dv == kda::kD;
}

namespace kda {
namespace {
// One launch per loop of the instance for this layout, order of the per-key factors and
// combination of fused steps (kVar: packed sequences, the ParamsVar block).  Internal linkage: a
// template's static table would otherwise be one object per process, shared with any other copy
// of this library loaded alongside (the debug build), whose kernels are not this library's.
template <bool kVar>
cudaError_t launch_loops(const TcCall& call, int64_t map_units, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mo, const CUtensorMap& ma, cudaStream_t stream)
{
    using K = decltype(&gdr_prefill_kda_tc_kernel<false, 0, kVar>);
    static const K kernels[2][8] = {
        {gdr_prefill_kda_tc_kernel<false, 0, kVar>, gdr_prefill_kda_tc_kernel<false, 1, kVar>,
         gdr_prefill_kda_tc_kernel<false, 2, kVar>, gdr_prefill_kda_tc_kernel<false, 3, kVar>,
         gdr_prefill_kda_tc_kernel<false, 4, kVar>, gdr_prefill_kda_tc_kernel<false, 5, kVar>,
         gdr_prefill_kda_tc_kernel<false, 6, kVar>, gdr_prefill_kda_tc_kernel<false, 7, kVar>},
        {gdr_prefill_kda_tc_kernel<true, 0, kVar>, gdr_prefill_kda_tc_kernel<true, 1, kVar>,
         gdr_prefill_kda_tc_kernel<true, 2, kVar>, gdr_prefill_kda_tc_kernel<true, 3, kVar>,
         gdr_prefill_kda_tc_kernel<true, 4, kVar>, gdr_prefill_kda_tc_kernel<true, 5, kVar>,
         gdr_prefill_kda_tc_kernel<true, 6, kVar>, gdr_prefill_kda_tc_kernel<true, 7, kVar>}};
    const K kernel = kernels[call.decay_first ? 1 : 0][fuse_bits(call)];
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess) return e;
    for (int64_t tau = 0; tau < call.T; ++tau) {
        NvtxRange loop_range("lt2 prefill loop (tensor core, per-key gating)");
        KdaParams<kVar> p;
        p.q = static_cast<const __nv_bfloat16*>(call.q);
        p.k = static_cast<const __nv_bfloat16*>(call.k);
        p.v = static_cast<const __nv_bfloat16*>(call.v);
        p.alpha = call.alpha;
        p.beta = call.beta;
        p.S0 = call.S0;
        p.o = call.o;
        p.S_out = call.S_out;
        p.L = call.L;
        p.unit0 = static_cast<int>(tau * call.units_per_loop);
        p.units_total = static_cast<int>(map_units);
        p.out_bf16 = call.out_bf16;
        p.err = call.err;
        p.qk_norm = call.qk_norm;
        p.gate_logits = call.gate_logits;
        p.alpha_scale = call.alpha_scale;
        p.z = static_cast<const __nv_bfloat16*>(call.z);
        if constexpr (kVar) {
            p.cu = call.cu_seqlens;
            p.H = static_cast<int>(call.H);
            p.loop = static_cast<int>(tau);
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(call.units_per_loop), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = tau > 0 ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, mo, ma, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
}  // namespace
}  // namespace kda

cudaError_t launch_prefill_kda_tc_all(const TcCall& call, cudaStream_t stream)
{
    using namespace kda;
    if (call.units_per_loop == 0 || call.T == 0) return cudaSuccess;
    const bool var = call.cu_seqlens != nullptr;
    // TMA unit axis and row extent: [T*B*H][L] for fixed lengths, [T*H][Ntot] for packed sequences
    const int64_t units = call.T * call.units_per_loop;
    const int64_t map_units = var ? call.T * call.H : units;
    CUtensorMap mq, mk, mv, mo;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_bf16_map_3d(&mq, call.q, map_units, call.L, kC, sw) ||
        !make_bf16_map_3d(&mk, call.k, map_units, call.L, kC, sw) ||
        !make_bf16_map_3d(&mv, call.v, map_units, call.L, kC, sw))
        return cudaErrorInvalidValue;
    if (call.out_bf16 && !make_bf16_map_3d(&mo, call.o, map_units, call.L, kC, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    CUtensorMap ma;
    if (!make_f32_map_3d(&ma, call.alpha, map_units, call.L, kC)) return cudaErrorInvalidValue;
    // (o's map is only read with bf16 output; a copy of a valid map stands in otherwise)
    const CUtensorMap& mo_or = call.out_bf16 ? mo : mv;
    return var ? launch_loops<true>(call, map_units, mq, mk, mv, mo_or, ma, stream)
               : launch_loops<false>(call, map_units, mq, mk, mv, mo_or, ma, stream);
}

}  // namespace lt2

#ifdef LT2_DEBUG
namespace lt2 {
cudaError_t debug_set_skip_chunk_per_key(int chunk)
{
    return cudaMemcpyToSymbol(kda::g_debug_skip_chunk, &chunk, sizeof(chunk));
}
}  // namespace lt2
#endif
