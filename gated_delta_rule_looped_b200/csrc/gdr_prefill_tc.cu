// gdr_prefill_tc.cu -- chunked prefill of the gated delta rule on Blackwell tensor cores
// (tcgen05 MMA with TMEM accumulators and TMEM operands, tiles staged by TMA), scalar gating,
// d_k = d_v = 128.
//
// The recurrence ("LT2 transformer looped a tempo lineare", section "Sostituire il motore",
// displayed equation)  S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T  with
// the readout o_t = S_t^T q_t is evaluated 64 tokens ("a chunk") at a time.  With the chunk's
// incoming state S, G_r = sum_{s<=r} log alpha_s, g_r = exp(G_r):
//
//   A_rs = beta_s e^{G_r-G_s} k_r.k_s  (s < r),   P_rs = beta_s e^{G_r-G_s} q_r.k_s  (s <= r)
//   T    = (I + A)^{-1}                              (unit lower triangular, 64 x 64)
//   X    = V - diag(g) K S                           (64 x d_v)
//   U    = T X,     o = diag(g) Q S + (P T) X
//   S'   = g_63 S + K^T diag(beta_s e^{G_63-G_s}) U
//
// (u_r = v_r - alpha_r S_{r-1}^T k_r unrolls the chunk; the identity is checked in fp64 by
// the test suite's chunked oracle.)  Everything that does not involve S -- the Gram products
// K K^T and Q K^T, the solve, P T -- is done ahead of the S-dependent chain.
//
// The chain works on the transposed quantities, one d_v column per TMEM lane, so that every
// S-dependent MMA operand is produced in tensor memory and never goes through shared memory:
//
//   MMA_A  (KQ S)^T  = S^T [K;Q]^T          A = S^T (TMEM, fp16)     B = [K;Q] tile
//   MMA_B  ([T;PT] X)^T = V^T [T;PT]^T + (-g K S)^T [T;PT]^T
//                                           A = V^T (smem) then (-g K S)^T (TMEM)   B = [T;PT]
//   MMA_C  S^T += U~^T K                    A = U~^T (TMEM, fp16)    B = K tile
//
// all M = 128 (d_v), N = 128.  The fp32 state S^T stays in TMEM for the whole sequence; its
// fp16 copy (the A operand of MMA_A) is rewritten once per chunk.
//
// Precision.  All MMA operands are fp16 (10-bit mantissa), not bf16: with bf16
// intermediates (S, X, [T;PT], U~ rounded to 8 significant bits) the error against the
// fp64 oracle reaches ~3% of rms(o) at the largest outputs, while fp16 keeps it near 0.5%.
// q, k, v arrive in bf16; converting a bf16 tile to fp16 in shared memory is exact for the
// magnitudes involved (|x| in [2^-14, 2^15]), so the inputs are not rounded again.
//
// CTA = one (loop, batch, head) unit, 16 warps:
//   warp 0       TMEM allocation, TMA producer and issuer of the chain's MMAs (MMA_A, MMA_B,
//                MMA_C): one loop that waits for each MMA's operands and issues it
//   warp 1       chunk gates, fp16 conversion of K, and the Gram MMA [K; Q] K^T
//   warps 2, 3   fp16 conversion of Q and of V
//   warps 4-7    "prep": Gram epilogue, the 64x64 triangular solve (16x16 blocks with
//                warp-level mma.sync), P T; writes [T; PT] for MMA_B
//   warps 8-11   the S-dependent chain: each thread arrives on a 128-count barrier once its
//                part of an MMA operand is in TMEM, and the issuer starts the MMA
//   warps 12-15  output epilogue: o = g (Q S) + P T X from TMEM to global memory
// Every wait on an mbarrier is bounded (see mbar_wait); a group's threads all poll and then
// agree on the outcome through one barrier reduction, so a timeout leaves every thread of the
// group on the same path.  On a timeout the CTA records it in the device status word, drains
// its in-flight copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "gdr_common.cuh"
#include "gdr_launch.h"
#include "gdr_nvtx.h"
#include "gdr_tc_common.cuh"
#include "gdr_tma_host.h"
#include "sm100_primitives.cuh"

namespace lt2 {
namespace tc {

using namespace sm100;
using namespace tcc;

constexpr int kC = 64;                 // tokens per chunk
constexpr int kThreads = 512;
constexpr int kStages = 3;             // K/Q/V tile stages (and gate stages)
constexpr uint64_t kTimeoutNs = kWaitTimeoutNs;

// Shared memory map (offsets from a 1024-byte aligned base).  A K/Q/V stage holds, as fp16
// after conversion, [K panel 0 | Q panel 0 | K panel 1 | Q panel 1 | V panel 0 | V panel 1],
// each panel 64 rows x 128 bytes with the 128-byte swizzle.
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t STAGE_BYTES = KQ_BYTES + V_BYTES;
constexpr uint32_t TP_STAGE = 16384;   // [T; PT], 128 rows x 64 fp16
constexpr uint32_t OFF_KQV = 0;
constexpr uint32_t OFF_TP = OFF_KQV + kStages * STAGE_BYTES;
constexpr uint32_t OFF_OST = OFF_TP + 2 * TP_STAGE;   // o staging for the TMA store: 2 x [64 tokens][64] bf16
constexpr uint32_t OFF_AS = OFF_OST + 16384;          // A (fp16) [64][64]
constexpr uint32_t OFF_PS = OFF_AS + 8192;            // P (fp16) [64][64]
constexpr uint32_t OFF_ADIAG = OFF_PS + 8192;         // diagonal 16x16 blocks of A, fp32, rows padded to 17
constexpr uint32_t ADIAG_BLOCK = 16 * kAdiagRow;
constexpr uint32_t OFF_GATES = OFF_ADIAG + 4608;
constexpr uint32_t GATE_STAGE = 1536;
constexpr uint32_t OFF_BAR = OFF_GATES + kStages * GATE_STAGE;
constexpr uint32_t BAR_BYTES = 512;
constexpr uint32_t SMEM_USED = OFF_BAR + BAR_BYTES;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;     // slack for aligning the base

struct Gates {
    float G[kC];       // chunk-local cumulative log-decay
    float gam[kC];     // e^{G_r}
    float bein[kC];    // beta_s e^{-G_s} (valid when `safe`)
    float beta[kC];    // beta_s (0 beyond the sequence end)
    float bgc[kC];     // beta_s e^{G_63 - G_s}
    float gC;          // e^{G_63}
    int safe;          // e^{-G} representable: A/P use the factored decay
};
static_assert(sizeof(Gates) <= GATE_STAGE, "gate stage too small");

// Barrier slots (8 bytes each) inside the OFF_BAR area.
enum Bar : uint32_t {
    B_FULL = 0,        // [3] TMA of a K/Q/V stage landed (tx count)
    B_CONV = 3,        // [3] K, Q, V of a stage converted to fp16 (3 arrivals)
    B_EMPTY = 6,       // [3] MMAs done with a K/Q/V stage
    B_GATE_FULL = 9,   // [3]
    B_GATE_EMPTY = 12, // [3] prep, chain and output epilogue done with a gate stage
    B_TP_FULL = 15,    // [2]
    B_TP_EMPTY = 17,   // [2]
    B_G_FULL = 19,     // Gram in TMEM
    B_G_EMPTY = 20,    // Gram read out
    B_A_FULL = 21,     // MMA_A done
    B_B_FULL = 22,     // MMA_B done
    B_S_FULL = 23,     // MMA_C done
    B_O_READY = 24,    // output epilogue may read its TMEM columns
    B_O_DONE = 25,     // output epilogue has read them
    B_DRAIN = 26,      // [2] drain on abort (chain, Gram issuer)
    B_Z = 28,          // output gate logits of a chunk landed in the staging tile (fused instance)
    B_SH_READY = 29,   // the chain wrote the fp16 state copy (initial state, then after each chunk)
    B_Y_READY = 30,    // the chain wrote (-g K S)^T: MMA_B may go
    B_U_READY = 31,    // the chain wrote U~^T: MMA_C may go
    B_COUNT = 32
};
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + B_COUNT * 8;        // tcgen05.alloc result
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 16;
// Balanced launches: this CTA's segments (count, then {unit, first chunk, end chunk, flags}).
constexpr int kMaxSeg = 8;
constexpr uint32_t OFF_SEGS = OFF_ABORT + 16;
static_assert(OFF_SEGS + 16 + kMaxSeg * 16 <= OFF_BAR + BAR_BYTES, "barrier area too small");
constexpr int kSegIn = 1;              // the segment's first state is handed over (flag, then S_out)
constexpr int kSegOut = 2;             // the segment's last state is handed on (S_out, then flag)

// Named barriers (bar.sync ids; 0 is __syncthreads).
constexpr int NB_PREP = 1;             // warps 4-7
constexpr int NB_CHAIN = 2;            // warps 8-11
constexpr int NB_OUT = 3;              // warps 12-15

// TMEM columns (128 lanes; lane j = d_v index in the chain's regions).
constexpr uint32_t TM_G = 0;           // Gram [K;Q] K^T (fp32, 64 columns; lane = token row)
constexpr uint32_t TM_S = 64;          // S^T, fp32 (128 columns)
constexpr uint32_t TM_SH = 192;        // S^T, fp16 pairs (64 columns): A operand of MMA_A
constexpr uint32_t TM_AB = 256;        // (KQ S)^T fp32 (128 columns); later the A operands:
constexpr uint32_t TM_Y = 256;         //   (-g K S)^T fp16 pairs (32 columns), MMA_B
constexpr uint32_t TM_U = 288;         //   U~^T fp16 pairs (32 columns), MMA_C
constexpr uint32_t TM_B = 384;         // ([T;PT] X)^T fp32 (128 columns)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_GRAM = idesc_f16_f32(128, 64, 0, 0);    // A, B K-major
constexpr uint32_t ID_TK = idesc_f16_f32(128, 128, 0, 0);     // A in TMEM, B K-major
constexpr uint32_t ID_MK = idesc_f16_f32(128, 128, 1, 0);     // A MN-major (smem), B K-major
constexpr uint32_t ID_TM = idesc_f16_f32(128, 128, 0, 1);     // A in TMEM, B MN-major

struct Params {
    const float* alpha;    // [units_total][L]
    const float* beta;
    const float* S0;       // [units_total][128][128] or null
    void* o;               // [units_total][L][128]
    float* S_out;          // nullable
    int64_t L;
    int unit0;             // first unit of this loop in the flattened [T*B*H] order
    int units_total;       // T*B*H (the extent of the tensor maps' unit axis)
    int out_bf16;
    unsigned int* err;
    // fused prologue and output gate (used by the instances that compile the step in)
    int qk_norm;
    int gate_logits;
    float alpha_scale;
    // packed sequences (the varlen instances): q/k/v/o [T][H][Ntot][128], gates [T][H][Ntot], CTA
    // = (sequence b, head h) of loop `loop`, tokens cu[b] .. cu[b+1]-1
    const int64_t* cu;
    int64_t Ntot;
    int H;
    int loop;
    // balanced launches (one launch for every loop): the units' chunks laid end to end, bal_per_cta
    // of them per CTA; a unit split between two CTAs hands its state over through S_out, and
    // bal_flags[unit] (zeroed before the launch) says when
    int bal_units;
    int bal_chunks;
    int bal_per_cta;
    unsigned int* bal_flags;
};

// Bounded wait for a handoff flag set by another CTA of the same launch (acquire).
__device__ __noinline__ bool wait_handoff(const unsigned int* f, volatile int* abort_flag, unsigned int* err)
{
    uint64_t t0 = 0;
    for (uint32_t it = 1;; ++it) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v) return true;
        if (*abort_flag) return false;
        const uint64_t now = global_timer_ns();
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            atomicOr(err, 1u);
            return false;
        }
        __nanosleep(200);
    }
}

#ifdef LT2_DEBUG
// Fault injection of the debug build: the producer stops before this chunk (-1: never), so its
// copies never arrive and the waits for them run out.
__device__ int g_debug_skip_chunk = -1;
#endif

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, uint32_t i) { return base + OFF_BAR + 8u * i; }

// Gram products [K; Q] K^T of stage s (M=128, N=64, K=128) into TMEM, then commit.
__device__ __forceinline__ void issue_gram(uint32_t sb, uint32_t tmem, int s)
{
    const uint32_t kq = sb + OFF_KQV + s * STAGE_BYTES;
    for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
        umma_f16(tmem + TM_G, smem_desc_sw128(kq + off, 16, 1024), smem_desc_sw128(kq + off, 16, 1024),
                 ID_GRAM, k > 0);
    }
    umma_commit(bar_addr(sb, B_G_FULL));
}

// ---- cold paths, kept out of line so that the per-chunk code stays compact ----------------

// Chain thread j: S0^T row j (column j of S0, or zeros) into TMEM, as fp16 pairs for MMA_A and
// as fp32 pre-scaled by the first chunk's decay g0.
__device__ __noinline__ void load_initial_state(uint32_t tm_s, uint32_t tm_sh, const float* s0, float g0)
{
    #pragma unroll 1
    for (int piece = 0; piece < 4; ++piece) {
        float v[32];
        #pragma unroll
        for (int d = 0; d < 32; ++d) v[d] = s0 ? s0[(32 * piece + d) * kD] : 0.f;
        uint32_t hpk[16];
        #pragma unroll
        for (int e = 0; e < 16; ++e) hpk[e] = pack_half2(v[2 * e], v[2 * e + 1]);
        tmem_st16(tm_sh + 16 * piece, hpk);
        #pragma unroll
        for (int d = 0; d < 32; ++d) v[d] *= g0;
        tmem_st32(tm_s + 32 * piece, v);
    }
    tmem_wait_st();
}

// Output thread j, fp32 output: o[r][j] = g_r (Q S)_rj + (P T X)_rj for the chunk's n tokens,
// times sigmoid(z[r][j]) when `zst` points at column j of the output gate in the staging tile
// (rows 128 bytes apart; the gate already taken through the sigmoid, fp16).  Returns false if any
// of them is not finite.
__device__ __noinline__ bool store_o_f32(uint32_t tm_qs, uint32_t tm_ptx, const float* gam, float* o, int n,
                                         const uint8_t* zst)
{
    bool fin = true;
    #pragma unroll 1
    for (int piece = 0; piece < 2; ++piece) {
        float qp[64];
        tmem_load_2x32(tm_qs + 32 * piece, tm_ptx + 32 * piece, qp);
        #pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int r = 32 * piece + e;
            float ov = gam[r] * qp[e] + qp[32 + e];
            if (zst) ov *= __half2float(*reinterpret_cast<const __half*>(zst + r * 128));
            if (r < n) {
                fin &= is_finite(ov);
                o[r * kD] = ov;
            }
        }
    }
    return fin;
}

// Prep thread t, chunks whose decay e^{-G} is not representable: row r of -A (t < 64) or of P
// with the unfactored e^{G_r - G_s}, masked to s < r (A) or s <= r (P), 8 columns at a time,
// to the fp16 tile `dst` and (A rows) the fp32 diagonal-block copy.
__device__ __noinline__ void gram_epilogue_unfactored(uint32_t tm_row, const Gates* gs, int r, bool is_a,
                                                      uint8_t* dst_ptr, uint32_t dst, float* adiag_row)
{
    const int lim = is_a ? r : r + 1;
    // the sign of the decay ratio is the product of the signs of gam_r and gam_s
    const float sg = copysignf(1.f, gs->gam[r]) * (is_a ? -1.f : 1.f);
    const float Gr = gs->G[r];
    #pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
        float v[8];
        tmem_load8(tm_row + 8 * ch, v);
        #pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int sc = 8 * ch + e;
            const float ss = gs->beta[sc] * copysignf(1.f, gs->gam[sc]);
            v[e] = (sc < lim) ? sg * ss * __expf(Gr - gs->G[sc]) * v[e] : 0.f;
        }
        if (is_a && (ch >> 1) == (r >> 4)) {
            #pragma unroll
            for (int e = 0; e < 8; ++e) adiag_row[(ch & 1) * 8 + e] = v[e];
        }
        *reinterpret_cast<uint4*>(dst_ptr + (sw128(dst, r, ch) - dst)) = pack8_half(v);
    }
}

// kF: the fused steps this instance compiles in (bits of FuseBits): q, k rows normalised to unit
// L2 norm while they are converted to fp16; alpha, beta from logits in the gate warp; the output
// gate (the logits z of a chunk are loaded by TMA into the o staging tile, and o <- sigmoid(z) o
// is applied as the tile is written).  One instance per combination, so that a call carries the
// code of the steps it uses only; kF = 0 compiles exactly as without them.
template <int kF, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
gdr_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_z, Params p, int use_pdl)
{
    (void)use_pdl;
    allow_next_loop_to_start();
    constexpr bool kVar = kMode == 1;       // packed sequences
    constexpr bool kBal = kMode == 2;       // balanced: segments of units, one launch for every loop

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;        // 1024-aligned base (swizzle atoms)
    uint8_t* sbase = smem_raw + (sb - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + OFF_ABORT);
    auto gate = [&](int s) -> Gates* {
        return reinterpret_cast<Gates*>(sbase + OFF_GATES + s * GATE_STAGE);
    };
    // Plain shared-memory accesses by absolute shared address (so the compiler can batch and
    // schedule them); ordering with other threads and with the async proxy comes from the
    // barriers and proxy fences, which are memory-clobbering asm statements.
    auto lds = [&](uint32_t addr) -> uint4 { return *reinterpret_cast<const uint4*>(sbase + (addr - sb)); };
    auto sts = [&](uint32_t addr, uint4 v) { *reinterpret_cast<uint4*>(sbase + (addr - sb)) = v; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ug = p.unit0 + blockIdx.x;               // global head-unit index (states)
    unsigned int* err = p.err;
    // Where the unit's tokens live: the TMA unit coordinate zc, the first row y0 and the length L
    // of the unit, and the element index gbase of its first token in the gate arrays (and, times
    // 128, in o).  Packed sequences take them from the offsets; a bad pair of offsets is reported
    // and the CTA does nothing.
    int32_t zc = ug;
    int64_t y0 = 0, L = p.L, gbase = static_cast<int64_t>(ug) * p.L;
    bool seq_ok = true;
    if constexpr (kVar) {
        const int b = blockIdx.x / p.H, h = blockIdx.x - b * p.H;
        const int64_t c0 = p.cu[b], c1 = p.cu[b + 1];
        seq_ok = 0 <= c0 && c0 <= c1 && c1 <= p.Ntot;
        if (!seq_ok && threadIdx.x == 0) atomicOr(err, kDevSeqlens);
        zc = p.loop * p.H + h;
        y0 = seq_ok ? c0 : 0;
        L = seq_ok ? c1 - c0 : 0;
        gbase = static_cast<int64_t>(zc) * p.Ntot + y0;
    }
    // this CTA's chunks: one unit's, or (balanced) the range [bal_a, bal_b) of all units' chunks
    // laid end to end
    const int64_t bal_a = kBal ? static_cast<int64_t>(blockIdx.x) * p.bal_per_cta : 0;
    const int64_t bal_b = kBal ? min(bal_a + p.bal_per_cta, static_cast<int64_t>(p.bal_units) * p.bal_chunks) : 0;
    const int nchunks = kBal ? static_cast<int>(bal_b > bal_a ? bal_b - bal_a : 0) : static_cast<int>((L + kC - 1) / kC);
    // Where chunk g of this CTA lives: its unit's TMA coordinate zc and state index unit, the
    // unit's first row y0 and gate/o base gbase, the chunk's index c in the unit, and (balanced)
    // whether it starts or ends its segment and how that segment's states are handed.
    struct Loc { int32_t zc; int unit; int64_t y0, gbase; int c; bool first, last; int flags; };
    auto loc = [&](int g) -> Loc {
        if constexpr (kBal) {
            const int* tab = reinterpret_cast<const int*>(sbase + OFF_SEGS);
            const int n = tab[0];
            int g0 = 0;
            for (int i = 0; i < n; ++i) {
                const int4 sg = reinterpret_cast<const int4*>(tab + 4)[i];
                const int len = sg.z - sg.y;
                if (g < g0 + len || i == n - 1)
                    return Loc{sg.x, sg.x, 0, static_cast<int64_t>(sg.x) * p.L, sg.y + (g - g0), g == g0,
                               g == g0 + len - 1, sg.w};
                g0 += len;
            }
            return Loc{ug, ug, 0, 0, g, true, true, 0};   // (no segment: not reached)
        } else {
            return Loc{zc, ug, y0, gbase, g, g == 0, g == nchunks - 1, 0};
        }
    };

    // ---- set-up: barriers, TMEM ----
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        if constexpr (kBal) {
            // the segments of [bal_a, bal_b), in this order: the start of a unit that the next
            // CTA finishes (its state handed on), whole units, then the end of a unit whose start
            // the previous CTA ran first (its state handed over)
            const int64_t N = p.bal_chunks;
            int* tab = reinterpret_cast<int*>(sbase + OFF_SEGS);
            int4* segs = reinterpret_cast<int4*>(tab + 4);
            int n = 0;
            for (int kind = 0; kind < 3; ++kind) {
                for (int64_t u = bal_a / N; u * N < bal_b && n < kMaxSeg; ++u) {
                    const int c0 = static_cast<int>(bal_a > u * N ? bal_a - u * N : 0);
                    const int c1 = static_cast<int>(bal_b - u * N < N ? bal_b - u * N : N);
                    const int k = c0 > 0 ? 2 : (c1 < N ? 0 : 1);
                    if (k != kind) continue;
                    segs[n++] = make_int4(static_cast<int>(u), c0, c1, (c0 > 0 ? kSegIn : 0) | (c1 < N ? kSegOut : 0));
                }
            }
            tab[0] = n;
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_addr(sb, B_FULL + s), 1);
            mbar_init(bar_addr(sb, B_CONV + s), 3);
            mbar_init(bar_addr(sb, B_EMPTY + s), 1);
            mbar_init(bar_addr(sb, B_GATE_FULL + s), 1);
            mbar_init(bar_addr(sb, B_GATE_EMPTY + s), 3);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_addr(sb, B_TP_FULL + s), 1);
            mbar_init(bar_addr(sb, B_TP_EMPTY + s), 1);
            mbar_init(bar_addr(sb, B_DRAIN + s), 1);
        }
        mbar_init(bar_addr(sb, B_G_FULL), 1);
        mbar_init(bar_addr(sb, B_G_EMPTY), 1);
        mbar_init(bar_addr(sb, B_A_FULL), 1);
        mbar_init(bar_addr(sb, B_B_FULL), 1);
        mbar_init(bar_addr(sb, B_S_FULL), 1);
        mbar_init(bar_addr(sb, B_O_READY), 1);
        mbar_init(bar_addr(sb, B_O_DONE), 128);          // every output thread, once it has read TMEM
        mbar_init(bar_addr(sb, B_Z), 1);
        mbar_init(bar_addr(sb, B_SH_READY), 128);        // every chain thread
        mbar_init(bar_addr(sb, B_Y_READY), 128);
        mbar_init(bar_addr(sb, B_U_READY), 128);
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
            if (kF & kFuseGate) prefetch_tmap(&tm_z);
        }
    }
    if (warp >= 4 && warp < 8) {
        // zero both [T; PT] stages once: the blocks above the diagonal are never written
        const int t = threadIdx.x - 128;
        for (uint32_t off = t * 16; off < 2 * TP_STAGE; off += 128 * 16)
            sts(sb + OFF_TP + off, make_uint4(0, 0, 0, 0));
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + OFF_TMEM_SLOT);
    // every TMEM column this CTA addresses lies inside its allocation
    if (threadIdx.x == 0) dbg_ok((tmem & 0xFFFFu) + TM_COLS <= 512u && (tmem >> 16) == 0u, err);

    if (warp == 0) {
        // ================= TMA producer and the chain's MMA issuer =================
        // The whole warp runs this loop in step -- every lane makes the same bounded waits -- and
        // one elected lane issues each batch of copies or MMAs.  Per chunk c it issues MMA_A,
        // MMA_B and MMA_C as soon as their operands are ready, then the TMA loads of chunk
        // c + kStages into the stage MMA_C(c) frees.  (Issued from a branch on the lane index
        // instead, the tcgen05 operands cannot stay in uniform registers and every batch costs
        // several hundred cycles more.)
        {
            uint32_t issuer = 0;
            int loaded = 0;                          // chunks whose K/Q/V loads were issued
            bool producing = true;
            auto produce = [&](int cc) -> bool {
#ifdef LT2_DEBUG
                if (cc == g_debug_skip_chunk) producing = false;
#endif
                if (!producing) return true;
                const int s = cc % kStages;
                if (!mbar_wait(bar_addr(sb, B_EMPTY + s), ((cc / kStages) & 1) ^ 1, abort_flag, err, kTimeoutNs))
                    return false;
                const Loc lc = loc(cc);
                if (elect_one(issuer) && dbg_ok(lc.c * kC < L && lc.zc < p.units_total, err)) {
                    const uint32_t fb = bar_addr(sb, B_FULL + s);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t st = sb + OFF_KQV + s * STAGE_BYTES;
                    const int32_t y = static_cast<int32_t>(lc.y0 + lc.c * kC);
                    tma_load_3d(st, &tm_k, 0, y, lc.zc, fb);
                    tma_load_3d(st + 16384, &tm_k, 64, y, lc.zc, fb);
                    tma_load_3d(st + 8192, &tm_q, 0, y, lc.zc, fb);
                    tma_load_3d(st + 24576, &tm_q, 64, y, lc.zc, fb);
                    tma_load_3d(st + KQ_BYTES, &tm_v, 0, y, lc.zc, fb);
                    tma_load_3d(st + KQ_BYTES + 8192, &tm_v, 64, y, lc.zc, fb);
                }
                loaded = cc + 1;
                return true;
            };
            bool ok = true;
            for (int cc = 0; ok && cc < kStages && cc < nchunks; ++cc) ok = produce(cc);
            bool issued_any = false;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % kStages;
                const uint32_t st = sb + OFF_KQV + s * STAGE_BYTES;
                // --- MMA_A: (KQ S)^T = S^T [K;Q]^T, once the stage is converted, the fp16 state
                // copy written and the output epilogue done with the previous chunk's columns ---
                if (!mbar_wait(bar_addr(sb, B_CONV + s), (c / kStages) & 1, abort_flag, err, kTimeoutNs) ||
                    !mbar_wait(bar_addr(sb, B_SH_READY), c & 1, abort_flag, err, kTimeoutNs) ||
                    (c > 0 && !mbar_wait(bar_addr(sb, B_O_DONE), (c - 1) & 1, abort_flag, err, kTimeoutNs))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one(issuer)) {
                    #pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t boff = (k >> 2) * 16384 + (k & 3) * 32;
                        umma_f16_tmem_a(tmem + TM_AB, tmem + TM_SH + 8 * k, smem_desc_sw128(st + boff, 16, 1024),
                                        ID_TK, k > 0);
                    }
                    umma_commit(bar_addr(sb, B_A_FULL));
                }
                issued_any = true;
                // --- MMA_B: ([T;PT] X)^T = V^T [T;PT]^T + Y^T [T;PT]^T ---
                const int tps = c & 1;
                if (!mbar_wait(bar_addr(sb, B_Y_READY), c & 1, abort_flag, err, kTimeoutNs) ||
                    !mbar_wait(bar_addr(sb, B_TP_FULL + tps), (c >> 1) & 1, abort_flag, err, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one(issuer)) {
                    const uint32_t tp = sb + OFF_TP + tps * TP_STAGE;
                    const uint32_t vt = st + KQ_BYTES;
                    #pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16(tmem + TM_B, smem_desc_sw128(vt + k * 2048, 8192, 1024),
                                 smem_desc_sw128(tp + k * 32, 16, 1024), ID_MK, k > 0);
                    #pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16_tmem_a(tmem + TM_B, tmem + TM_Y + 8 * k, smem_desc_sw128(tp + k * 32, 16, 1024),
                                        ID_TK, 1);
                    umma_commit(bar_addr(sb, B_B_FULL));
                    umma_commit(bar_addr(sb, B_TP_EMPTY + tps));
                }
                // --- MMA_C: S^T += U~^T K ---
                if (!mbar_wait(bar_addr(sb, B_U_READY), c & 1, abort_flag, err, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one(issuer)) {
                    #pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16_tmem_a(tmem + TM_S, tmem + TM_U + 8 * k,
                                        smem_desc_sw128(st + k * 2048, 16384, 1024), ID_TM, 1);
                    umma_commit(bar_addr(sb, B_S_FULL));
                    umma_commit(bar_addr(sb, B_EMPTY + s));
                    mbar_arrive(bar_addr(sb, B_GATE_EMPTY + s));     // the chain is done with chunk c's gates
                }
                if (c + kStages < nchunks && !produce(c + kStages)) ok = false;
            }
            if (issued_any && lane == issuer) {
                // every MMA this thread issued completes before TMEM is released (the chain may
                // have left early on an abort elsewhere)
                umma_commit(bar_addr(sb, B_DRAIN + 0));
                mbar_wait(bar_addr(sb, B_DRAIN + 0), 0, abort_flag, err, kTimeoutNs / 4);
            }
            if (!ok && lane == 0) {
                // the copies already in flight land before the CTA's memory goes away
                for (int cc = loaded - kStages < 0 ? 0 : loaded - kStages; cc < loaded; ++cc)
                    mbar_wait(bar_addr(sb, B_FULL + cc % kStages), (cc / kStages) & 1, abort_flag, err, kTimeoutNs / 4);
            }
        }
        __syncwarp();
    } else if (warp < 4) {
        // ================= gates (warp 1), conversion of K / Q / V (warps 1 / 2 / 3), Gram ===
        uint32_t gram_issuer = 0;
        int gram_issued = 0;
        // warp 1: alpha and beta of the next chunk are loaded one chunk ahead, so the latency of
        // the global loads hides behind this chunk's gates, conversion and Gram issue
        float a_nx[2] = {1.f, 1.f}, b_nx[2] = {0.f, 0.f};
        auto load_gate_inputs = [&](int cn) {
            const Loc ln = loc(cn < nchunks ? cn : 0);
            #pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int64_t tok = static_cast<int64_t>(ln.c) * kC + lane + 32 * i;
                const bool valid = cn < nchunks && tok < L;
                a_nx[i] = valid ? p.alpha[ln.gbase + tok] : 1.f;
                b_nx[i] = valid ? p.beta[ln.gbase + tok] : 0.f;
            }
        };
        if (warp == 1) load_gate_inputs(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const uint32_t ph = (c / kStages) & 1;
            if (warp == 1) {
                if (!mbar_wait(bar_addr(sb, B_GATE_EMPTY + s), ph ^ 1, abort_flag, err, kTimeoutNs)) break;
                Gates* gs = gate(s);
                const float a_cur[2] = {a_nx[0], a_nx[1]}, b_cur[2] = {b_nx[0], b_nx[1]};
                load_gate_inputs(c + 1);
                // alpha = |alpha| * sign: the magnitudes go through log-domain prefix sums, the
                // signs through a parity count of the negatives (alpha = 0 is taken as 1e-30, a
                // reset to within 1e-30 of the state).  Pass 1, one row of 32 tokens at a time:
                // G_r and the sign of the product up to r (kept in gam[r] for pass 2).
                float carry = 0.f;
                uint32_t negs_before = 0;
                bool in_range = true;                   // every |G_r| < 80
                const int64_t tok0 = static_cast<int64_t>(loc(c).c) * kC;   // the chunk's first token in its unit
                #pragma unroll 1
                for (int i = 0; i < 2; ++i) {
                    float a = i ? a_cur[1] : a_cur[0];
                    // (past the sequence end alpha = 1 and beta = 0 already: no logits there)
                    const bool valid = tok0 + lane + 32 * i < L;
                    if ((kF & kFuseLogits) && valid) a = alpha_from_logit_fast(a, p.alpha_scale);
                    float g = __logf(fmaxf(fabsf(a), 1e-30f));
                    #pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float y = __shfl_up_sync(0xffffffffu, g, off);
                        if (lane >= off) g += y;
                    }
                    g += carry;
                    carry = __shfl_sync(0xffffffffu, g, 31);
                    const uint32_t neg = __ballot_sync(0xffffffffu, a < 0.f);
                    const uint32_t upto = 0xffffffffu >> (31 - lane);
                    const int r = lane + 32 * i;
                    gs->G[r] = g;
                    gs->gam[r] = ((negs_before + __popc(neg & upto)) & 1) ? -1.f : 1.f;
                    const float bb = i ? b_cur[1] : b_cur[0];
                    gs->beta[r] = (kF & kFuseLogits) && valid ? sigmoid_fast(bb) : bb;
                    negs_before += __popc(neg);
                    in_range &= fabsf(g) < 80.f;
                }
                // the factored decay e^{G_r} e^{-G_s} needs both factors representable
                const bool safe = __all_sync(0xffffffffu, in_range);
                const float GC = carry;
                const float sgnC = (negs_before & 1) ? -1.f : 1.f;
                __syncwarp();
                // pass 2: the decay factors (the sign of gam[r], kept by a zero, is the sign of
                // the product of the alphas up to token r)
                #pragma unroll 1
                for (int r = lane; r < kC; r += 32) {
                    const float g = gs->G[r], sg = gs->gam[r], bb = gs->beta[r];
                    gs->gam[r] = sg * __expf(g);
                    gs->bein[r] = safe ? sg * bb * __expf(-g) : 0.f;
                    gs->bgc[r] = sgnC * sg * bb * __expf(GC - g);
                }
                if (lane == 0) {
                    gs->gC = sgnC * __expf(GC);
                    gs->safe = safe ? 1 : 0;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_addr(sb, B_GATE_FULL + s));
            }
            if (!mbar_wait(bar_addr(sb, B_FULL + s), ph, abort_flag, err, kTimeoutNs)) break;
            const uint32_t st = sb + OFF_KQV + s * STAGE_BYTES;
            // K panels (warp 1) at +0 and +16 KB, Q panels (warp 2) at +8 and +24 KB, both V panels
            // (warp 3) at +32 KB: one copy of the conversion loop for all three
            if (kF & kFuseNorm) {
                // Q (warp 2) and K (warp 3): every row divided by its L2 norm on the way to fp16;
                // warp 1, which also computes the gates and issues the Gram, takes V instead
                if (warp == 1) {
                    #pragma unroll 1
                    for (int panel = 0; panel < 2; ++panel) convert_tile(st + KQ_BYTES + panel * 8192, 512, lane, lds, sts);
                } else {
                    const uint32_t t = warp == 2 ? st + 8192 : st;
                    convert_rows_l2(t, t + 16384, lane, lds, sts);
                }
            } else {
                #pragma unroll 1
                for (int panel = 0; panel < 2; ++panel) {
                    const uint32_t src = warp == 3 ? st + KQ_BYTES + panel * 8192
                                                   : st + (warp - 1) * 8192 + panel * 16384;
                    if (dbg_ok(src >= sb + OFF_KQV && src + 8192 <= sb + OFF_KQV + kStages * STAGE_BYTES, err))
                        convert_tile(src, 512, lane, lds, sts);
                }
            }
            if constexpr (kVar) {
                const int64_t nrow = L - static_cast<int64_t>(c) * kC;
                if (nrow < kC) {
                    // rows past a packed sequence's end hold the next sequence's tokens: zeroed,
                    // as the tensor map's fill leaves them for fixed lengths (this warp's tile:
                    // 0 K, 1 Q, 2 V; two 64-row panels of 64 vectors of 16 bytes per 8 rows)
                    __syncwarp();
                    const int which = (kF & kFuseNorm) ? (warp == 1 ? 2 : warp == 2 ? 1 : 0) : warp - 1;
                    const uint32_t p0 = which == 2 ? st + KQ_BYTES : st + which * 8192;
                    const uint32_t pstride = which == 2 ? 8192 : 16384;
                    for (int i = lane; i < 1024; i += 32) {
                        if (((i & 511) >> 3) >= nrow)
                            sts(p0 + (i >> 9) * pstride + (i & 511) * 16, make_uint4(0u, 0u, 0u, 0u));
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_addr(sb, B_CONV + s));
            if (warp == 1) {
                // Gram products of this chunk, once all of its tiles are in fp16 and the prep
                // group has read the previous chunk's
                const bool gram_ok =
                    mbar_wait(bar_addr(sb, B_CONV + s), ph, abort_flag, err, kTimeoutNs) &&
                    (c == 0 || mbar_wait(bar_addr(sb, B_G_EMPTY), (c - 1) & 1, abort_flag, err, kTimeoutNs));
                if (__all_sync(0xffffffffu, gram_ok)) {
                    tc_fence_after();
                    if (elect_one(gram_issuer)) issue_gram(sb, tmem, s);
                    __syncwarp();
                    gram_issued = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        }
        if (warp == 1 && lane == gram_issuer && gram_issued && *abort_flag) {
            // wait for the Gram MMAs this thread issued before TMEM is released
            umma_commit(bar_addr(sb, B_DRAIN + 1));
            mbar_wait(bar_addr(sb, B_DRAIN + 1), 0, abort_flag, err, kTimeoutNs / 4);
        }
    } else if (warp < 8) {
        // ================= prep: Gram epilogue, solve, P T =================
        const int t = threadIdx.x - 128;            // 0..127 = TMEM lane
        const int q = warp - 4;                     // warp within the group
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
        Group grp{NB_PREP, 128, t == 0, abort_flag, err};
        const uint32_t as = sb + OFF_AS, ps = sb + OFF_PS;
        float* adiag = reinterpret_cast<float*>(sbase + OFF_ADIAG);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const int tps = c & 1;
            // Gram of chunk c in TMEM, its gates, and a free [T; PT] stage
            if (!grp.wait(bar_addr(sb, B_G_FULL), c & 1, bar_addr(sb, B_GATE_FULL + s), (c / kStages) & 1,
                          bar_addr(sb, B_TP_EMPTY + tps), ((c >> 1) & 1) ^ 1))
                break;
            tc_fence_after();
            const Gates* gs = gate(s);
            const int r = t & 63;
            const bool is_a = t < 64;               // rows of K K^T (A) or Q K^T (P)
            const float gr = gs->gam[r];
            const bool safe = gs->safe != 0;
            const uint32_t dst = is_a ? as : ps;
            dbg_ok(dst >= sb + OFF_AS && dst + 8192 <= sb + OFF_ADIAG && r < kC, err);
            if (safe) {
                // A is kept negated (the solve only accumulates).  Entries on or above the
                // diagonal (s >= r in A, s > r in P) are never read, apart from the diagonal P
                // block, which the solve masks in registers, so no mask is applied here.
                const float sg = is_a ? -gr : gr;
                #pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float v[32];
                    tmem_load32(tmem + TM_G + lane_addr + 32 * h, v);
                    const float* be = gs->bein + 32 * h;
                    #pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const float4 b4 = *reinterpret_cast<const float4*>(be + j4);
                        v[j4 + 0] *= sg * b4.x;
                        v[j4 + 1] *= sg * b4.y;
                        v[j4 + 2] *= sg * b4.z;
                        v[j4 + 3] *= sg * b4.w;
                    }
                    if (is_a && h == q) {
                        // this warp's rows r = 32q..32q+31 have their diagonal blocks in columns
                        // 32h..32h+31: keep the fp32 copy for the diagonal inverses
                        const bool upper = (r & 16) != 0;
                        float* ad = adiag + (r >> 4) * ADIAG_BLOCK + (r & 15) * kAdiagRow;
                        #pragma unroll
                        for (int jj = 0; jj < 16; ++jj) ad[jj] = upper ? v[16 + jj] : v[jj];
                    }
                    #pragma unroll
                    for (int ch = 0; ch < 4; ++ch) sts(sw128(dst, r, 4 * h + ch), pack8_half(v + 8 * ch));
                }
            } else {
                gram_epilogue_unfactored(tmem + TM_G + lane_addr, gs, r, is_a, sbase + (dst - sb), dst,
                                         adiag + (r >> 4) * ADIAG_BLOCK + (r & 15) * kAdiagRow);
            }
            tc_fence_before();
            grp.sync();
            if (t == 0) {
                mbar_arrive(bar_addr(sb, B_G_EMPTY));
                mbar_arrive(bar_addr(sb, B_GATE_EMPTY + s));
            }
            const uint32_t tp = sb + OFF_TP + tps * TP_STAGE;
            if (is_a) {
                diag_block_inverse_row(tp, r, adiag + (r >> 4) * ADIAG_BLOCK);
            }
            grp.sync();
            // warp q: the T rows of block q and the PT rows of block 3 - q
            solve_row_block(tp, as, 0, ps, 0, q, 4, lane);
            solve_row_block(tp, as, 0, ps, 0, 7 - q, 4, lane);
            fence_proxy_async_smem();
            grp.sync();
            if (t == 0) mbar_arrive(bar_addr(sb, B_TP_FULL + tps));
        }
    } else if (warp < 12) {
        // ================= the S-dependent chain (lane j = d_v column j of S) =================
        const int j = threadIdx.x - 256;            // 0..127 = TMEM lane = d_v index
        const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const bool leader = j == 0;
        Group grp{NB_CHAIN, 128, leader, abort_flag, err};
        bool ok = nchunks > 0;
        if constexpr (kVar) {
            // an empty packed sequence: the state passes through unchanged
            if (nchunks == 0 && seq_ok && p.S_out) {
                const int64_t base = static_cast<int64_t>(ug) * kD * kD + j;
                for (int i = 0; i < kD; ++i) p.S_out[base + i * kD] = p.S0 ? p.S0[base + i * kD] : 0.f;
            }
        }
        // a segment's initial state: S0^T, or (balanced, the end of a unit begun by the previous
        // CTA) the state it handed over in S_out; fp32 in TMEM, pre-scaled by the first chunk's
        // decay, and an fp16 copy.  Chunk g's gates are in (its stage's GATE_FULL was waited).
        auto segment_start = [&](int g) -> bool {
            const Loc ls = loc(g);
            const float* src = p.S0 ? p.S0 + static_cast<int64_t>(ls.unit) * kD * kD + j : nullptr;
            if constexpr (kBal) {
                if (ls.flags & kSegIn) {
                    const unsigned int* f = p.bal_flags + ls.unit;
                    const int got = leader ? (wait_handoff(f, abort_flag, err) ? 1 : 0) : 1;
                    unsigned int all;
                    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                                 "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                                 : "=r"(all) : "r"(got), "r"(NB_CHAIN), "r"(128) : "memory");
                    if (!all) return false;
                    unsigned int v;                      // (every thread acquires the handoff)
                    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
                    (void)v;
                    src = p.S_out + static_cast<int64_t>(ls.unit) * kD * kD + j;
                }
            }
            load_initial_state(tmem + TM_S + lane_addr, tmem + TM_SH + lane_addr, src, gate(g % kStages)->gC);
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_SH_READY));           // MMA_A of chunk g may read it
            return true;
        };
        if (ok) ok = grp.wait(bar_addr(sb, B_GATE_FULL + 0), 0);
        if (ok) ok = segment_start(0);
        for (int c = 0; ok && c < nchunks; ++c) {
            const int s = c % kStages;
            const Gates* gs = gate(s);
            ok = grp.wait(bar_addr(sb, B_A_FULL), c & 1);
            if (!ok) break;
            tc_fence_after();
            // --- Y^T = -g (K S)^T, fp16, into TMEM as the second A operand of MMA_B ---
            {
                float ks[64];
                tmem_load_2x32(tmem + TM_AB + lane_addr, tmem + TM_AB + lane_addr + 32, ks);
                uint32_t hpk[32];
                #pragma unroll
                for (int e4 = 0; e4 < 64; e4 += 4) {
                    const float4 g4 = *reinterpret_cast<const float4*>(&gs->gam[e4]);
                    hpk[e4 / 2] = pack_half2(-g4.x * ks[e4], -g4.y * ks[e4 + 1]);
                    hpk[e4 / 2 + 1] = pack_half2(-g4.z * ks[e4 + 2], -g4.w * ks[e4 + 3]);
                }
                tmem_st16(tmem + TM_Y + lane_addr, *reinterpret_cast<uint32_t(*)[16]>(hpk));
                tmem_st16(tmem + TM_Y + lane_addr + 16, *reinterpret_cast<uint32_t(*)[16]>(hpk + 16));
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_Y_READY));
            ok = grp.wait(bar_addr(sb, B_B_FULL), c & 1);
            if (!ok) break;
            tc_fence_after();
            if (leader) mbar_arrive(bar_addr(sb, B_O_READY));
            // --- U~^T = diag(beta e^{G_63 - G}) U^T, fp16, into TMEM for MMA_C ---
            {
                float u[64];
                tmem_load_2x32(tmem + TM_B + lane_addr, tmem + TM_B + lane_addr + 32, u);
                uint32_t hpk[32];
                #pragma unroll
                for (int e4 = 0; e4 < 64; e4 += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(&gs->bgc[e4]);
                    hpk[e4 / 2] = pack_half2(b4.x * u[e4], b4.y * u[e4 + 1]);
                    hpk[e4 / 2 + 1] = pack_half2(b4.z * u[e4 + 2], b4.w * u[e4 + 3]);
                }
                tmem_st16(tmem + TM_U + lane_addr, *reinterpret_cast<uint32_t(*)[16]>(hpk));
                tmem_st16(tmem + TM_U + lane_addr + 16, *reinterpret_cast<uint32_t(*)[16]>(hpk + 16));
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_U_READY));
            // --- the new state ---
            const bool last = c + 1 == nchunks;
            const int s1 = (c + 1) % kStages;
            ok = last ? grp.wait(bar_addr(sb, B_S_FULL), c & 1)
                      : grp.wait(bar_addr(sb, B_S_FULL), c & 1, bar_addr(sb, B_GATE_FULL + s1),
                                 ((c + 1) / kStages) & 1);
            if (!ok) break;
            tc_fence_after();
            const Loc lc = loc(c);
            if (kBal ? lc.last : last) {
                // the segment's last state: the final state of its unit, or (balanced) the state
                // handed on to the CTA that finishes the unit
                if (p.S_out) {
                    const bool sfin = store_final_state(tmem + TM_S + lane_addr,
                                                        p.S_out + static_cast<int64_t>(lc.unit) * kD * kD + j);
                    if (__any_sync(0xffffffffu, !sfin) && lane == 0) atomicOr(err, kDevRange);
                }
                if constexpr (kBal) {
                    if (lc.flags & kSegOut) {
                        __threadfence();                 // this thread's column, then the flag
                        grp.sync();
                        if (leader)
                            asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p.bal_flags + lc.unit), "r"(1u)
                                         : "memory");
                    }
                    if (!last) {
                        ok = segment_start(c + 1);       // the next segment, from its first chunk
                        if (!ok) break;
                    }
                }
            } else {
                const float gn = gate(s1)->gC;
                #pragma unroll 1
                for (int piece = 0; piece < 4; piece += 2) {
                    float v[64];
                    tmem_load_2x32(tmem + TM_S + lane_addr + 32 * piece, tmem + TM_S + lane_addr + 32 * piece + 32, v);
                    uint32_t hpk[32];
                    #pragma unroll
                    for (int e = 0; e < 32; ++e) hpk[e] = pack_half2(v[2 * e], v[2 * e + 1]);
                    tmem_st16(tmem + TM_SH + lane_addr + 16 * piece, *reinterpret_cast<uint32_t(*)[16]>(hpk));
                    tmem_st16(tmem + TM_SH + lane_addr + 16 * piece + 16, *reinterpret_cast<uint32_t(*)[16]>(hpk + 16));
                    #pragma unroll
                    for (int d = 0; d < 64; ++d) v[d] *= gn;
                    tmem_st32(tmem + TM_S + lane_addr + 32 * piece, *reinterpret_cast<float(*)[32]>(v));
                    tmem_st32(tmem + TM_S + lane_addr + 32 * piece + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_addr(sb, B_SH_READY));      // MMA_A of the next chunk may read it
            }
        }
    } else {
        // ================= output epilogue: o = g (Q S) + P T X =================
        const int j = threadIdx.x - 384;            // TMEM lane = d_v index
        const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        Group grp{NB_OUT, 128, j == 0, abort_flag, err};
        bool fin = true;                             // every output so far is finite
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const Loc lo = loc(c);
            const int64_t t0 = static_cast<int64_t>(lo.c) * kC;      // the chunk's first token in its unit
            if (j == 0) bulk_wait_read_all();        // the staging tile is free again
            constexpr bool gated = (kF & kFuseGate) != 0;
            if (gated && j == 0) {
                // the output gate logits of this chunk, into the staging tile the outputs are
                // written to (the same two 64 x 64 boxes; rows past L read as 0)
                const uint32_t zb = bar_addr(sb, B_Z);
                mbar_arrive_expect_tx(zb, 16384);
                tma_load_3d(sb + OFF_OST, &tm_z, 0, static_cast<int32_t>(lo.y0 + t0), lo.zc, zb);
                tma_load_3d(sb + OFF_OST + 8192, &tm_z, 64, static_cast<int32_t>(lo.y0 + t0), lo.zc, zb);
            }
            if constexpr (gated) {
                // sigmoid(z) of this thread's column, in place as fp16, while the chain is still
                // working on the chunk: the output's own wait below is then free of MUFU work
                if (!grp.wait(bar_addr(sb, B_Z), c & 1)) break;
                uint8_t* zcol = sbase + OFF_OST + (j >> 6) * 8192 + (j & 63) * 2;
                #pragma unroll 8
                for (int r = 0; r < kC; ++r) {
                    const float zr = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(zcol + r * 128));
                    *reinterpret_cast<__half*>(zcol + r * 128) = __float2half_rn(sigmoid_fast(zr));
                }
            }
            if (!grp.wait(bar_addr(sb, B_O_READY), c & 1)) break;
            tc_fence_after();
            const Gates* gs = gate(s);
            if (!p.out_bf16) {
                // fp32 output: plain stores, done before the TMEM columns are released
                const int n = static_cast<int>(L - t0 < kC ? L - t0 : kC);
                fin &= store_o_f32(tmem + TM_AB + lane_addr + 64, tmem + TM_B + lane_addr + 64, gs->gam,
                                   static_cast<float*>(p.o) + (lo.gbase + t0) * kD + j, n,
                                   gated ? sbase + OFF_OST + (j >> 6) * 8192 + (j & 63) * 2 : nullptr);
                tc_fence_before();
                mbar_arrive(bar_addr(sb, B_O_DONE));
                grp.sync();
                if (j == 0) mbar_arrive(bar_addr(sb, B_GATE_EMPTY + s));
                continue;
            }
            // o[r][j] = g_r (Q S)^T[j][r] + (P T X)^T[j][r]: all 64 tokens of column j read from
            // TMEM and rounded into registers first, so MMA_A of the next chunk may overwrite the
            // columns while this thread transposes them through the staging tile (a warp writes
            // 64 contiguous bytes per token), which the TMA unit writes out as two 64 x 64 boxes;
            // rows past L are clipped
            uint8_t* ost = sbase + OFF_OST + (j >> 6) * 8192 + (j & 63) * 2;
            uint32_t opk[32];                        // bf16 pairs: tokens 2e, 2e + 1
            #pragma unroll
            for (int q = 0; q < 4; ++q) {
                float qp[32];                        // (Q S)^T, then (P T X)^T, for 16 tokens
                tmem_load_2x16(tmem + TM_AB + lane_addr + 64 + 16 * q, tmem + TM_B + lane_addr + 64 + 16 * q, qp);
                #pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const int r = 16 * q + e;
                    const float2 g2 = *reinterpret_cast<const float2*>(&gs->gam[r]);
                    float o0 = g2.x * qp[e] + qp[16 + e];
                    float o1 = g2.y * qp[e + 1] + qp[16 + e + 1];
                    if (gated) {                     // sigmoid(z), fp16, from the staging tile
                        o0 *= __half2float(*reinterpret_cast<const __half*>(ost + r * 128));
                        o1 *= __half2float(*reinterpret_cast<const __half*>(ost + (r + 1) * 128));
                    }
                    if constexpr (kVar) {
                        // rows past the sequence end hold the next sequence's tokens: not outputs
                        fin &= (r >= L - t0 || is_finite(o0)) & (r + 1 >= L - t0 || is_finite(o1));
                    } else {
                        fin &= is_finite(o0) & is_finite(o1);
                    }
                    opk[r / 2] = pack_bf16x2(o0, o1);
                }
            }
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_O_DONE));     // this thread is done with the TMEM columns
            #pragma unroll
            for (int e = 0; e < 32; ++e) {
                *reinterpret_cast<uint16_t*>(ost + (2 * e) * 128) = static_cast<uint16_t>(opk[e] & 0xFFFFu);
                *reinterpret_cast<uint16_t*>(ost + (2 * e + 1) * 128) = static_cast<uint16_t>(opk[e] >> 16);
            }
            fence_proxy_async_smem();
            grp.sync();
            if (kVar && t0 + kC > L) {
                // a packed sequence's last, partial chunk: the rows past its end belong to the next
                // sequence, so the n rows are copied out by plain 16-byte stores (both 64-column
                // halves of a row: 16 pieces), not by the two box stores
                const int n = static_cast<int>(L - t0);
                __nv_bfloat16* orow0 = static_cast<__nv_bfloat16*>(p.o) + (lo.gbase + t0) * kD;
                for (int i = j; i < n * 16; i += 128) {
                    const int r = i >> 4, part = i & 15;
                    const uint4 w = *reinterpret_cast<const uint4*>(sbase + OFF_OST + (part >> 3) * 8192 + r * 128 +
                                                                    (part & 7) * 16);
                    *reinterpret_cast<uint4*>(orow0 + static_cast<int64_t>(r) * kD + (part >> 3) * 64 + (part & 7) * 8) = w;
                }
                if (j == 0) mbar_arrive(bar_addr(sb, B_GATE_EMPTY + s));
            } else if (j == 0) {
                mbar_arrive(bar_addr(sb, B_GATE_EMPTY + s));
                if (dbg_ok(t0 < L && lo.zc < p.units_total, err)) {
                    tma_store_3d(&tm_o, sb + OFF_OST, 0, static_cast<int32_t>(lo.y0 + t0), lo.zc);
                    tma_store_3d(&tm_o, sb + OFF_OST + 8192, 64, static_cast<int32_t>(lo.y0 + t0), lo.zc);
                }
                bulk_commit_group();
            }
        }
        if (j == 0) bulk_wait_all();     // every output tile written before the CTA exits
        // rows past L of the last chunk are finite too (zero inputs), so a flag here means a
        // real output went out of range
        if (__any_sync(0xffffffffu, !fin) && lane == 0) atomicOr(err, kDevRange);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---- host side ----------------------------------------------------------------------------

}  // namespace tc

bool prefill_tc_supports(int dtype_bf16, int dk, int dv, int per_key)
{
    if (per_key) return prefill_kda_tc_supports(dtype_bf16, dk, dv);
    return dtype_bf16 && dk == tc::kD && dv == tc::kD;
}

size_t prefill_tc_flag_bytes(int64_t units)
{
    return static_cast<size_t>((units * 4 + 255) / 256 * 256);
}

cudaError_t launch_prefill_tc_all(const TcCall& call, cudaStream_t stream)
{
    using namespace tc;
    if (call.units_per_loop == 0 || call.T == 0) return cudaSuccess;
    const bool var = call.cu_seqlens != nullptr;
    // TMA unit axis and row extent: [T*B*H][L] for fixed lengths, [T*H][Ntot] for packed sequences
    const int64_t units = call.T * call.units_per_loop;
    const int64_t map_units = var ? call.T * call.H : units;
    CUtensorMap mq, mk, mv, mo, mz;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_bf16_map_3d(&mq, call.q, map_units, call.L, kC, sw) ||
        !make_bf16_map_3d(&mk, call.k, map_units, call.L, kC, sw) ||
        !make_bf16_map_3d(&mv, call.v, map_units, call.L, kC, sw))
        return cudaErrorInvalidValue;
    // o (bf16 output only): plain row-major tile, written by the TMA store from shared memory;
    // the output gate logits z (fused) are read into the same tile the same way
    if (call.out_bf16 && !make_bf16_map_3d(&mo, call.o, map_units, call.L, kC, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (call.z && !make_bf16_map_3d(&mz, call.z, map_units, call.L, kC, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int fb = fuse_bits(call);
    using K = decltype(&gdr_prefill_tc_kernel<0, 0>);
    static const K kernels[3][8] = {
        {gdr_prefill_tc_kernel<0, 0>, gdr_prefill_tc_kernel<1, 0>, gdr_prefill_tc_kernel<2, 0>,
         gdr_prefill_tc_kernel<3, 0>, gdr_prefill_tc_kernel<4, 0>, gdr_prefill_tc_kernel<5, 0>,
         gdr_prefill_tc_kernel<6, 0>, gdr_prefill_tc_kernel<7, 0>},
        {gdr_prefill_tc_kernel<0, 1>, gdr_prefill_tc_kernel<1, 1>, gdr_prefill_tc_kernel<2, 1>,
         gdr_prefill_tc_kernel<3, 1>, gdr_prefill_tc_kernel<4, 1>, gdr_prefill_tc_kernel<5, 1>,
         gdr_prefill_tc_kernel<6, 1>, gdr_prefill_tc_kernel<7, 1>},
        {gdr_prefill_tc_kernel<0, 2>, gdr_prefill_tc_kernel<1, 2>, gdr_prefill_tc_kernel<2, 2>,
         gdr_prefill_tc_kernel<3, 2>, gdr_prefill_tc_kernel<4, 2>, gdr_prefill_tc_kernel<5, 2>,
         gdr_prefill_tc_kernel<6, 2>, gdr_prefill_tc_kernel<7, 2>}};
    // Balanced schedule: with more units than SMs, one CTA per SM takes an equal share of all
    // units' chunks (so no SM idles through a partial second wave); it needs S_out (a unit split
    // between two CTAs hands its state over there) and the caller's workspace (one flag a unit).
    int sms = 0;
    if (!var && call.S_out && call.workspace && call.workspace_bytes >= prefill_tc_flag_bytes(units)) {
        int dev = 0;
        cudaError_t e0 = cudaGetDevice(&dev);
        if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e0 != cudaSuccess) return e0;
    }
    const int64_t nch = (call.L + kC - 1) / kC;
    const int64_t per_cta = sms > 0 ? (units * nch + sms - 1) / sms : 0;
    // (a share of per_cta chunks touches at most per_cta / nch + 2 units: kMaxSeg bounds it)
    if (sms > 0 && units > sms && units <= INT32_MAX / nch && per_cta <= (kMaxSeg - 2) * nch) {
        const K kernel = kernels[2][fb];
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(SMEM_BYTES));
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(call.workspace, 0, prefill_tc_flag_bytes(units), stream);
        if (e != cudaSuccess) return e;
        NvtxRange range("lt2 prefill, all loops (tensor core, scalar gating, balanced)");
        Params p;
        p.alpha = call.alpha;
        p.beta = call.beta;
        p.S0 = call.S0;
        p.o = call.o;
        p.S_out = call.S_out;
        p.L = call.L;
        p.unit0 = 0;
        p.units_total = static_cast<int>(map_units);
        p.out_bf16 = call.out_bf16;
        p.err = call.err;
        p.qk_norm = call.qk_norm;
        p.gate_logits = call.gate_logits;
        p.alpha_scale = call.alpha_scale;
        p.cu = nullptr;
        p.Ntot = call.L;
        p.H = 0;
        p.loop = 0;
        p.bal_units = static_cast<int>(units);
        p.bal_chunks = static_cast<int>(nch);
        p.bal_per_cta = static_cast<int>(per_cta);     // >= nch, since units > sms
        p.bal_flags = static_cast<unsigned int*>(call.workspace);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sms), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = stream;
        return cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, call.out_bf16 ? mo : mv, call.z ? mz : mv, p, 0);
    }
    const K kernel = kernels[var ? 1 : 0][fb];
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess) return e;
    for (int64_t tau = 0; tau < call.T; ++tau) {
        NvtxRange loop_range("lt2 prefill loop (tensor core, scalar gating)");
        Params p;
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
        p.cu = call.cu_seqlens;
        p.Ntot = call.L;
        p.H = static_cast<int>(call.H);
        p.loop = static_cast<int>(tau);
        p.bal_units = 0;
        p.bal_chunks = 0;
        p.bal_per_cta = 0;
        p.bal_flags = nullptr;
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
        const int use_pdl = tau > 0 ? 1 : 0;
        // unused maps are passed as copies of a valid one (never dereferenced)
        e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, call.out_bf16 ? mo : mv, call.z ? mz : mv, p, use_pdl);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lt2

#ifdef LT2_DEBUG
namespace lt2 {
cudaError_t debug_set_skip_chunk_scalar(int chunk)
{
    return cudaMemcpyToSymbol(tc::g_debug_skip_chunk, &chunk, sizeof(chunk));
}
}  // namespace lt2
#endif
