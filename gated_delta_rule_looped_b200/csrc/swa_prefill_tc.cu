// swa_prefill_tc.cu -- the looped sliding-window attention mixer on Blackwell tensor cores
// (tcgen05 MMA with TMEM accumulators, tiles staged by TMA), bf16 q/k/v, d = 128.
//
// "LT2 transformer looped a tempo lineare", section "Sostituire il motore": the second family of
// sub-quadratic mixers is sparse attention, every token looking at a window of the w most recent
// positions; section "Il giro trasforma il calcolo in contesto": repeated T times, the window
// reaches back O(T w) tokens.  For every (loop, batch, head) unit and token t:
//
//     o_t = sum_{s = t-w+1 .. t, s >= 0} softmax_s(scale q_t . k_s) v_s
//
// CTA = one unit x one block of 128 queries; the keys of its window are visited in blocks of 64.
// Per key block j (one pipeline step):
//     S  = Q K_j^T          tcgen05, M = 128 queries, N = 64 keys, K = 128; A = Q, B = K_j (smem)
//     P  = exp2(x - m)      softmax warps: x = log2(e) scale S, masked to the window; m the
//                           running row maximum, raised only when a block's maximum exceeds it
//                           by more than 8 (P <= 2^8), and then O and the row sum rescaled
//     O += P V_j            tcgen05, M = 128, N = 128, K = 64; A = P (TMEM, bf16), B = V_j (smem)
// and at the end o = O / l.  Operands are bf16 (as the inputs; P rounded to bf16), accumulation
// fp32 in tensor memory.
//
// Warps: 0 TMA producer (Q once, then K and V blocks through two-stage rings of their own: a K
// stage is free again as soon as Q K^T is done with it), 1 MMA issuer, 2-5 softmax (one query
// row per thread; the warp's TMEM lane quadrant is warp % 4) and output.  The producer and the
// issuer warps run their loops in step -- every lane makes the same bounded waits, so no lane
// waits alone and no reconvergence follows -- and one elected lane issues each batch of copies
// or MMAs (from a warp-uniform branch, so the tcgen05 operands stay in uniform registers).
// About 97 KB of shared memory and 256 TMEM columns per CTA, so two CTAs share an SM and one's
// softmax runs under the other's MMAs.  Every mbarrier wait is bounded as in the prefills of the
// linear mixer; on a timeout the CTA records it, drains its copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "gdr_common.cuh"
#include "gdr_launch.h"
#include "gdr_nvtx.h"
#include "gdr_tc_common.cuh"
#include "gdr_tma_host.h"
#include "sm100_primitives.cuh"

namespace lt2 {
namespace swa {

using namespace sm100;
using namespace tcc;

constexpr int kBM = 128;               // queries per CTA
constexpr int kBN = 64;                // keys per block
constexpr int kThreads = 192;          // 6 warps
constexpr uint64_t kTimeoutNs = kWaitTimeoutNs;

// Shared memory (offsets from a 1024-byte aligned base), 128-byte swizzled panels of 64 bf16
// columns: Q [2 panels][128 rows] (reused as the o staging tile at the end), and two-stage rings
// of K [2 panels][64 rows] and of V [2 panels][64 rows].
constexpr uint32_t Q_PANEL = kBM * 128;                 // 16 KB
constexpr uint32_t KV_PANEL = kBN * 128;                // 8 KB
constexpr uint32_t KV_STAGE = 2 * KV_PANEL;             // one K or V block
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + 2 * Q_PANEL;
constexpr uint32_t OFF_V = OFF_K + 2 * KV_STAGE;
constexpr uint32_t OFF_BAR = OFF_V + 2 * KV_STAGE;
// P_FULL and PV_DONE come in pairs (even and odd blocks): the softmax warps may run a block ahead of
// the MMA issuer, and with one barrier of each the waiter could then see two phases complete at
// once and misread the parity.  Each of a pair completes once every two blocks, at most one phase
// ahead of its waiter (Q K_{j+2}^T, which the softmax of block j+2 needs, is issued after
// O += P_j V_j).
enum Bar : uint32_t {
    B_Q = 0,          // Q landed
    B_K_FULL = 1,     // [2] K of a stage landed
    B_K_EMPTY = 3,    // [2] Q K^T is done with a K stage
    B_V_FULL = 5,     // [2] V of a stage landed
    B_V_EMPTY = 7,    // [2] O += P V is done with a V stage
    B_S_FULL = 9,     // S = Q K^T done
    B_S_FREE = 10,    // the softmax warps have read S
    B_P_FULL = 11,    // [2] P_j written (and O rescaled when needed), for even and odd j
    B_PV_DONE = 13,   // [2] O += P_j V_j done, for even and odd j
    B_DRAIN = 15,     // drain on abort (MMA issuer)
    B_COUNT = 16
};
constexpr uint32_t OFF_TMEM_SLOT = OFF_BAR + B_COUNT * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEM_SLOT + 16;
constexpr uint32_t SMEM_USED = OFF_ABORT + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

// TMEM columns (lane = query row)
constexpr uint32_t TM_S = 0;           // S, fp32 (64 columns)
constexpr uint32_t TM_P = 64;          // P_j, bf16 pairs, two buffers of 32 columns (j even, odd):
                                       // the A operand of O += P_j V_j
constexpr uint32_t TM_O = 128;         // O, fp32 (128 columns)
constexpr uint32_t TM_COLS = 256;

constexpr int NB_SOFT = 1;             // named barrier of the softmax warps
constexpr int kSoftThreads = 128;


// Instruction descriptor, kind::f16 with bf16 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn)
{
    return idesc_f16_f32(M, N, a_mn, b_mn) | (1u << 7) | (1u << 10);
}
constexpr uint32_t ID_QK = idesc_bf16_f32(kBM, kBN, 0, 0);      // A, B K-major
constexpr uint32_t ID_PV = idesc_bf16_f32(kBM, 128, 0, 1);      // A in TMEM, B MN-major

struct Params {
    void* o;               // [units][L][128], bf16 or fp32
    int64_t L;
    int window;
    float xscale;          // scale * log2(e)
    int nqb;               // query blocks per unit
    int units;             // T*B*H
    int out_bf16;
    unsigned int* err;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, uint32_t i) { return base + OFF_BAR + 8u * i; }

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Softmax thread (query row r): O / l to the staging tile (bf16, 128-byte swizzled like Q, for
// the TMA store) or, with an fp32 output, straight to global memory (row `o32`, null past L).
__device__ __noinline__ void write_output(uint32_t tm_o, float inv_l, uint32_t stage, int r, float* o32,
                                          uint8_t* sbase, uint32_t sb)
{
    #pragma unroll 1
    for (int piece = 0; piece < 4; ++piece) {          // 32 columns of d
        float v[32];
        tmem_load32(tm_o + 32 * piece, v);
        #pragma unroll
        for (int d = 0; d < 32; ++d) v[d] *= inv_l;
        if (o32) {
            #pragma unroll
            for (int d4 = 0; d4 < 32; d4 += 4)
                *reinterpret_cast<float4*>(o32 + 32 * piece + d4) = make_float4(v[d4], v[d4 + 1], v[d4 + 2], v[d4 + 3]);
        } else if (stage) {
            #pragma unroll
            for (int c = 0; c < 4; ++c) {               // four 16-byte chunks
                const int chunk = piece * 4 + c;
                const uint32_t a = sw128(stage + (chunk >> 3) * Q_PANEL, static_cast<uint32_t>(r), chunk & 7);
                *reinterpret_cast<uint4*>(sbase + (a - sb)) =
                    make_uint4(pack_bf16x2(v[8 * c + 0], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                               pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
            }
        }
    }
}

// Softmax thread: row r of O times `corr` (the row's running maximum went up).
__device__ __noinline__ void rescale_o(uint32_t tm_o, float corr)
{
    #pragma unroll 1
    for (int piece = 0; piece < 4; ++piece) {
        float v[32];
        tmem_load32(tm_o + 32 * piece, v);
        #pragma unroll
        for (int d = 0; d < 32; ++d) v[d] *= corr;
        tmem_st32(tm_o + 32 * piece, v);
    }
    tmem_wait_st();
}

__global__ void __launch_bounds__(kThreads, 2)
swa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sbase = smem_raw + (sb - raw);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + OFF_ABORT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x / p.nqb;
    const int qb = blockIdx.x - unit * p.nqb;
    const int64_t L = p.L;
    const int i0 = qb * kBM;                                             // first query of the CTA
    const int64_t kv_lo = i0 - p.window + 1 > 0 ? i0 - p.window + 1 : 0;  // first key any row sees
    const int64_t kv_hi = i0 + kBM - 1 < L - 1 ? i0 + kBM - 1 : L - 1;   // last key any row sees
    const int j_first = static_cast<int>(kv_lo / kBN);
    const int nblk = static_cast<int>(kv_hi / kBN) - j_first + 1;
    unsigned int* err = p.err;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (uint32_t b = 0; b < B_COUNT; ++b)
            mbar_init(bar_addr(sb, b), b == B_S_FREE || b == B_P_FULL || b == B_P_FULL + 1 ? kSoftThreads : 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(sb + OFF_TMEM_SLOT, TM_COLS);
        tmem_relinquish();
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            if (p.out_bf16) prefetch_tmap(&tm_o);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + OFF_TMEM_SLOT);
    if (threadIdx.x == 0) dbg_ok((tmem & 0xFFFFu) + TM_COLS <= 512u && (tmem >> 16) == 0u, err);

    if (warp == 0) {
        // ================= TMA producer: Q, then K and V of the window =================
        // K_j is released by Q K_j^T and V_j only by O += P_j V_j, one block later, so each ring
        // advances on its own: step j issues K_j (once Q K_{j-2}^T is done), then V_{j-1} (once
        // O += P_{j-3} V_{j-3} is done) -- the order in which the MMAs free their stages.
        {
            uint32_t leader = 0;
            const uint32_t qbar = bar_addr(sb, B_Q);
            if (elect_one(leader)) {
                mbar_arrive_expect_tx(qbar, 2 * Q_PANEL);
                tma_load_3d(sb + OFF_Q, &tm_q, 0, i0, unit, qbar);
                tma_load_3d(sb + OFF_Q + Q_PANEL, &tm_q, 64, i0, unit, qbar);
            }
            int k_issued = 0, v_issued = 0;
            auto load = [&](bool is_v, int j) -> bool {
                const int s = j & 1;
                const uint32_t empty = bar_addr(sb, (is_v ? B_V_EMPTY : B_K_EMPTY) + s);
                if (!mbar_wait(empty, ((j >> 1) & 1) ^ 1, abort_flag, err, kTimeoutNs)) return false;
                const int32_t y = (j_first + j) * kBN;
                if (elect_one(leader) && dbg_ok(y < L && unit < p.units, err)) {
                    const uint32_t fb = bar_addr(sb, (is_v ? B_V_FULL : B_K_FULL) + s);
                    const uint32_t st = sb + (is_v ? OFF_V : OFF_K) + s * KV_STAGE;
                    mbar_arrive_expect_tx(fb, KV_STAGE);
                    tma_load_3d(st, is_v ? &tm_v : &tm_k, 0, y, unit, fb);
                    tma_load_3d(st + KV_PANEL, is_v ? &tm_v : &tm_k, 64, y, unit, fb);
                }
                return true;
            };
            for (int j = 0; j <= nblk; ++j) {
                if (j < nblk) {
                    if (!load(false, j)) break;
                    k_issued = j + 1;
                }
                if (j > 0) {
                    if (!load(true, j - 1)) break;
                    v_issued = j;
                }
            }
            if (lane == leader && *abort_flag) {
                // the copies in flight land before the CTA's memory goes away
                mbar_wait(qbar, 0, abort_flag, err, kTimeoutNs / 4);
                for (int j = k_issued - 2 < 0 ? 0 : k_issued - 2; j < k_issued; ++j)
                    mbar_wait(bar_addr(sb, B_K_FULL + (j & 1)), (j >> 1) & 1, abort_flag, err, kTimeoutNs / 4);
                for (int j = v_issued - 2 < 0 ? 0 : v_issued - 2; j < v_issued; ++j)
                    mbar_wait(bar_addr(sb, B_V_FULL + (j & 1)), (j >> 1) & 1, abort_flag, err, kTimeoutNs / 4);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer =================
        {
            uint32_t issuer = 0;
            bool issued_any = false;
            bool ok = mbar_wait(bar_addr(sb, B_Q), 0, abort_flag, err, kTimeoutNs);
            // O += P_j V_j, once the softmax warps have written P_j and V_j has landed
            auto issue_pv = [&](int j) -> bool {
                if (!mbar_wait(bar_addr(sb, B_V_FULL + (j & 1)), (j >> 1) & 1, abort_flag, err, kTimeoutNs) ||
                    !mbar_wait(bar_addr(sb, B_P_FULL + (j & 1)), (j >> 1) & 1, abort_flag, err, kTimeoutNs))
                    return false;
                tc_fence_after();
                if (elect_one(issuer)) {
                    const uint32_t vt = sb + OFF_V + (j & 1) * KV_STAGE;
                    #pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16_tmem_a(tmem + TM_O, tmem + TM_P + 32 * (j & 1) + 8 * k,
                                        smem_desc_sw128(vt + k * 2048, KV_PANEL, 1024), ID_PV,
                                        (j > 0 || k > 0) ? 1u : 0u);
                    umma_commit(bar_addr(sb, B_PV_DONE + (j & 1)));
                    umma_commit(bar_addr(sb, B_V_EMPTY + (j & 1)));
                }
                return true;
            };
            for (int j = 0; ok && j < nblk; ++j) {
                // S = Q K_j^T into the single S buffer, once the softmax warps have read S_{j-1}
                if (!mbar_wait(bar_addr(sb, B_K_FULL + (j & 1)), (j >> 1) & 1, abort_flag, err, kTimeoutNs) ||
                    (j > 0 && !mbar_wait(bar_addr(sb, B_S_FREE), (j - 1) & 1, abort_flag, err, kTimeoutNs))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one(issuer)) {
                    const uint32_t kt = sb + OFF_K + (j & 1) * KV_STAGE;
                    #pragma unroll
                    for (int k = 0; k < 8; ++k)
                        umma_f16(tmem + TM_S,
                                 smem_desc_sw128(sb + OFF_Q + (k >> 2) * Q_PANEL + (k & 3) * 32, 16, 1024),
                                 smem_desc_sw128(kt + (k >> 2) * KV_PANEL + (k & 3) * 32, 16, 1024), ID_QK, k > 0);
                    umma_commit(bar_addr(sb, B_S_FULL));
                    umma_commit(bar_addr(sb, B_K_EMPTY + (j & 1)));
                }
                issued_any = true;
                if (j > 0 && !issue_pv(j - 1)) ok = false;
            }
            if (ok) ok = issue_pv(nblk - 1);
            if (issued_any && !ok && lane == issuer) {
                // every MMA this thread issued completes before TMEM is released
                umma_commit(bar_addr(sb, B_DRAIN));
                mbar_wait(bar_addr(sb, B_DRAIN), 0, abort_flag, err, kTimeoutNs / 4);
            }
        }
        __syncwarp();
    } else {
        // ================= softmax and output (query row r, TMEM lane r) =================
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const int64_t qi = static_cast<int64_t>(i0) + r;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
        const bool leader = warp == 2 && lane == 0;
        Group grp{NB_SOFT, kSoftThreads, leader, abort_flag, err};
        // this row's window relative to the CTA's first query: keys i0 + rel, rel in [wlo, whi]
        const int64_t wlo = static_cast<int64_t>(r) - p.window + 1;
        const int64_t whi = r < L - i0 ? r : L - 1 - i0;
        float m = -INFINITY, l = 0.f;                        // running maximum (log2 units), sum
        bool ok = true;
        // Inside the loop the softmax warps meet at no group barrier: every wait is a warp's own
        // (all its lanes poll), so no warp waits for the slowest one.  A failed wait raises the
        // abort flag and takes its warp out of the loop; the other warps' waits then run out or
        // see the flag, and every thread meets the others once, at the consensus after the loop.
        for (int idx = 0; idx < nblk; ++idx) {
            const bool got = mbar_wait(bar_addr(sb, B_S_FULL), idx & 1, abort_flag, err, kTimeoutNs);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[64];
            tmem_load_2x32(tmem + TM_S + lane_addr, tmem + TM_S + lane_addr + 32, x);
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_S_FREE));             // all 128 read: the next Q K^T may overwrite S
            // the window, causality and the sequence end as a column range [c_lo, c_hi] of this
            // block; blocks inside every window of the warp skip the mask
            const int64_t kb = static_cast<int64_t>(j_first + idx) * kBN - i0;
            const int c_lo = static_cast<int>(wlo - kb < 0 ? 0 : (wlo - kb > kBN ? kBN : wlo - kb));
            const int c_hi = static_cast<int>(whi - kb < -1 ? -1 : (whi - kb > kBN - 1 ? kBN - 1 : whi - kb));
            if (!__all_sync(0xffffffffu, c_lo == 0 && c_hi == kBN - 1)) {
                #pragma unroll
                for (int c = 0; c < kBN; ++c) x[c] = c >= c_lo && c <= c_hi ? x[c] : -INFINITY;
            }
            float mx[8];
            #pragma unroll
            for (int j = 0; j < 8; ++j) mx[j] = fmaxf(x[j], x[j + 8]);
            #pragma unroll
            for (int c = 16; c < kBN; c += 8) {
                #pragma unroll
                for (int j = 0; j < 8; ++j) mx[j] = fmaxf(mx[j], x[c + j]);
            }
            const float bm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * p.xscale;
            // raise the row's reference maximum only when the block exceeds it by more than 8
            // (so P <= 2^8); O and l then shrink by 2^(m - m_new)
            const bool raise = bm > m + 8.f;
            const float mnew = raise ? bm : m;
            const float corr = raise && m != -INFINITY ? ex2_approx(m - mnew) : 1.f;
            // p = 2^(x xscale - m); a masked score (-inf) gives 0, and a row that has seen no key
            // yet (m = -inf) subtracts 0 instead
            const float msub = mnew == -INFINITY ? 0.f : mnew;
            uint32_t pk[32];
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
            #pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = ex2_approx(fmaf(x[2 * e], p.xscale, -msub));
                const float p1 = ex2_approx(fmaf(x[2 * e + 1], p.xscale, -msub));
                pk[e] = pack_bf16x2(p0, p1);
                ps[e & 3] += p0 + p1;
            }
            l = l * corr + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
            m = mnew;
            // P is double-buffered: P_idx takes the buffer of P_{idx-2}, free once O += P_{idx-2} V
            // is done (barrier idx & 1 completes once every two blocks: phase (idx - 2) / 2)
            if (idx >= 2)
                mbar_wait(bar_addr(sb, B_PV_DONE + (idx & 1)), ((idx - 2) >> 1) & 1, abort_flag, err, kTimeoutNs);
            tc_fence_after();
            if (__any_sync(0xffffffffu, corr != 1.f)) {
                // a raised maximum rescales O, so the latest O += P V (block idx - 1) must be done;
                // only this warp waits (a timeout raises the CTA's abort, which the group's next
                // wait sees)
                if (idx >= 1)
                    mbar_wait(bar_addr(sb, B_PV_DONE + ((idx - 1) & 1)), ((idx - 1) >> 1) & 1, abort_flag, err,
                              kTimeoutNs);
                tc_fence_after();
                rescale_o(tmem + TM_O + lane_addr, corr);
            }
            const uint32_t tp = tmem + TM_P + 32 * (idx & 1) + lane_addr;
            tmem_st16(tp, *reinterpret_cast<uint32_t(*)[16]>(pk));
            tmem_st16(tp + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_addr(sb, B_P_FULL + (idx & 1)));
        }
        // o = O / l after the last O += P V
        const bool mine =
            ok && mbar_wait(bar_addr(sb, B_PV_DONE + ((nblk - 1) & 1)), ((nblk - 1) >> 1) & 1, abort_flag, err, kTimeoutNs);
        uint32_t all;
        asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                     "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                     : "=r"(all) : "r"(mine ? 1u : 0u), "r"(NB_SOFT), "r"(kSoftThreads) : "memory");
        if (all) {
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            float* o32 = !p.out_bf16 && qi < L ? static_cast<float*>(p.o) + (static_cast<int64_t>(unit) * L + qi) * 128
                                               : nullptr;
            write_output(tmem + TM_O + lane_addr, inv_l, p.out_bf16 ? sb + OFF_Q : 0u, r, o32, sbase, sb);
            if (p.out_bf16) {
                // the Q tile is free (every MMA is done) and holds o, swizzled like Q; rows past L
                // are clipped by the store
                fence_proxy_async_smem();
                grp.sync();
                if (leader) {
                    if (dbg_ok(i0 < L && unit < p.units, err)) {
                        tma_store_3d(&tm_o, sb + OFF_Q, 0, i0, unit);
                        tma_store_3d(&tm_o, sb + OFF_Q + Q_PANEL, 64, i0, unit);
                    }
                    bulk_commit_group();
                    bulk_wait_all();
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace swa

bool swa_tc_supports(int dtype_bf16, int d) { return dtype_bf16 && d == 128; }

cudaError_t launch_swa_tc(const SwaCall& c, cudaStream_t stream)
{
    using namespace swa;
    if (c.units == 0 || c.L == 0) return cudaSuccess;
    const int64_t nqb = (c.L + kBM - 1) / kBM;
    if (c.units * nqb >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_bf16_map_3d(&mq, c.q, c.units, c.L, kBM, sw) || !make_bf16_map_3d(&mk, c.k, c.units, c.L, kBN, sw) ||
        !make_bf16_map_3d(&mv, c.v, c.units, c.L, kBN, sw))
        return cudaErrorInvalidValue;
    // o (bf16 output): stored from the swizzled staging tile by TMA
    if (c.out_bf16 && !make_bf16_map_3d(&mo, c.o, c.units, c.L, kBM, sw)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(swa_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess) return e;
    NvtxRange range("lt2 sliding-window prefill (tensor core)");
    Params p;
    p.o = c.o;
    p.L = c.L;
    p.window = static_cast<int>(c.window < c.L ? c.window : c.L);
    p.xscale = c.scale * 1.4426950408889634f;               // log2(e)
    p.nqb = static_cast<int>(nqb);
    p.units = static_cast<int>(c.units);
    p.out_bf16 = c.out_bf16;
    p.err = c.err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(c.units * nqb), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, swa_prefill_tc_kernel, mq, mk, mv, c.out_bf16 ? mo : mq, p);
}

}  // namespace lt2
