// gdr_tc_common.cuh -- pieces shared by the tensor-core chunked prefills (scalar and per-key
// gating): group waits, the 16x16-block helpers of the triangular solve on warp-level fp16
// mma, the solve itself, the diagonal-block inverse and the in-place bf16 -> fp16 conversion.
//
// All tiles here are row-major fp16 with 128-byte rows under the 128-byte swizzle (`sw128`),
// the layout the tcgen05 descriptors of both kernels use.
#pragma once

#include <cstdint>

#include "gdr_common.cuh"
#include "sm100_primitives.cuh"

namespace lt2 {
namespace tcc {

using namespace sm100;

constexpr int kD = 128;                          // d_k = d_v
// Bound of every mbarrier wait: 4 s in the product build; the debug build (LT2_DEBUG) shortens it
// so that its fault-injection test ends in milliseconds.
#ifndef LT2_WAIT_TIMEOUT_NS
#define LT2_WAIT_TIMEOUT_NS 4000000000ull
#endif
constexpr uint64_t kWaitTimeoutNs = LT2_WAIT_TIMEOUT_NS;
constexpr int kAdiagRow = 17;                    // fp32 diagonal blocks: rows padded to 17

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// A group of warps that waits together: every thread polls the mbarrier itself, then one
// barrier reduction (bar.red.and) over the group's named barrier makes the outcome the group's --
// if any thread gave up (timeout or abort) all of them see it, so the group always leaves a
// pipeline at the same step.  (A single polling leader with the rest parked at the named barrier
// costs the leader's warp a reconvergence per wait.)  `leader` names the one thread that makes
// the group's single arrivals.
struct Group {
    int nb;             // named barrier id
    int nthreads;
    bool leader;
    volatile int* abort_flag;
    unsigned int* err;

    __device__ bool wait(uint32_t bar0, uint32_t par0, uint32_t bar1 = 0, uint32_t par1 = 0,
                         uint32_t bar2 = 0, uint32_t par2 = 0)
    {
        bool ok = mbar_wait(bar0, par0, abort_flag, err, kWaitTimeoutNs);
        if (ok && bar1) ok = mbar_wait(bar1, par1, abort_flag, err, kWaitTimeoutNs);
        if (ok && bar2) ok = mbar_wait(bar2, par2, abort_flag, err, kWaitTimeoutNs);
        uint32_t all;
        asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                     "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                     : "=r"(all) : "r"(ok ? 1u : 0u), "r"(nb), "r"(nthreads) : "memory");
        return all != 0;
    }
    __device__ void sync() { named_sync(nb, nthreads); }
};

// --- 16x16 fp16 blocks of row-major 128B-swizzled tiles, as m16n8k16 fragments ------------
__device__ __forceinline__ void frag_a(uint32_t tile, int row0, int col0, int lane, uint32_t (&a)[4])
{
    const uint32_t row = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const uint32_t chunk = (col0 >> 3) + (lane >> 4);
    ldsm_x4(sw128(tile, row, chunk), a);
}
__device__ __forceinline__ void frag_b(uint32_t tile, int k0, int n0, int lane, uint32_t (&b)[4])
{
    const uint32_t row = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const uint32_t chunk = (n0 >> 3) + (lane >> 4);
    ldsm_x4_trans(sw128(tile, row, chunk), b);
}
__device__ __forceinline__ void mma_block(float (&c)[2][4], const uint32_t (&a)[4], const uint32_t (&b)[4])
{
    mma16816(c[0], a, b[0], b[1]);
    mma16816(c[1], a, b[2], b[3]);
}
__device__ __forceinline__ void c_to_a(const float (&c)[2][4], uint32_t (&a)[4])
{
    a[0] = pack_half2(c[0][0], c[0][1]);
    a[1] = pack_half2(c[0][2], c[0][3]);
    a[2] = pack_half2(c[1][0], c[1][1]);
    a[3] = pack_half2(c[1][2], c[1][3]);
}
__device__ __forceinline__ void store_block(uint32_t tile, int row0, int col0, int lane,
                                            const float (&c)[2][4], float sign)
{
    const uint32_t g = lane >> 2, tq = lane & 3;
    #pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
        const uint32_t chunk = (col0 >> 3) + nb;
        sts32(sw128(tile, row0 + g, chunk) + tq * 4, pack_half2(sign * c[nb][0], sign * c[nb][1]));
        sts32(sw128(tile, row0 + g + 8, chunk) + tq * 4, pack_half2(sign * c[nb][2], sign * c[nb][3]));
    }
}
__device__ __forceinline__ void zero_c(float (&c)[2][4])
{
    #pragma unroll
    for (int i = 0; i < 2; ++i)
        #pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] = 0.f;
}

// Zeroes the entries above the diagonal of a diagonal 16x16 block held as an m16n8k16 A
// fragment (a0: row g, columns 2tq..2tq+1; a1: row g+8, same columns; a2/a3: columns +8).
__device__ __forceinline__ void keep_lower(uint32_t (&a)[4], int lane)
{
    const int g = lane >> 2, c0 = 2 * (lane & 3);
    const uint32_t m = (c0 + 1 <= g) ? 0xffffffffu : ((c0 <= g) ? 0x0000ffffu : 0u);
    a[0] &= m;
    a[2] = 0u;
    a[3] &= m;
}

__device__ __forceinline__ uint4 pack8_half(const float* v)
{
    uint4 w;
    w.x = pack_half2(v[0], v[1]);
    w.y = pack_half2(v[2], v[3]);
    w.z = pack_half2(v[4], v[5]);
    w.w = pack_half2(v[6], v[7]);
    return w;
}

// One 16-row block `rb` of X = [T; PT] for a chunk of 16*nblk tokens: T = (I + A)^{-1} in rows
// 0..16*nblk-1, PT below it.  X solves X (I + A) = [I; P]; with A strictly lower triangular
// this is a back substitution over the 16-column blocks j = nblk-1, ..., 0:
//     X_j = (E_j + sum_{k>j} X_k (-A)_{kj}) D_j,      D_j = (I + A_jj)^{-1}  (already in TP)
// where E = I for the T rows and E = P for the PT rows, and X_j = 0 right of the diagonal
// block (T_jj = D_j itself).  AS holds -A.  Each X_j goes to TP as soon as it is known and is
// read back from there by the warp's later steps, so both loops stay rolled.  -A and P start
// at columns as_col / ps_col of their tiles (two 32-column matrices may share 128-byte rows).
static __device__ __noinline__ void solve_row_block(uint32_t tp, uint32_t as, int as_col, uint32_t ps, int ps_col,
                                                    int rb, int nblk, int lane)
{
    const bool is_t = rb < nblk;
    const int qd = is_t ? rb : rb - nblk;       // diagonal column block of this row block
    #pragma unroll 1
    for (int j = is_t ? qd - 1 : qd; j >= 0; --j) {
        float acc[2][4];
        zero_c(acc);
        #pragma unroll 1
        for (int k = j + 1; k <= qd; ++k) {
            uint32_t xa[4], b[4];
            frag_a(tp, 16 * rb, 16 * k, lane, xa);
            frag_b(as, 16 * k, as_col + 16 * j, lane, b);
            mma_block(acc, xa, b);              // += X_k (-A)_kj
        }
        uint32_t dj[4];
        frag_b(tp, 16 * j, 16 * j, lane, dj);
        float x[2][4];
        zero_c(x);
        if (!is_t) {
            uint32_t pa[4];
            frag_a(ps, 16 * qd, ps_col + 16 * j, lane, pa);
            if (j == qd) keep_lower(pa, lane);
            mma_block(x, pa, dj);               // P_qj D_j
        }
        if (j < qd) {
            uint32_t aa[4];
            c_to_a(acc, aa);
            mma_block(x, aa, dj);
        }
        store_block(tp, 16 * rb, 16 * j, lane, x, 1.f);
        __syncwarp();                           // X_j is read back by this warp's next steps
    }
}

// Row i = r & 15 of D_b = (I + A_bb)^{-1}, b = r >> 4, from the fp32 copy `ad` of -A_bb (rows
// padded to kAdiagRow): x_j = delta_ij + sum_{m>j} x_m (-A)_mj for j = 15..0.  The sum runs from
// m = 15 down so that only its last term waits for x_{j+1}.  Written to row r, columns
// 16b..16b+15 of the fp16 tile `tp`.
__device__ __forceinline__ void diag_block_inverse_row(uint32_t tp, int r, const float* ad)
{
    const int b = r >> 4, i = r & 15;
    float x[16];
    #pragma unroll
    for (int j = 15; j >= 0; --j) {
        float acc = 0.f;
        #pragma unroll
        for (int m = 15; m > j; --m) acc = fmaf(x[m], ad[m * kAdiagRow + j], acc);
        x[j] = (j == i) ? 1.f : ((j < i) ? acc : 0.f);
    }
    sts128(sw128(tp, r, 2 * b), pack8_half(x));
    sts128(sw128(tp, r, 2 * b + 1), pack8_half(x + 8));
}

// bf16 -> fp16, in place, for `n16` 16-byte vectors starting at shared address `base`.
template <typename LdFn, typename StFn>
__device__ __forceinline__ void convert_tile(uint32_t base, int n16, int lane, LdFn lds, StFn sts)
{
    for (int i0 = 0; i0 < n16; i0 += 8 * 32) {
        uint4 w[8];
        #pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = lds(base + static_cast<uint32_t>(i0 + i * 32 + lane) * 16u);
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint4 hv;
            hv.x = pack_half2(bf16_lo(w[i].x), bf16_hi(w[i].x));
            hv.y = pack_half2(bf16_lo(w[i].y), bf16_hi(w[i].y));
            hv.z = pack_half2(bf16_lo(w[i].z), bf16_hi(w[i].z));
            hv.w = pack_half2(bf16_lo(w[i].w), bf16_hi(w[i].w));
            sts(base + static_cast<uint32_t>(i0 + i * 32 + lane) * 16u, hv);
        }
    }
}

// False for an infinity or a NaN.
__device__ __forceinline__ bool is_finite(float x) { return fabsf(x) <= 3.402823466e38f; }

// bf16 -> fp16, in place, of a 64-row tile held as two 64 x 64 panels (columns 0-63 at p0,
// 64-127 at p1, 128-byte swizzled rows), every row divided by its L2 norm on the way (the fused
// normalisation of q and k): lane l owns rows l and l + 32.  Pass 1 sums the squares of the row
// in fp32, pass 2 rescales and converts; each pass loads a panel's eight vectors together.
template <typename LdFn, typename StFn>
__device__ __forceinline__ void convert_rows_l2(uint32_t p0, uint32_t p1, int lane, LdFn lds, StFn sts)
{
    #pragma unroll 1
    for (int rr = 0; rr < 2; ++rr) {
        const uint32_t r = static_cast<uint32_t>(lane + 32 * rr);
        float ss = 0.f;
        #pragma unroll 1
        for (int pn = 0; pn < 2; ++pn) {
            uint4 w[8];
            #pragma unroll
            for (uint32_t c = 0; c < 8; ++c) w[c] = lds(sw128(pn ? p1 : p0, r, c));
            #pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t ws[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = bf16_lo(ws[e]), hi = bf16_hi(ws[e]);
                    ss = fmaf(lo, lo, ss);
                    ss = fmaf(hi, hi, ss);
                }
            }
        }
        const float inv = inv_l2_fast(ss);
        #pragma unroll 1
        for (int pn = 0; pn < 2; ++pn) {
            uint4 w[8];
            #pragma unroll
            for (uint32_t c = 0; c < 8; ++c) w[c] = lds(sw128(pn ? p1 : p0, r, c));
            #pragma unroll
            for (uint32_t c = 0; c < 8; ++c) {
                uint4 h;
                h.x = pack_half2(bf16_lo(w[c].x) * inv, bf16_hi(w[c].x) * inv);
                h.y = pack_half2(bf16_lo(w[c].y) * inv, bf16_hi(w[c].y) * inv);
                h.z = pack_half2(bf16_lo(w[c].z) * inv, bf16_hi(w[c].z) * inv);
                h.w = pack_half2(bf16_lo(w[c].w) * inv, bf16_hi(w[c].w) * inv);
                sts(sw128(pn ? p1 : p0, r, c), h);
            }
        }
    }
}

// Chain thread j: column j of the final state (row j of S^T in TMEM) to S_out.  Returns false
// if any entry is not finite.
static __device__ __noinline__ bool store_final_state(uint32_t tm_s, float* so)
{
    bool fin = true;
    #pragma unroll 1
    for (int piece = 0; piece < 4; piece += 2) {
        float v[64];
        tmem_load_2x32(tm_s + 32 * piece, tm_s + 32 * piece + 32, v);
        #pragma unroll
        for (int d = 0; d < 64; ++d) {
            fin &= is_finite(v[d]);
            so[(32 * piece + d) * kD] = v[d];
        }
    }
    return fin;
}

}  // namespace tcc
}  // namespace lt2
