/*
 * lt2_gdr.h -- C ABI of the B200 (sm_100a) looped gated-delta-rule mixer.
 *
 * The operation.  "LT2 transformer looped a tempo lineare" (paithon.it), section
 * "Sostituire il motore", displayed equation: a linear mixer keeps a d_k x d_v state per
 * (batch, head) and, for every token t, applies
 *
 *     S_t = A_t S_{t-1} + beta_t k_t v_t^T,      A_t = Diag(alpha_t) (I - beta_t k_t k_t^T)
 *
 * and this library reads it out as o_t = S_t^T q_t (after token t's update, no extra
 * scale).  alpha_t is a scalar per (token, head) ("GDN" gating, Diag(alpha) = alpha I) or a
 * d_k vector per (token, head) (per-key-channel "KDA-style" gating).  Section "Profondita
 * presa in prestito" of the same page re-applies one weight-tied block T times; every loop
 * runs its own recurrence over its own q/k/v with its own initial and final state (the
 * page lists carrying state from loop to loop as unexplored, section "Dove il quadro si
 * incrina").  So every (loop, batch, head) triple is independent.
 *
 * Layouts (all row-major, contiguous, last index fastest; tau = loop index):
 *   q, k     [T][B][H][L][dk]    dtype of dims->dtype
 *   v        [T][B][H][L][dv]    dtype of dims->dtype
 *   o        [T][B][H][L][dv]    dims->out_dtype (default: same as dims->dtype)
 *   alpha    [T][B][H][L] fp32 (LT2_GATE_SCALAR) or [T][B][H][L][dk] fp32 (both per-key gates)
 *   beta     [T][B][H][L] fp32
 *   S0, S_out, S  [T][B][H][dk][dv] fp32 (d_v fastest)
 * Decode uses the same layouts with L = 1.
 *
 * Ownership and execution.  Every pointer is a DEVICE pointer owned by the caller (the
 * library never allocates, frees or synchronises on these entry points).  Work is enqueued
 * on `stream` (a cudaStream_t; NULL = legacy default stream) of the current device and
 * completes asynchronously.  The T loops are launched back to back on that stream with no
 * host synchronisation.
 *
 * Errors.  Argument validation happens before any launch and returns synchronously.  A
 * failed launch returns LT2_ERR_CUDA (the CUDA error text is available from
 * lt2_last_cuda_error_string()).  Waits inside kernels are bounded: a wait that runs out
 * makes the kernel record LT2_ERR_DEVICE_TIMEOUT in a device-side status word and return;
 * lt2_gdr_last_device_error() reads (and clears) it.  No C++ exception crosses the ABI.
 *
 * Supported set.
 *   The tensor-core chunked prefills serve bf16 inputs with dk = dv = 128, for scalar gating
 *   (64-token chunks) and per-key gating (32-token chunks); every other supported shape runs
 *   on the CUDA-core path.  With per-key gating, a chunk in which some key decays by more than
 *   ~e^-19, or with any alpha <= 0 (a reset), is evaluated token by token inside the same
 *   kernel (exact, slower).  The tensor-core paths take their operands in fp16: alpha is
 *   expected in (0, 1] (a growing alpha > 1 works while the state stays below ~3e4 in
 *   magnitude), with |q|, |k| entries of order 1.
 *   fp32 inputs: dk, dv multiples of 8 up to 128 (CUDA-core fp32 arithmetic throughout).
 *   bf16 inputs: dk, dv multiples of 8 up to 128.
 *   Any L >= 0 (a ragged final chunk is fine; L = 0 copies S0 to S_out).
 *   Pointers must be 16-byte aligned.  o must not alias any input.  S0 == S_out is allowed
 *   (in-place resume of a segmented prefill).
 */
#ifndef LT2_GDR_H
#define LT2_GDR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lt2_status {
    LT2_OK = 0,
    LT2_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, aliasing, bad enum */
    LT2_ERR_UNSUPPORTED = 2,      /* valid but outside the supported set above            */
    LT2_ERR_WORKSPACE = 3,        /* workspace smaller than lt2_gdr_prefill_workspace_bytes */
    LT2_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed                   */
    LT2_ERR_DEVICE_TIMEOUT = 5    /* a bounded in-kernel wait ran out (see header comment)  */
} lt2_status;

typedef enum lt2_dtype { LT2_DTYPE_F32 = 0, LT2_DTYPE_BF16 = 1 } lt2_dtype;

/* Storage type of the output o.  All arithmetic is fp32 either way; a bf16 output is the
 * fp32 result rounded to nearest-even (bit-identical to rounding the fp32 output). */
typedef enum lt2_out_dtype {
    LT2_OUT_SAME = 0,   /* same as the inputs (lt2_gdr_dims.dtype) */
    LT2_OUT_F32 = 1,
    LT2_OUT_BF16 = 2
} lt2_out_dtype;
/* Gating.  PER_KEY is the equation as printed, A_t = Diag(alpha_t)(I - beta_t k_t k_t^T): the
 * delta step, then the per-key decay.  PER_KEY_DECAY_FIRST takes the other reading of the same
 * symbols, A_t = (I - beta_t k_t k_t^T) Diag(alpha_t): the decay, then the delta step on the
 * decayed state (the order a right-multiplying convention for S gives).  Both take alpha as a
 * d_k vector per token; for a scalar alpha the two are the same matrix. */
typedef enum lt2_gate {
    LT2_GATE_SCALAR = 0,
    LT2_GATE_PER_KEY = 1,
    LT2_GATE_PER_KEY_DECAY_FIRST = 2
} lt2_gate;

/* Prefill algorithm selector (lt2_gdr_dims.algo).  AUTO picks the tensor-core kernel
 * whenever it supports the shape.  The others force one path (for testing). */
typedef enum lt2_algo {
    LT2_ALGO_AUTO = 0,
    LT2_ALGO_TENSOR_CORE = 1, /* tcgen05/TMA chunked prefill: bf16, dk = dv = 128 only */
    LT2_ALGO_CUDA_CORE = 2    /* token-sequential fp32 CUDA-core prefill, any supported shape */
} lt2_algo;

/* Problem description.  All sizes are element counts. */
typedef struct lt2_gdr_dims {
    int64_t T;       /* loops (weight-tied block repetitions)                    */
    int64_t B;       /* batch                                                    */
    int64_t H;       /* heads                                                    */
    int64_t L;       /* tokens per sequence (1 for decode)                       */
    int64_t dk;      /* key / query width                                        */
    int64_t dv;      /* value width                                              */
    int32_t dtype;   /* lt2_dtype of q, k and v                                  */
    int32_t gate;    /* lt2_gate                                                 */
    int32_t algo;    /* lt2_algo (prefill only; ignored by decode)               */
    int32_t out_dtype; /* lt2_out_dtype of o                                     */
} lt2_gdr_dims;

/*
 * Bytes of device workspace lt2_gdr_prefill needs for `dims` (0 when none).  Pure host
 * function; returns 0 for invalid dims as well.
 */
size_t lt2_gdr_prefill_workspace_bytes(const lt2_gdr_dims* dims);

/*
 * Chunked prefill over all T loops (the displayed equation over L tokens, for every
 * (loop, batch, head)).  Writes every o_t and, if S_out is non-NULL, the state after the
 * last token.  S0 == NULL means a zero initial state.  `workspace` may be NULL when
 * lt2_gdr_prefill_workspace_bytes(dims) is 0.
 */
lt2_status lt2_gdr_prefill(const lt2_gdr_dims* dims,
                           const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta,
                           const float* S0,
                           void* o, float* S_out,
                           void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * One decode token per (loop, batch, head): dims->L must be 1.  S is read and replaced in
 * place by the state after the token; o receives o = S_new^T q.  Each state is streamed
 * through HBM once (read once, written once).
 */
lt2_status lt2_gdr_decode(const lt2_gdr_dims* dims,
                          const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta,
                          float* S, void* o,
                          void* stream);

/*
 * Status word written by bounded in-kernel waits on the CURRENT device.  Blocks until all
 * previously issued work on the device has finished (it reads device memory), returns
 * LT2_ERR_DEVICE_TIMEOUT if any kernel gave up on a wait since the last call (and clears
 * the word), LT2_OK otherwise, or LT2_ERR_CUDA if the read itself failed.
 */
lt2_status lt2_gdr_last_device_error(void);

/* Static, human-readable name of a status code. */
const char* lt2_status_string(lt2_status status);

/* Text of the last CUDA error seen by this library on the calling thread ("" if none). */
const char* lt2_last_cuda_error_string(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int lt2_gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LT2_GDR_H */
