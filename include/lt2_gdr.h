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
 * Ownership and execution.  Every pointer is a DEVICE pointer owned by the caller, in memory
 * of the CURRENT device (cudaGetDevice); the library never allocates, frees or synchronises on
 * the compute entry points.  Work is enqueued on `stream` (a cudaStream_t of the current
 * device; NULL = legacy default stream) and completes asynchronously.  The T loops are
 * launched back to back on that stream with no host synchronisation.
 *
 * Errors.  Argument validation happens before any launch and returns synchronously: a pointer
 * that is not device memory of the current device is LT2_ERR_INVALID_ARGUMENT.  A failed
 * launch returns LT2_ERR_CUDA (the CUDA error text is available from
 * lt2_last_cuda_error_string()).  Conditions found while the kernels run are recorded as bit
 * flags in one status word per device, shared by every call on that device, and read (and
 * cleared) by lt2_gdr_last_device_error():
 *   - waits inside kernels are bounded; a wait that runs out makes the kernel record
 *     LT2_ERR_DEVICE_TIMEOUT, release what it holds and return;
 *   - a tensor-core prefill whose output or final state is not finite (its fp16 operands went
 *     out of range, or an input was not finite) records LT2_ERR_RANGE; the results of that
 *     call are then not valid, and LT2_ALGO_CUDA_CORE computes the same call in fp32.
 * No C++ exception crosses the ABI.
 *
 * Supported set.
 *   The tensor-core chunked prefills serve bf16 inputs with dk = dv = 128, for scalar gating
 *   (64-token chunks) and per-key gating (32-token chunks); every other supported shape runs
 *   on the CUDA-core path.  With per-key gating, a chunk in which some key decays by more than
 *   ~e^-19, or with any alpha <= 0 (a reset), is evaluated token by token inside the same
 *   kernel (exact, slower).  The tensor-core paths take their operands in fp16: alpha is
 *   expected in (0, 1] (a growing alpha > 1 works while the state stays below ~3e4 in
 *   magnitude), with |q|, |k| entries of order 1.  Outside that range the call records
 *   LT2_ERR_RANGE instead of returning silent infinities.  Scalar gating takes any real alpha
 *   (alpha = 0 is a reset; a negative alpha flips the sign of the decayed state).
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
    LT2_ERR_DEVICE_TIMEOUT = 5,   /* a bounded in-kernel wait ran out (see header comment)  */
    LT2_ERR_RANGE = 6,            /* a tensor-core path produced non-finite results         */
    LT2_ERR_DEVICE_CHECK = 7,     /* a debug build's device-side check failed (lt2_gdr_debug.h) */
    LT2_ERR_SEQLENS = 8           /* packed-sequence offsets out of order or past the packed length */
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
 * The steps on either side of the mixer, fused into its kernels: the prologue that
 * turns a layer's raw projections into the recurrence's inputs, and the sigmoid output gate of
 * "LT2 transformer looped a tempo lineare", section "Dove il quadro si incrina" (a sigmoid gate
 * inside the loop keeps the state norm under control; the wispaper.ai blog, section "Critical
 * Insight: The Attention Sink Mitigation", calls it an SDPA output gate).  A zeroed struct
 * selects none of them, which is exactly lt2_gdr_prefill / lt2_gdr_decode.
 */
typedef struct lt2_gdr_fused {
    int32_t qk_l2norm;     /* 1: q and k are raw; every (token, head) row is divided by
                              max(||row||_2, 1e-12) inside the kernels before it is used        */
    int32_t gate_logits;   /* 1: alpha and beta hold logits a, b (same layouts as alpha, beta):
                              beta = sigmoid(b), alpha = exp(-softplus(a) * alpha_scale)       */
    float alpha_scale;     /* c of the alpha formula above (used when gate_logits = 1)          */
    int32_t reserved;      /* must be 0                                                          */
    const void* z;         /* output gate logits, dims->dtype, layout of v ([T][B][H][L][dv]);
                              NULL = no gate.  Else every output is o <- sigmoid(z) * o          */
} lt2_gdr_fused;

/*
 * Bytes of device workspace lt2_gdr_prefill can use for `dims`: one 4-byte flag per (loop, batch,
 * head) unit, rounded up to 256, for scalar gating with bf16 inputs and d = 128 (the tensor-core
 * kernel); 0 otherwise and for invalid dims.  Pure host function, no CUDA call.
 * The workspace is optional.  Given (with S_out, and more units than the GPU has SMs), the
 * tensor-core kernel runs every loop in ONE balanced launch: one CTA per SM takes an equal share
 * of all units' 64-token chunks, so no SM idles through a partial second wave; a unit split
 * between two CTAs hands its state over through S_out and a flag in the workspace.  Without it,
 * one launch per loop and one CTA per unit.  The results are the same bit for bit either way.
 */
size_t lt2_gdr_prefill_workspace_bytes(const lt2_gdr_dims* dims);

/*
 * Prefill: the recurrence of "LT2 transformer looped a tempo lineare", section "Sostituire il
 * motore", displayed equation, over all L tokens of every (loop, batch, head), for all T
 * loops of section "Profondita presa in prestito", each loop with its own q/k/v, S0 and final
 * state.  Writes every o_t = S_t^T q_t and, if S_out is non-NULL, the state after the last
 * token.
 *   dims       problem sizes, dtypes, gating, algorithm (host pointer, read during the call)
 *   q, k, v    inputs in the layouts above (device, read only)
 *   alpha      decay: [T][B][H][L] fp32 for LT2_GATE_SCALAR, [T][B][H][L][dk] per key
 *   beta       write strength [T][B][H][L] fp32
 *   S0         initial states, or NULL for zero states
 *   o          outputs, dims->out_dtype (device, written; must not alias an input)
 *   S_out      final states, or NULL (may equal S0 exactly: in-place resume)
 *   workspace  NULL, or device scratch of lt2_gdr_prefill_workspace_bytes(dims) bytes (16-byte
 *              aligned, not overlapping any other argument; the library zeroes what it uses, on
 *              `stream`).  Optional: see lt2_gdr_prefill_workspace_bytes.  Calls that overlap on
 *              the GPU need workspaces of their own
 *   stream     cudaStream_t of the current device
 * Returns LT2_OK once the launches are enqueued; LT2_ERR_INVALID_ARGUMENT, _UNSUPPORTED or
 * _WORKSPACE before any launch; LT2_ERR_CUDA if a launch failed.  Device-side conditions come
 * later from lt2_gdr_last_device_error().
 */
lt2_status lt2_gdr_prefill(const lt2_gdr_dims* dims,
                           const void* q, const void* k, const void* v,
                           const float* alpha, const float* beta,
                           const float* S0,
                           void* o, float* S_out,
                           void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * lt2_gdr_prefill with the fused prologue and output gate that `fused` selects (NULL or a zeroed
 * struct: exactly lt2_gdr_prefill).  q, k, alpha and beta then hold the raw values the struct
 * describes, and z, when given, must not alias o.  Every path of lt2_gdr_prefill fuses the steps
 * into its own kernels: nothing extra is written to or read back from global memory.
 * LT2_ERR_INVALID_ARGUMENT for reserved != 0, a flag other than 0 or 1, a non-finite or
 * negative alpha_scale, a misaligned z or a z that overlaps o.
 */
lt2_status lt2_gdr_prefill_fused(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused,
                                 const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta,
                                 const float* S0,
                                 void* o, float* S_out,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * The same prefill over packed sequences of different lengths ("varlen" batches: the pages batch
 * sequences but give no layout; this is the plainest packed one).  dims->B is the number of
 * sequences and dims->L the packed length Ntot; sequence b holds tokens cu_seqlens[b] ..
 * cu_seqlens[b+1]-1 of every (loop, head).  Each (loop, sequence, head) is an independent
 * recurrence, exactly as a separate lt2_gdr_prefill call on that sequence would compute it.
 *   cu_seqlens  int64 [B+1] (device, 8-byte aligned, read only): 0 <= cu[b] <= cu[b+1] <= Ntot;
 *               offsets out of that order are reported as LT2_ERR_SEQLENS by
 *               lt2_gdr_last_device_error() and their sequences left unwritten
 *   q, k, z     [T][H][Ntot][dk] (z: [T][H][Ntot][dv]), dims->dtype
 *   v, o        [T][H][Ntot][dv]
 *   alpha       [T][H][Ntot] fp32 for scalar gating, [T][H][Ntot][dk] per key; beta [T][H][Ntot]
 *   S0, S_out   [T][B][H][dk][dv] fp32, as for lt2_gdr_prefill (an empty sequence passes S0,
 *               or zeros, to S_out)
 *   fused       as lt2_gdr_prefill_fused (NULL: none)
 * bf16 inputs with d = 128 run on the tensor-core kernels, scalar or per-key gating, either
 * order (each CTA reads its sequence's rows; the rows of a partial last chunk that belong to the
 * next sequence are masked out and its outputs are written row by row); every other case runs on
 * the CUDA-core path.  No workspace is used (workspace may be NULL).  Same return convention as
 * lt2_gdr_prefill.
 */
lt2_status lt2_gdr_prefill_varlen(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused,
                                  const int64_t* cu_seqlens,
                                  const void* q, const void* k, const void* v,
                                  const float* alpha, const float* beta,
                                  const float* S0,
                                  void* o, float* S_out,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * Bytes of device workspace lt2_gdr_backward needs for `dims` (0 for invalid dims): per
 * (unit, 32-column slice of d_v), a checkpoint of the state every 32 tokens and the 33 states of
 * one chunk, fp32.  Pure host function, no CUDA call.
 */
size_t lt2_gdr_backward_workspace_bytes(const lt2_gdr_dims* dims);

/*
 * Backward pass of lt2_gdr_prefill (training; the pages train looped models but give no training
 * kernel): the gradients of loss = sum(dO * o) + sum(dS_L * S_out) with respect to every input of
 * the recurrence of "LT2 transformer looped a tempo lineare", section "Sostituire il motore",
 * displayed equation, for every (loop, batch, head) unit.  The reverse-mode derivative of each
 * line of the token step, swept from the last token to the first with the states recomputed from
 * 64-token checkpoints (no forward activations are needed from the caller).  fp32 arithmetic on
 * CUDA cores, every gating and order of lt2_gdr_dims (dims->algo: AUTO or CUDA_CORE;
 * TENSOR_CORE returns LT2_ERR_UNSUPPORTED; out_dtype is ignored).
 *   q, k, v, alpha, beta, S0   the forward call's inputs (layouts and dtypes of lt2_gdr_prefill)
 *   dO          upstream gradient of o, [T][B][H][L][dv], dims->dtype (device, read only)
 *   dS_L        upstream gradient of S_out, [T][B][H][dk][dv] fp32, or NULL for zero
 *   dq, dk      [T][B][H][L][dk] fp32 (device, written)
 *   dv          [T][B][H][L][dv] fp32
 *   dalpha      fp32, the layout of alpha; dbeta [T][B][H][L] fp32
 *   dS0         [T][B][H][dk][dv] fp32, or NULL (not wanted)
 *   workspace   lt2_gdr_backward_workspace_bytes(dims) bytes of device scratch (16-byte aligned)
 * No gradient may overlap an input, another gradient or the workspace.  Same return convention
 * as lt2_gdr_prefill (LT2_ERR_WORKSPACE for a missing or short workspace).
 */
lt2_status lt2_gdr_backward(const lt2_gdr_dims* dims,
                            const void* q, const void* k, const void* v,
                            const float* alpha, const float* beta, const float* S0,
                            const void* dO, const float* dS_L,
                            float* dq, float* dk, float* dv, float* dalpha, float* dbeta, float* dS0,
                            void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * lt2_gdr_backward without a workspace argument, for callers that cannot allocate device memory:
 * a program whose device memory is handed out entirely by a host application's or framework's own
 * allocator, or a service that must not call cudaMalloc while it serves (the call can block the
 * whole device).  This entry point allocates nothing: its scratch is a fixed 64 MiB array of
 * device memory inside the library, reserved on every GPU that loads the library until the
 * process exits.  (The paper has no counterpart: this is the library's own arrangement.)
 *   Arguments, layouts and results: exactly those of lt2_gdr_backward.
 *   Limit: a problem whose lt2_gdr_backward_workspace_bytes(dims) exceeds 64 MiB (67108864 bytes)
 *          returns LT2_ERR_WORKSPACE before any launch; for d_k = d_v = 128 that is 15 (loop,
 *          batch, head) units of 1,024 tokens, or 3 units of 8,192.
 *   Set-up: the first call on each device looks up the array's device address (with that device
 *          current) and keeps it; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array.  Nothing in it has to start at zero
 *          (a call writes each word before it reads it), but calls that overlap on the GPU, from
 *          two streams or two host threads, race on it: serialise them.
 */
lt2_status lt2_gdr_backward_static(const lt2_gdr_dims* dims,
                                   const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const float* S0,
                                   const void* dO, const float* dS_L,
                                   float* dq, float* dk, float* dv, float* dalpha, float* dbeta, float* dS0,
                                   void* stream);

/*
 * Decode: one step of the same recurrence ("LT2 transformer looped a tempo lineare", section
 * "Sostituire il motore", displayed equation) for one new token per (loop, batch, head);
 * dims->L must be 1 and dims->algo is ignored.  S [T][B][H][dk][dv] fp32 is read and replaced
 * in place by the state after the token; o receives o = S_new^T q.  Each state is streamed
 * through HBM once (read once, written once).  q, k, v, alpha, beta, o: the layouts above with
 * L = 1; o must alias neither S nor an input.  Same return convention as lt2_gdr_prefill.
 */
lt2_status lt2_gdr_decode(const lt2_gdr_dims* dims,
                          const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta,
                          float* S, void* o,
                          void* stream);

/* lt2_gdr_decode with the fused prologue and output gate of `fused` (as lt2_gdr_prefill_fused,
 * with L = 1). */
lt2_status lt2_gdr_decode_fused(const lt2_gdr_dims* dims, const lt2_gdr_fused* fused,
                                const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta,
                                float* S, void* o,
                                void* stream);

/*
 * The other mixer of "LT2 transformer looped a tempo lineare", section "Sostituire il motore":
 * sliding-window (sparse) attention, every token looking at the w most recent positions, itself
 * included; section "Il giro trasforma il calcolo in contesto": repeated over T loops, the window
 * reaches back O(T w) tokens.  For every (loop, batch, head) unit and token t,
 *     o_t = sum_{s = max(0, t-w+1) .. t} softmax_s(scale * q_t . k_s) v_s.
 * The pages give no formula; this is the plainest reading (the softmax over the window of scaled
 * dot products, scale = 1/sqrt(d) by default).  As for the linear mixer, every loop comes with its
 * own q, k, v: the T loops of one call are independent.
 */
typedef struct lt2_swa_dims {
    int64_t T;         /* loops                                                            */
    int64_t B;         /* batch                                                            */
    int64_t H;         /* heads                                                            */
    int64_t L;         /* tokens per sequence                                              */
    int64_t d;         /* head width (q, k and v): 1..256                                  */
    int64_t window;    /* w >= 1 (w >= L is causal softmax attention)                      */
    float scale;       /* multiplies q . k; 0 selects 1/sqrt(d)                            */
    int32_t dtype;     /* lt2_dtype of q, k and v                                          */
    int32_t algo;      /* lt2_algo: TENSOR_CORE = tcgen05/TMA kernel (bf16, d = 128 only),
                          CUDA_CORE = fp32 arithmetic, one warp per query; AUTO picks the
                          tensor-core kernel when it supports the shape                    */
    int32_t out_dtype; /* lt2_out_dtype of o                                               */
} lt2_swa_dims;

/*
 * Sliding-window prefill over all L tokens of every unit, all T loops in one call.
 *   q, k, v    [T][B][H][L][d], dims->dtype, contiguous (device, read only)
 *   o          [T][B][H][L][d], dims->out_dtype (device, written; must not alias an input)
 *   stream     cudaStream_t of the current device
 * Nothing is allocated; no workspace.  Returns LT2_OK once the launch is enqueued;
 * LT2_ERR_INVALID_ARGUMENT (a NULL or misaligned pointer, a size out of range, window < 1, a
 * negative or non-finite scale, o overlapping an input) or LT2_ERR_UNSUPPORTED (a forced
 * algorithm that does not take the shape, or the device pointers not on the current device)
 * before any launch; LT2_ERR_CUDA if the launch failed.  A bounded wait that gave up is reported
 * by lt2_gdr_last_device_error().
 */
lt2_status lt2_swa_prefill(const lt2_swa_dims* dims,
                           const void* q, const void* k, const void* v,
                           void* o, void* stream);

/*
 * The device-side status word of the CURRENT device (not an operation of the pages: the
 * library's own failure reporting).  Synchronises the device (every stream), then reads and
 * clears the word in one atomic exchange.  Returns LT2_ERR_DEVICE_TIMEOUT if a kernel gave up
 * on a bounded wait since the last read, else LT2_ERR_SEQLENS if a packed-sequence call met bad
 * offsets, else LT2_ERR_RANGE if a tensor-core prefill produced non-finite results, else
 * LT2_ERR_DEVICE_CHECK if a device-side check of the debug build failed (never in the product
 * build), else LT2_OK; LT2_ERR_CUDA if the synchronisation or the read failed.
 * The word is shared by every call on the device, from any thread or stream: a flag belongs
 * to whichever work ran since the previous read.
 */
lt2_status lt2_gdr_last_device_error(void);

/* Static, human-readable name of a status code (library bookkeeping, no counterpart on the
 * pages; never NULL). */
const char* lt2_status_string(lt2_status status);

/* Text of the last CUDA error seen by this library on the calling thread ("" if none;
 * library bookkeeping, no counterpart on the pages). */
const char* lt2_last_cuda_error_string(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH (library bookkeeping). */
int lt2_gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LT2_GDR_H */
