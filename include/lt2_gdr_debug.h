/*
 * lt2_gdr_debug.h -- extra entry points of the DEBUG build of the library,
 * liblt2gdr_debug.so (the same sources compiled with LT2_DEBUG).  They are test hooks for the
 * library's own failure handling and have no counterpart on the pages; the product library,
 * liblt2gdr.so, does not export them.
 *
 * What the debug build changes:
 *   - every bounded wait inside the tensor-core kernels gives up after
 *     lt2_debug_wait_timeout_ns() (milliseconds) instead of 4 s;
 *   - device-side invariants are checked: TMA coordinates inside the tensors, the shared-memory
 *     tiles a warp converts or writes inside the CTA's allocation, the TMEM columns inside the
 *     CTA's allocation.  A failed check is recorded for lt2_gdr_last_device_error() as
 *     LT2_ERR_DEVICE_CHECK and the access is skipped; nothing traps;
 *   - lt2_debug_set_skip_chunk() can make the TMA producer of a tensor-core prefill stop before a
 *     chosen chunk.  The copies of that chunk are then never issued, the waits for them run out,
 *     and the kernel takes its abort path: it records LT2_ERR_DEVICE_TIMEOUT, waits (bounded) for
 *     its own copies and MMAs in flight, frees its tensor memory and returns.
 * Everything else (arguments, layouts, results) is as in lt2_gdr.h.
 */
#ifndef LT2_GDR_DEBUG_H
#define LT2_GDR_DEBUG_H

#include "lt2_gdr.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Which kernel a fault injection applies to. */
typedef enum lt2_debug_kernel {
    LT2_DEBUG_SCALAR_TC = 0,   /* tensor-core prefill, scalar gating  */
    LT2_DEBUG_PER_KEY_TC = 1   /* tensor-core prefill, per-key gating */
} lt2_debug_kernel;

/*
 * From now on, every launch of `kernel` on the CURRENT device stops loading before chunk
 * `chunk` (0-based, per head-unit); chunk = -1 turns the injection off.  Synchronous (a small
 * host-to-device copy).  Returns LT2_ERR_INVALID_ARGUMENT for an unknown kernel or chunk < -1,
 * LT2_ERR_CUDA if the copy failed.
 */
lt2_status lt2_debug_set_skip_chunk(int kernel, int chunk);

/* The bound of every in-kernel wait of this build, in nanoseconds. */
uint64_t lt2_debug_wait_timeout_ns(void);

#ifdef __cplusplus
}
#endif

#endif /* LT2_GDR_DEBUG_H */
