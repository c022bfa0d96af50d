/*
 * dynconv_diag.h -- diagnostics of libdynconv.so (no counterpart in the pages:
 * these check the library's own sm_100a building blocks, not the method).
 */
#ifndef DYNCONV_DIAG_H
#define DYNCONV_DIAG_H

#include "dynconv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One 128-row tile of D = A * B^T (bf16 in, fp32 out) through TMA loads with
 * 128-byte swizzle and one CTA's tcgen05.mma, using the descriptor helpers of
 * the product kernels.
 *   variant 0: A is [128, Kd] and B is [N, Kd], row-major (both K-major);
 *              Kd in {64, 128, 192}.
 *   variant 1: A is stored [Kd, 128] and B is stored [Kd, N] (both MN-major);
 *              Kd a multiple of 16 up to 128.
 *   variant 2: A is [128, 64] (K-major) and B is stored [64, N] (MN-major);
 *              Kd = 64.
 *   variants 3, 4: A is [136, 64] and B is [N, 64] (both K-major); the A
 *              operand starts Kd rows (1..7) into the 136-row tile, so
 *              D = A[Kd:Kd+128] B^T.  Variant 3 leaves the descriptor's
 *              base-offset field 0, variant 4 sets it from the start address.
 *   N: multiple of 16, 16..256.  D: [128, N] fp32, row-major.
 * All pointers are device pointers (16-byte aligned); err_word is a device
 * uint32 that receives the wait-timeout bit if the tile never completes.
 * Asynchronous on `stream`; returns DYNCONV_ERR_INVALID for other shapes. */
DYNCONV_API dynconv_status dynconv_selftest_umma(int variant, const void *A, const void *B, float *D, int N, int Kd,
                                                 void *err_word, void *stream);

/* A bounded wait that runs out, on purpose and safely: one CTA waits on an
 * mbarrier that nothing completes, one thread with a limit of limit_ns
 * nanoseconds (1 .. 2e9) and a thread of another warp with the kernels' own
 * limit, which must give up as soon as the first has (the CTA's abort flag).
 * Both waits end; out2 (a device uint32[2]) receives 2, 2 (1 would mean a wait
 * returned success), and err_word (a device uint32) receives the wait-timeout
 * bit that dynconv_device_status reports as DYNCONV_ERR_DEVICE_CHECK.  The CUDA
 * context stays usable.  Asynchronous on `stream`; DYNCONV_ERR_INVALID for null
 * pointers or a limit outside 1 .. 2e9. */
DYNCONV_API dynconv_status dynconv_selftest_wait(uint64_t limit_ns, void *err_word, void *out2, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DYNCONV_DIAG_H */
