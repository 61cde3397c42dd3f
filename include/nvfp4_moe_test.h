/*
 * Test hooks of the NVFP4 MoE layer library (libnvfp4_moe.so).
 *
 * The pages have no counterpart: these exist only so that the library's own
 * fault tests can drive its error paths without faulting, trapping or hanging
 * a GPU. Production code never calls them; with the hooks off (the default)
 * the library behaves exactly as nvfp4_moe.h describes.
 */
#ifndef NVFP4_MOE_TEST_H
#define NVFP4_MOE_TEST_H

#include "nvfp4_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Decode (T <= 8): CTA 0 never arrives at the grid barrier between the gate/up
 * and down phases, so every CTA's bounded wait there runs out (after about
 * 200 ms), the call latches NVFP4_MOE_ERR_TIMEOUT and leaves out unwritten.
 * nvfp4_moe_get_status then returns TIMEOUT and clears the decode state, after
 * which calls with the flag off are correct again. */
#define NVFP4_MOE_TEST_DECODE_STALL 1

/* Grouped-GEMM path (T > 8): every used expert takes the tensor-core tiles,
 * none the small-expert streaming kernels (experts with at most 16 pairs), so
 * that tests can check both paths on the same inputs. The result agrees with
 * the default within the documented tolerance, not bit for bit (the two sum K
 * in a different order). */
#define NVFP4_MOE_TEST_NO_SMALL 2

/* Sets the test flags of a handle (0 = none). Returns NVFP4_MOE_OK, or
 * NVFP4_MOE_ERR_INVALID_ARG for a NULL handle or an unknown flag. */
NVFP4_MOE_API int nvfp4_moe_test_set_flags(nvfp4_moe_t *h, int32_t flags);

/* The detail word that came with the status the last nvfp4_moe_get_status on h
 * returned (0 when it returned 0). For NVFP4_MOE_ERR_NONFINITE raised by a
 * computed value: (1 << 20) | expert for h, (2 << 20) | expert for a per-pair
 * down row, (3 << 20) | (token or row) for the output; a token index for a
 * routing logit. For NVFP4_MOE_ERR_TIMEOUT: where the wait gave up. Returns 0 for
 * a NULL handle. */
NVFP4_MOE_API int nvfp4_moe_test_last_detail(const nvfp4_moe_t *h);

/* Makes the n-th device allocation (counting from 1) made by later
 * nvfp4_moe_create calls fail as if the device were out of memory; the hook
 * then disarms itself. n <= 0 disarms it. create must then return
 * NVFP4_MOE_ERR_CUDA with nothing left allocated. Process-wide; not
 * thread-safe. */
NVFP4_MOE_API void nvfp4_moe_test_fail_alloc(int32_t n);

#ifdef __cplusplus
}
#endif
#endif
