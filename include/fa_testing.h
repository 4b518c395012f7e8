/*
 * fa_testing.h -- test hooks of the B200 attention library.  Not needed to
 * compute attention; they expose internal device routines so tests can check
 * them in isolation.
 */
#ifndef FA_B200_FA_TESTING_H
#define FA_B200_FA_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fa_test_exp2_poly -- y[i] = 2^x[i] computed by the polynomial routine the
 * bf16 kernel uses for part of its softmax exponentials (range reduction to
 * [-1/2, 1/2], a cubic fitted for minimax relative error, exponent add; the
 * method belongs to the online-softmax step, FlashAttention, Playable, EP 04,
 * whose exponentials it computes).  x and y are device pointers to n >= 0
 * floats (n even not required), 4-byte aligned, non-overlapping.  Valid for
 * x <= 127; inputs below -125 return 2^-125 (a negligible stand-in for 0 next
 * to a softmax denominator of at least 1).  Asynchronous on `stream`.
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (null pointer with n > 0, n < 0) or
 * FA_ERR_CUDA.
 */
int fa_test_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/*
 * fa_test_skip_one_arrival -- the next bf16 forward launch in this process
 * (through fa_fwd or fa_fwd_noalloc) runs with one arrival missing: CTA 0 never loads its first Q tile, so the
 * MMA warp's bounded wait on that tile runs out (about two seconds).  The
 * kernel then records FA_ERR_DEVICE_TIMEOUT in the status word of the entry
 * point that launched it,
 * drains its copies and MMAs, frees its tensor memory and exits; the context
 * stays usable.  Exercises the failure-detection path of the bounded waits
 * (the pages have no counterpart).  Always returns FA_OK.
 */
int fa_test_skip_one_arrival(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_TESTING_H */
