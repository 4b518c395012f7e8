/*
 * fa_testing.h -- test hooks of the B200 attention library.  Not needed to
 * compute attention; they let tests drive internal paths (a bounded wait
 * that runs out) without faulting the GPU.
 */
#ifndef FA_B200_FA_TESTING_H
#define FA_B200_FA_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fa_test_skip_one_arrival -- the next bf16 forward launch in this process
 * (through fa_fwd or fa_fwd_noalloc) runs with one arrival missing: CTA 0
 * never loads its first Q tile, so the MMA warp's bounded wait on that tile
 * runs out (about two seconds).  The
 * kernel then records FA_ERR_DEVICE_TIMEOUT in the status word of the entry
 * point that launched it,
 * drains its copies and MMAs, frees its tensor memory and exits; the context
 * stays usable.  Exercises the failure-detection path of the bounded waits
 * (the pages have no counterpart).  Always returns FA_OK.
 */
int fa_test_skip_one_arrival(void);

/*
 * fa_test_force_forward_kernel -- which bf16 forward kernel fa_fwd and
 * fa_fwd_host launch from now on in this process: 0 (the default) the one
 * fa_fwd_kernel_choice names for the shape, 1 always the two-tile kernel,
 * 2 always the one-tile kernel.  Both compute the same result; the
 * hook lets tests check each on every shape; it applies to fa_fwd_noalloc
 * too.  Returns FA_OK, or FA_ERR_INVALID_ARGUMENT for any other value.
 */
int fa_test_force_forward_kernel(int which);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_TESTING_H */
