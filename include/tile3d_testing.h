/*
 * tile3d_testing.h — test hooks of libtile3d.so (not part of the computation's interface).
 *
 * These calls exist so that a test can drive a kernel's error handling without a GPU fault: they
 * change library-wide settings and are meant for test programs only. They are not thread-safe
 * with respect to concurrent calls of the library.
 */
#ifndef TILE3D_TESTING_H_
#define TILE3D_TESTING_H_

#include "tile3d.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * t3d_testing_set_wait_cycles — limit of every pipeline wait of block_sparse_attn_fwd.
 * The paper has no counterpart: this is a hook for testing the kernel's bounded waits.
 *   cycles: clock cycles a pipeline wait may take before the kernel gives up, records
 *           T3D_DEV_TIMEOUT in the caller's status word, lets its copies and MMAs in flight
 *           complete (those waits keep the default limit of ~2 s), frees its tensor memory and
 *           returns; 0 restores the default (4e9 cycles, ~2 s). A limit of a few cycles makes the
 *           first wait that is not already satisfied give up, so the output is then undefined.
 *           Applies to launches made after the call. Negative: T3D_ERR_INVALID.
 */
t3d_status t3d_testing_set_wait_cycles(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* TILE3D_TESTING_H_ */
