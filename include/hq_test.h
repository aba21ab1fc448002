/*
 * hq_test.h -- test-only entry points of libhq (failure detection without a GPU fault).
 *
 * The encoder places each item (a block of 128 tile rows of one tile column) by a decoupled
 * look-back over the items before it; every wait in it is bounded.  This entry point makes one
 * item withhold its offset, so that the bounded wait of its successor runs out: the kernel then
 * records HQ_ERR_TIMEOUT in the workspace status word, finishes, and the CUDA context stays
 * usable.  It exists to test that path; the method has no counterpart.  These entry points are
 * built only into the test library libhq_test.so (sources compiled with HQ_TEST_HOOKS); the
 * product library libhq.so neither exports them nor carries the hook in its kernels.
 */
#ifndef HQ_TEST_H
#define HQ_TEST_H

#include "hq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * As hq_encode, except that item `silent_item` (>= 1; items are numbered tile column by tile
 * column, ceil(rows / 128) per column at n = 64 or 128, ceil(rows / 64) at n = 256) never
 * publishes its word offset.  Expect HQ_ERR_TIMEOUT from hq_status_read and a code that is not
 * usable; the call takes about as long as the look-back limit (about a second).  HQ_ERR_ARG for
 * silent_item < 1 and for everything hq_encode rejects; HQ_ERR_UNSUPPORTED for lattices other than
 * E8 (only the E8 kernels of the test library carry the hook).
 */
hq_status_t hq_test_encode_silent_item(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols,
                                       const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes,
                                       int64_t silent_item, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_TEST_H */
