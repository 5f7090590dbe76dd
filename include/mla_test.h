/*
 * mla_test.h - test hooks of libmla.so.  These are not part of the decode
 * API described in mla.h and have no counterpart in the pages; they exist so
 * that tests can drive the library's failure handling without faulting or
 * hanging a GPU.
 */
#ifndef MLA_TEST_H_
#define MLA_TEST_H_

#include "mla.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * mla_test_set_decode_wait (host function; affects later launches)
 * Every barrier wait inside the tensor-core decode kernel gives up after
 * `limit_cycles` SM clock cycles; the kernel then sets MLA_DEVERR_TIMEOUT in
 * err_word, lets the copies it already issued land, frees its tensor memory
 * and returns.  limit_cycles = 0 restores the default (4e9 cycles, about 2 s).
 * withhold_q_load != 0 makes the leader CTA of every CTA pair leave the query
 * load of its first unit out, so that the MMA issuer's wait for it runs out:
 * the launch then aborts by the path above.  Results of such a launch are
 * invalid.  The settings are process-wide and not synchronised with launches
 * in flight: change them only between synchronised calls.  Returns MLA_OK.
 */
mla_status mla_test_set_decode_wait(unsigned long long limit_cycles, int withhold_q_load);

#ifdef __cplusplus
}
#endif

#endif /* MLA_TEST_H_ */
