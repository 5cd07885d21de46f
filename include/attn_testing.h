/*
 * attn_testing.h - test hooks of libattn.so.  Not part of the product interface:
 * nothing in normal use calls them, and with their defaults (zero) the library
 * behaves exactly as attn.h describes.
 *
 * They exist so that the failure path of the bounded waits can be made to run on a
 * GPU without faulting it: every wait inside a kernel gives up after a time limit
 * (1 s by default), records where it gave up in the device status word, and lets
 * the kernel end with its copies drained and its tensor memory freed; the host then
 * reads ATTN_ERR_TIMEOUT from attn_check_status.  A test shortens the limit and
 * withholds one bulk copy (the copy is never issued, so nothing lands late), so that
 * one wait runs out.
 */
#ifndef ATTN_TESTING_H_
#define ATTN_TESTING_H_

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The tensor-core forward kernel's producer (CTA 0, its first work item) skips the
 * copy of its first V tile and that copy's transaction count, so the MMA issuer's
 * wait for that tile can only end by timing out. */
#define ATTN_TEST_DROP_FIRST_V 0x1u

/*
 * attn_testing_set - set the current device's wait limit and test flags for the
 * launches that follow (process-wide for that device, until set again).
 * wait_limit_ns: limit of every bounded wait in nanoseconds; 0 restores the default
 * of 1 s.  flags: 0 or ATTN_TEST_DROP_FIRST_V; any other bit is ATTN_ERR_INVALID_ARG.
 * Synchronous (a small host-to-device copy).  Call it with no kernel of this library
 * running on the device, and call attn_testing_set(0, 0) when done.
 */
attn_status_t attn_testing_set(unsigned long long wait_limit_ns, unsigned int flags);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_TESTING_H_ */
