/*
 * kmip_testing.h -- test hooks of libkmip (not needed by ordinary callers).
 */
#ifndef KMIP_TESTING_H
#define KMIP_TESTING_H

#include "kmip.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Runs, on `stream`, one CTA that waits on a shared-memory mbarrier nobody
 * arrives at, through the same bounded wait every pipeline wait of the
 * tensor-core forward uses, with a limit of `timeout_us` microseconds
 * (1 .. 1,000,000).  The wait runs out, the kernel records KMIP_ERR_TIMEOUT
 * in the device status word and returns; kmip_get_status() then reports it.
 * Exists so tests can check the timeout path without hanging a GPU.
 * Returns KMIP_OK once enqueued, KMIP_ERR_INVALID_ARG for a bad limit.
 */
kmip_status_t kmip_test_wait_timeout(kmip_stream_t stream, int timeout_us);

#ifdef __cplusplus
}
#endif

#endif /* KMIP_TESTING_H */
