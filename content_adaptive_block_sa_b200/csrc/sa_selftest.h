/*
 * sa_selftest.h - test-only export of libsa.so (not part of the public C ABI
 * in include/sa.h).
 *
 * sa_selftest_wait_timeout runs the device failure path with no fault: n_ctas
 * (1..1024) CTAs each wait on an mbarrier that nothing completes, through the
 * same bounded wait every kernel of the library uses, 4 s wall-time limit
 * included. The first to give up records SA_ERR_TIMEOUT and the location code
 * 900 in the workspace's status word (read it with sa_get_device_status after
 * the stream synchronises, about 4 s later); the rest leave on seeing the
 * word. Returns SA_OK once launched; SA_ERR_INVALID_ARG or SA_ERR_WORKSPACE
 * (ws shorter than 256 bytes) before any launch.
 */
#ifndef SA_SELFTEST_H_
#define SA_SELFTEST_H_

#include "sa.h"

#ifdef __cplusplus
extern "C" {
#endif

sa_status sa_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t n_ctas,
                                   sa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SA_SELFTEST_H_ */
