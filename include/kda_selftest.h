/*
 * kda_selftest.h — self-test of the KDA library's failure detection (C ABI, see kda.h).
 *
 * Every wait inside the library's kernels (the mbarrier phases of the bulk-copy and tensor-core
 * pipelines) is bounded in time: when a phase does not complete within its limit, the waiting
 * thread sets the timeout bit of the per-device status word and its kernel leaves through its
 * normal exit path; kda_last_device_error() then returns KDA_ERR_TIMEOUT and the CUDA context
 * stays usable. The entry point below runs that give-up path on purpose, without faulting or
 * hanging the GPU: nothing in it can wait longer than its limit.
 */
#ifndef KDA_SELFTEST_H_
#define KDA_SELFTEST_H_

#include "kda.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * kda_selftest_wait_timeout — launch one block on `stream` whose first thread initialises an
 * mbarrier that nothing arrives on and waits for its first phase with the library's bounded
 * wait, giving up after `limit_ns` nanoseconds (1 <= limit_ns <= 1,000,000,000); the give-up
 * sets the timeout bit of the status word and the block exits.
 * Returns KDA_ERR_INVALID_ARG (on the host, nothing launched) for a limit outside that range,
 * KDA_ERR_CUDA when the launch fails, else KDA_OK; the timeout itself is read afterwards with
 * kda_last_device_error(stream).
 */
KDA_API kda_status_t kda_selftest_wait_timeout(uint64_t limit_ns, kda_stream_t stream);

/*
 * kda_selftest_bounds — in the bounds-checked build of the library (compiled with
 * KDA_BOUNDS_CHECK; see _build.build(checked=True)), registers `buffer` (device, `bytes` long) as
 * the only extent of the call and launches one thread that tests, with the kernels' own check and
 * without performing it, a 4-byte access starting just past the buffer's end. The check refuses
 * it and sets the bounds bit of the status word, which kda_last_device_error(stream) then reports
 * as KDA_ERR_INVALID_ARG. Nothing is read or written outside the buffer.
 * Returns KDA_ERR_UNSUPPORTED in the normal build (no checks compiled in), KDA_ERR_INVALID_ARG for
 * a null buffer or zero bytes, KDA_ERR_CUDA when a CUDA call fails, else KDA_OK.
 */
KDA_API kda_status_t kda_selftest_bounds(const void* buffer, size_t bytes, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_SELFTEST_H_ */
