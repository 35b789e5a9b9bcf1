/*
 * msa_testing.h -- test hooks of libmsa.so.  Not part of the MSA method (the
 * pages have no counterpart); they exist so tests can check the library's
 * failure handling on a GPU without faulting or hanging it.
 */
#ifndef MSA_TESTING_H_
#define MSA_TESTING_H_

#include "msa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Launches one kernel whose thread waits on an mbarrier that nothing ever
 * signals, bounded by deadline_ns (1 ns .. 2 s).  The wait gives up, records
 * a timeout in the status word at the start of `ws` (a device buffer of at
 * least 256 bytes, cleared first) and the kernel exits normally; afterwards
 * msa_device_status(ws, stream) returns MSA_ERR_TIMEOUT and the CUDA context
 * remains usable.
 */
MSA_API int msa_test_never_ready_wait(void* ws, size_t ws_bytes, long long deadline_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_TESTING_H_ */
