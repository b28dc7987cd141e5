/*
 * nvfp4_testing.h -- test hooks of libnvfp4.so.  Not part of the stable ABI;
 * the test suite uses them to exercise the GEMM's bounded-wait failure path
 * without faulting or hanging a GPU.
 */
#ifndef NVFP4_TESTING_H
#define NVFP4_TESTING_H

#include <stdint.h>

#include "nvfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sets, for the following nvfp4_gemm calls in this process, the timeout of
 * every bounded wait inside the GEMM kernel (timeout_ns, counted from the
 * start of each wait, so it bounds a lack of progress, not the kernel's run
 * time; 0 restores the default of 4 s) and debug flags (bit 0: the producer never issues the
 * copies of the first pipeline stage, so the consumer's wait for it runs out
 * and the kernel reports NVFP4_ERR_TIMEOUT through the workspace status word
 * after draining its in-flight work).  Not thread-safe; tests only. */
NVFP4_API void nvfp4_testing_set_gemm_wait(uint64_t timeout_ns, int debug_flags);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_TESTING_H */
