/*
 * frt_debug.h -- the bounds-checked build of the library (libfrt_debug.so).
 *
 * libfrt_debug.so is the same library as libfrt.so, with every entry point of
 * frt.h and the same results for valid calls, compiled with FRT_DEBUG_BOUNDS:
 * before each global-memory access a kernel checks the element index it is
 * about to use against the extent that the call's own sizes give that buffer
 * (for example M * D elements of x, capacity * Hkv * hd of a KV cache).  An
 * index outside the extent skips the access and adds one to a device-wide
 * violation counter.  A stand-in for an address sanitizer when none can run:
 * tests run the ops through this library and require a count of zero.  It is
 * slower than libfrt.so and is never the default.
 */
#ifndef FRT_DEBUG_H_
#define FRT_DEBUG_H_

#include "frt.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Waits for the device to finish all work (cudaDeviceSynchronize), writes the
 * number of out-of-range accesses skipped since the previous call to *count,
 * and resets the counter to zero.  Host pointer count must not be NULL
 * (FRT_ERR_INVALID_ARG); FRT_ERR_CUDA if the synchronisation or the copies
 * fail.  Only libfrt_debug.so exports it.
 */
frt_status frt_debug_bounds_violations(unsigned int* count);

#ifdef __cplusplus
}
#endif

#endif /* FRT_DEBUG_H_ */
