/*
 * Profiling entry points of libattn25_trace.so, the build of attn25 compiled
 * with -DATTN25_TRACE.  Its kernels time selected barrier waits and phases
 * per warp role with clock64 and add them into a device counter buffer
 * (256 x uint64: forward roles at 0..63, backward roles at 128..255, 16 per
 * role; word 255 holds the first step of the event window).  After the
 * counters, 512 words hold the clock64 of 16 events in each of 32
 * consecutive backward steps of CTA 0.  The normal library (libattn25.so)
 * does not export these.
 */
#ifndef ATTN25_TRACE_H
#define ATTN25_TRACE_H

#include "attn25.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Synchronise the device, then copy the first n (<= 768) words to host memory. */
ATTN25_API int attn_trace_read(unsigned long long* host_out, int n);

/* Synchronise the device, then zero all counters. */
ATTN25_API int attn_trace_reset(void);

/* Set the first backward step of the event window (after attn_trace_reset). */
ATTN25_API int attn_trace_window(int first_step);

#ifdef __cplusplus
}
#endif

#endif /* ATTN25_TRACE_H */
