/*
 * Pipeline trace of the paired tensor-core attention kernel -- present only in
 * the tracing build of the library (libinfini_attn_trace.so, compiled with
 * INFINI_TRACE defined: python -m compressive_memory_segment_b200.build --trace).
 * The regular library has none of these symbols and records nothing.
 *
 * In the tracing build, CTA 0 of every tc_attn_pair_kernel launch appends
 * records to 8 channels (0 K-ring TMA producer, 1/2 MMA issuer of slot 0/1,
 * 3/4 softmax warp 0/4 of slot 0/1, 5/6 retrieval warp 8 for slot 0/1, 7 V-ring
 * and Q TMA producer). A record is a 64-bit word: the SM clock (clock64, low
 * 40 bits) | event code << 40 | index << 48. Event codes and what they mark
 * are listed in compressive_memory_segment_b200/trace_timeline.py. Each
 * channel has one writer thread, which keeps its count in a register: a
 * record costs a clock read and one global store on CTA 0.
 */
#ifndef INFINI_ATTN_TRACE_H
#define INFINI_ATTN_TRACE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define INFINI_TRACE_API __attribute__((visibility("default")))
#define INFINI_TRACE_CHANNELS 8

/* Clears every channel (host call; synchronises the device). Returns 0, or
 * INFINI_ERR_CUDA. */
INFINI_TRACE_API int infini_attn_trace_reset(void);

/* Copies up to `cap` records of `channel` (0 .. INFINI_TRACE_CHANNELS-1) into
 * the host array `host` (synchronises the device). Returns the number of
 * records the channel holds (which may exceed cap; the device keeps at most
 * 32768 per channel), or a negative error code: INFINI_ERR_SHAPE for a bad
 * channel or cap < 0, INFINI_ERR_NULL for host == NULL with cap > 0,
 * INFINI_ERR_CUDA if a copy fails. */
INFINI_TRACE_API int infini_attn_trace_read(int channel, uint64_t* host, int cap);

#ifdef __cplusplus
}
#endif

#endif
