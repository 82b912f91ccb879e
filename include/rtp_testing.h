/*
 * rtp_testing.h - test hooks of librtp.so. Not part of the library's public
 * interface (include/rtp.h): these entry points exist so that the test suite
 * can drive failure paths that ordinary inputs never reach, without faulting
 * or hanging the GPU.
 */
#ifndef RTP_TESTING_H_
#define RTP_TESTING_H_

#include "rtp.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * rtp_debug_prefill_timeout_probe - exercises the bounded waits of the
 * tensor-core prefill attention kernel.
 *   Launches one thread block of that kernel on a 128-token, one-head
 *   sliding-window problem whose producer deliberately never loads Q, so the
 *   block's waits run out (after about 2 s of SM clock); it drains the copies
 *   it issued, frees its tensor memory and records RTP_ERR_TIMEOUT in the
 *   status word of `ws` (read it with rtp_get_device_status). The device and
 *   the context stay usable afterwards.
 *   q, k, v, o  bf16 [1, 128, 1, 128] device buffers (o is not written).
 *   ws          at least 256 bytes, 256-byte aligned.
 */
RTP_API rtp_status rtp_debug_prefill_timeout_probe(const void* q, const void* k, const void* v, void* o, void* ws,
                                                   size_t ws_bytes, rtp_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* RTP_TESTING_H_ */
