/*
 * kvc_testing.h - test hooks of libkvc.so.  Not part of the codec; the pages
 * have no counterpart.  They exist so that tests can exercise the library's
 * error paths on a real GPU without faulting or hanging it.
 */
#ifndef KVC_TESTING_H
#define KVC_TESTING_H

#include "kvc.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Arms a one-shot fault for the next tensor-core cross-layer codec launch
 * (kvc_encode_layer / kvc_decode_layer with KVC_PRED_XLAYER_DPLR, bf16,
 * head_dim 128).  what = 1: in that launch, the TMA producer of CTA 0 leaves
 * its first pipeline stage unarmed and unloaded, so the consumer's wait on that
 * stage runs out after the kernel's bounded wait time (about 2^32 SM cycles,
 * roughly two seconds); the kernel then raises its abort flag, every role
 * returns, the loads already issued are drained, and
 * kvc_get_device_error() reports KVC_ERR_DEVICE_TIMEOUT.  The codes written by
 * that launch are meaningless.  what = 0 disarms.  Process-wide; the launch
 * that consumes the fault clears it. */
KVC_API void kvc_testing_inject_stall(int what);

#ifdef __cplusplus
}
#endif

#endif /* KVC_TESTING_H */
