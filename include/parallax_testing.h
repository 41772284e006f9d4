/*
 * parallax_testing.h - testing hook of libparallax.so.
 *
 * Not part of the decode API, and with no counterpart in the pages: it exists
 * so that tests can watch the kernels' bounded waits give up on a GPU without
 * hanging or faulting it.
 */
#ifndef PARALLAX_TESTING_H
#define PARALLAX_TESTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * parallax_decode (same arguments and checks) with two changes: every wait
 * inside the split-KV kernel is bounded by timeout_ms (1 .. 10000) instead of
 * the default 2 s, and the producer never fills the first pipeline stage of
 * each CTA, so the consumers' wait on it must run out. The kernels then set
 * PARALLAX_DEVICE_STATUS_TIMEOUT in the workspace status word and return; the
 * output is invalid; the CUDA context stays usable. Returns
 * PARALLAX_ERR_BAD_SHAPE for a timeout outside the range.
 */
int parallax_testing_decode_stalled(const void* q, const void* r, const void* k_cache,
                                    const void* v_cache, const int32_t* cache_seqlens,
                                    void* out, int B, int Hq, int Hkv, int D, float scale,
                                    void* stream, int Lmax, int num_splits, void* workspace,
                                    size_t workspace_bytes, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* PARALLAX_TESTING_H */
