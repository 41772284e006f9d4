/*
 * parallax_testing.h - testing hook of libparallax.so.
 *
 * Not part of the API, and with no counterpart in the pages: these hooks
 * exist so that tests can watch the kernels' bounded waits give up on a GPU
 * without hanging or faulting it.
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

/*
 * parallax_prefill (same arguments and checks) with the same two changes for
 * the tcgen05 forward: every wait bounded by timeout_ms (1 .. 10000), and the
 * TMA producer never loads the first K tile of each CTA, so the UMMA issuer's
 * wait on it runs out. Each CTA then records PARALLAX_DEVICE_STATUS_TIMEOUT,
 * waits (bounded) for its own copies in flight, frees its tensor memory and
 * returns; the output is invalid; the CUDA context stays usable.
 */
int parallax_testing_prefill_stalled(const void* q, const void* r, const void* k, const void* v,
                                     void* out, int B, int Hq, int Hkv, int L, int D,
                                     float scale, int causal, void* stream, int out_dtype,
                                     void* workspace, size_t workspace_bytes, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* PARALLAX_TESTING_H */
