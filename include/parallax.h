/*
 * parallax.h - C ABI of libparallax.so, the B200 (sm_100a) Parallax decode.
 *
 * Parallax (parameterized Local Linear Attention) keeps softmax attention's
 * readout and adds a learned covariance correction: each query head carries
 * its query q and a probe r produced by a learned projector, and the decode
 * output over the cached keys k_i and values v_i is
 *
 *     w_i = softmax_i(scale * q.k_i),   s_i = r.k_i,
 *     o   = vbar + sum_i w_i (s_i - sbar)(v_i - vbar)
 *         = A/l + C/l - (b/l)(A/l),
 *     l = sum e_i, A = sum e_i v_i, b = sum e_i s_i, C = sum e_i s_i v_i,
 *     e_i = exp(scale * q.k_i - m).
 *
 * Sources: "Parallax: Parameterized Local Linear Attention for Language
 * Modeling" (neuraltrendhub summary, "What the paper found" and "Original
 * abstract": the learned query-like projector that probes the KV covariance
 * in place of LLA's solve, one streaming pass over FlashAttention's K/V
 * tiles); same title (bayesiansapien blog, opening diagram and "TL;DR":
 * softmax is the local-constant estimate, LLA the local-linear one);
 * parallax-kernel 0.1.0 README, "Decoding (CuTeDSL)": the decode call takes
 * q, r (shaped like q), k, v and qk_scale; "Integrazioni AI personalizzate
 * dopo l'attenzione Parallax" (encorp.ai), FAQ: with the projection at zero
 * the layer is exactly softmax attention.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no device memory and keeps no per-call state; the workspace is
 *    caller-owned scratch (see parallax_decode_workspace_bytes).
 *  - Layouts are contiguous, row-major, innermost last:
 *        q, r, out      [B][Hq][D]            (the pages' (B, 1, H, D))
 *        k_cache,v_cache[B][Hkv][Lmax][D]     (max-length-padded cache;
 *                       parallax_decode_ex also takes [B][Lmax][Hkv][D],
 *                       the pages' (B, kv_len, H, D))
 *        cache_seqlens  [B] int32 in device memory, or NULL: every sequence
 *                       then holds all Lmax keys (the pages' call passes no
 *                       lengths)
 *    Query head h reads kv head h / (Hq/Hkv) (contiguous GQA groups). Keys
 *    0 .. cache_seqlens[b]-1 of sequence b are attended; padding positions
 *    are never read into any accumulator. Values outside [0, Lmax] are
 *    clamped on the device and reported through the workspace status word.
 *    A sequence with no keys gets a zero output.
 *  - in_dtype: PARALLAX_DTYPE_BF16 or PARALLAX_DTYPE_F32 (q, r, k, v alike).
 *    out_dtype: PARALLAX_DTYPE_BF16 (round-to-nearest-even from fp32) or
 *    PARALLAX_DTYPE_F32 (the fp32 debug output). Accumulation is fp32.
 *  - D must be 64 or 128. Hq must be a multiple of Hkv. All pointers must be
 *    16-byte aligned.
 *  - scale is the softmax scale applied to q.k only (qk_scale); the probe
 *    score s_i = r.k_i is not scaled.
 *  - stream is a cudaStream_t (NULL = legacy default stream). Calls are
 *    stream-ordered and asynchronous: no host synchronisation, no allocation,
 *    so they can be captured in a CUDA graph.
 *  - num_splits: 0 picks the number of key-range partitions for the device
 *    and the kernel the call runs on (parallax_choose_splits); a positive
 *    value forces it (1 .. 65536).
 *    Results do not depend on it beyond fp32 rounding, and are bitwise
 *    reproducible for a fixed value and device.
 *  - Return value: PARALLAX_OK (0) or a negative status. Argument errors are
 *    detected on the host before anything is launched. Launch failures return
 *    PARALLAX_ERR_CUDA. Nothing is thrown across the ABI.
 */
#ifndef PARALLAX_H
#define PARALLAX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PARALLAX_OK 0
#define PARALLAX_ERR_NULL_POINTER (-1)
#define PARALLAX_ERR_BAD_SHAPE (-2)
#define PARALLAX_ERR_UNSUPPORTED_HEAD_DIM (-3)
#define PARALLAX_ERR_UNSUPPORTED_DTYPE (-4)
#define PARALLAX_ERR_MISALIGNED (-5)
#define PARALLAX_ERR_WORKSPACE_TOO_SMALL (-6)
#define PARALLAX_ERR_BAD_SPLITS (-7)
#define PARALLAX_ERR_CUDA (-8)
#define PARALLAX_ERR_DEVICE_TIMEOUT (-9)
#define PARALLAX_ERR_BAD_PHASE (-10)
#define PARALLAX_ERR_SEQLEN_CLAMPED (-11)

#define PARALLAX_DTYPE_BF16 0
#define PARALLAX_DTYPE_F32 1

#define PARALLAX_MAX_SPLITS 65536

/* Cache layouts for parallax_decode_ex. */
#define PARALLAX_KV_BHSD 0 /* [B][Hkv][Lmax][D] */
#define PARALLAX_KV_BSHD 1 /* [B][Lmax][Hkv][D] */

/* Bits of the device status word kept at the start of the workspace. */
#define PARALLAX_DEVICE_STATUS_TIMEOUT 1u
#define PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED 2u

/*
 * Number of key-range partitions (CTAs of the persistent split-KV kernel) the
 * library uses by default for the TMA kernel (bf16 caches, up to 4 query
 * heads per kv head with the probe, 8 without): the flattened (batch, kv
 * head, key) range is cut into this many equal parts of at least 128 keys,
 * at most one per SM, so every SM streams the same bytes whatever the batch
 * size and lengths. Calls on the generic kernel (fp32 inputs, larger groups)
 * take parts of at least 64 keys by default, still at most one per SM; the
 * workspace size for num_splits = 0 covers both. sm_count <= 0 queries the
 * current device. Returns >= 1, or a negative status for bad arguments. The
 * environment variable PARALLAX_SPLITS (a positive integer, read once per
 * process) replaces the heuristic, here and wherever num_splits is 0, for
 * experiments.
 */
int parallax_choose_splits(int B, int Hkv, int Lmax, int sm_count);

/*
 * The partition count a decode call with num_splits = 0 uses: the
 * parallax_choose_splits count on the TMA kernel's path, the generic
 * kernel's finer count otherwise (in_dtype PARALLAX_DTYPE_F32, or more than
 * 4 query heads per kv head with probe != 0, or more than 8 without).
 * sm_count <= 0 queries the current device. Returns >= 1, or a negative
 * status for bad arguments.
 */
int parallax_default_splits(int B, int Hq, int Hkv, int Lmax, int in_dtype, int probe,
                            int sm_count);

/*
 * Bytes of workspace one decode call needs: a 256-byte header (the device
 * status word) plus two fp32 partial records (m, l, b, A[D], C[D]) per
 * partition and query head of a group. num_splits as in parallax_decode (0 =
 * the default for the current device). Returns 0 for invalid arguments.
 * The workspace must be zero-filled once after allocation (the status word);
 * the partial records need no initialisation.
 */
size_t parallax_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int Lmax,
                                       int num_splits);

/*
 * The Parallax decode forward: out = vbar + C/l - (b/l) vbar per query head
 * (see the top of this file). r holds the probe rows, one per query head,
 * shaped like q. Launches, on `stream`, either one cluster kernel (few
 * (batch row, kv head) items) or the split-KV kernel and the split-merge
 * kernel; parallax_decode_plan says which.
 */
int parallax_decode(const void* q, const void* r, const void* k_cache,
                    const void* v_cache, const int32_t* cache_seqlens, void* out,
                    int B, int Hq, int Hkv, int D, float scale, void* stream,
                    int Lmax, int in_dtype, int out_dtype, int num_splits,
                    void* workspace, size_t workspace_bytes);

/*
 * The R = 0 comparator: plain softmax attention decode (out = A/l), the
 * FlashAttention-style kernel Parallax reduces to when the probe projection
 * is zero. Same pipeline and arguments as parallax_decode, without r.
 */
int parallax_softmax_decode(const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* cache_seqlens,
                            void* out, int B, int Hq, int Hkv, int D, float scale,
                            void* stream, int Lmax, int in_dtype, int out_dtype,
                            int num_splits, void* workspace,
                            size_t workspace_bytes);

/*
 * The general form of parallax_decode and parallax_softmax_decode.
 *  - probe: 1 for the Parallax decode, 0 for the R = 0 softmax decode (r may
 *    then be NULL).
 *  - kv_layout: PARALLAX_KV_BHSD ([B][Hkv][Lmax][D], as parallax_decode) or
 *    PARALLAX_KV_BSHD ([B][Lmax][Hkv][D], the cache layout of the
 *    parallax-kernel 0.1.0 README, "Quickstart / Decoding (CuTeDSL)").
 *  - window: 0 attends all cached keys; W > 0 attends only the last
 *    min(n, W) keys of each sequence of length n (sliding-window decode; the
 *    README's introduction calls sliding windows structurally compatible with
 *    Parallax). The workspace size is that of Lmax = min(Lmax, W).
 *  - phases: 3 runs both kernels; 1 or 2 runs only the split-KV or only the
 *    merge kernel (as parallax_decode_phase).
 * parallax_decode(...) is parallax_decode_ex(..., 1, PARALLAX_KV_BHSD, 0, 3).
 * Errors as parallax_decode; a bad kv_layout or a negative window gives
 * PARALLAX_ERR_BAD_SHAPE, a bad phases value PARALLAX_ERR_BAD_PHASE.
 */
int parallax_decode_ex(const void* q, const void* r, const void* k_cache,
                       const void* v_cache, const int32_t* cache_seqlens, void* out,
                       int B, int Hq, int Hkv, int D, float scale, void* stream,
                       int Lmax, int in_dtype, int out_dtype, int num_splits,
                       void* workspace, size_t workspace_bytes, int probe,
                       int kv_layout, int window, int phases);

/*
 * One phase of a decode call, for per-kernel timing and for tests of the
 * partial records: phase 1 runs only the split-KV kernel (writes `out` for
 * sequences covered by one partition and partial records for the others),
 * phase 2 only the split-merge kernel. Calling phase 1 then phase 2 with the
 * same arguments is equivalent to one call of parallax_decode (probe = 1) or
 * parallax_softmax_decode (probe = 0; r may be NULL). Returns
 * PARALLAX_ERR_BAD_PHASE for any other phase.
 */
int parallax_decode_phase(int phase, int probe, const void* q, const void* r,
                          const void* k_cache, const void* v_cache,
                          const int32_t* cache_seqlens, void* out, int B, int Hq,
                          int Hkv, int D, float scale, void* stream, int Lmax,
                          int in_dtype, int out_dtype, int num_splits,
                          void* workspace, size_t workspace_bytes);

/*
 * How a decode call with num_splits = 0 runs these shapes on the current
 * device (any key space: contiguous, windowed, paged or block-sparse rows).
 * Two schedules exist:
 *  - split-KV + merge: *grid_ctas partitions of the flattened key range (one
 *    CTA each), partial records in the workspace, then the merge kernel;
 *    *cluster_ctas = 0.
 *  - one thread-block cluster per (batch row, kv head) item, for few items
 *    (B * Hkv at most half the SM count) on the TMA kernel's inputs: the
 *    item's 64-key tiles are dealt round-robin to *cluster_ctas CTAs (2 to
 *    8, the most that leave every cluster resident at once), which combine
 *    their (m, l, b, A, C) through distributed shared memory; no merge
 *    kernel and no partial records; *grid_ctas = B * Hkv * *cluster_ctas.
 * The results of the two agree within the decode tolerances (the sums are
 * grouped differently); each is deterministic. An explicit num_splits > 0
 * always takes the first. Returns PARALLAX_OK or an argument error.
 */
int parallax_decode_plan(int B, int Hq, int Hkv, int D, int Lmax, int in_dtype, int out_dtype,
                         int probe, int* grid_ctas, int* cluster_ctas);

/*
 * Decode over a paged KV cache: the pages' decode (parallax-kernel 0.1.0
 * README, "Decoding (CuTeDSL)") with its (B, kv_len, H, D) cache cut into
 * fixed-size pages, the layout serving engines keep their caches in.
 *  - k_pages, v_pages [num_pages][page_size][Hkv][D] (a pool of pages), bf16
 *    or fp32 (in_dtype, which q and r share);
 *    block_table [B][max_pages_per_seq] int32: key i of sequence b is slot
 *    i % page_size of page block_table[b][i / page_size]. Entries past a
 *    sequence's length may be read (the cluster schedule fetches a row's
 *    first tiles before its length is known) but attend nothing, whatever
 *    they hold.
 *  - page_size a multiple of 64 (every 64-key tile lies in one page);
 *    max_pages_per_seq * page_size plays the role of Lmax (cache_seqlens are
 *    clamped to it; NULL lengths mean that many keys).
 *  - A page id outside [0, num_pages) is not read: its keys are left out and,
 *    for an entry the length reaches, PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED
 *    is set.
 *  - probe != 0: the Parallax output (r required); probe == 0: R = 0 softmax.
 *  - bf16 or fp32 inputs (in_dtype); any query-head group. bf16 pools with
 *    up to 4 query heads per kv head with the probe (8 without) run on the
 *    TMA kernel; fp32 pools and larger groups on the generic kernel, which
 *    resolves the pages the same way.
 *  - Workspace: parallax_decode_workspace_bytes(B, Hq, Hkv, D,
 *    max_pages_per_seq * page_size, num_splits). Other rules as parallax_decode.
 */
int parallax_decode_paged(const void* q, const void* r, const void* k_pages, const void* v_pages,
                          const int32_t* block_table, const int32_t* cache_seqlens, void* out,
                          int B, int Hq, int Hkv, int D, float scale, void* stream, int num_pages,
                          int page_size, int max_pages_per_seq, int probe, int in_dtype,
                          int out_dtype, int num_splits, void* workspace, size_t workspace_bytes);

/*
 * Block-sparse decode: parallax-kernel 0.1.0 README (opening section) notes
 * that block sparsity is structurally compatible with Parallax. Sequence b
 * attends only the listed 64-key blocks of its cache row: block_ids
 * [B][max_blocks] int32, the first num_blocks[b] entries used; block j holds
 * cache keys 64 j .. 64 j + 63, of which those below cache_seqlens[b] count.
 * The weights are the softmax over the selected keys only; the output is the
 * Parallax output over that key set (zero if it is empty).
 *  - Cache as parallax_decode_ex (kv_layout BHSD or BSHD, Lmax keys per row).
 *  - A block id outside [0, ceil(Lmax / 64)) or a count outside [0,
 *    max_blocks] is clamped away and sets PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED.
 *  - A block listed twice is attended twice (its keys count twice).
 *  - bf16 or fp32 inputs (in_dtype); any query-head group, as
 *    parallax_decode_paged.
 *  - Workspace: parallax_decode_workspace_bytes(B, Hq, Hkv, D, 64 * max_blocks,
 *    num_splits). Other rules as parallax_decode.
 */
int parallax_decode_block_sparse(const void* q, const void* r, const void* k_cache,
                                 const void* v_cache, const int32_t* cache_seqlens,
                                 const int32_t* block_ids, const int32_t* num_blocks, void* out,
                                 int B, int Hq, int Hkv, int D, float scale, void* stream, int Lmax,
                                 int kv_layout, int max_blocks, int probe, int in_dtype,
                                 int out_dtype, int num_splits, void* workspace,
                                 size_t workspace_bytes);

/*
 * The training-shape (prefill) forward: parallax-kernel 0.1.0 README,
 * "Training (Triton)": parallax_func(q, r, k, v) maps (B, H, L, D) to
 * (B, H, L, D), causal. Row i of query head h is the decode output above over
 * keys 0..i of kv head h / (Hq/Hkv) (all L keys when causal == 0).
 *  - q, r, out [B][Hq][L][D]; k, v [B][Hkv][L][D]; bf16 inputs (device
 *    pointers, 16-byte aligned); out bf16 or fp32 (out_dtype).
 *  - D is 64 or 128; B and Hq at most 65535; scale positive and finite (the
 *    softmax temperature; PARALLAX_ERR_BAD_SHAPE otherwise).
 *  - The products Q K^T, R K^T, P V and (P o T) V run on the tcgen05 tensor
 *    cores (accumulators in tensor memory, P read from tensor memory). The
 *    weights e and e*s enter the value products as follows:
 *      fp32 output: three bf16 terms each, which sum to the fp32 values exactly;
 *      bf16 output, workspace of parallax_prefill_workspace_bytes(B, L, Hkv, D)
 *      bytes or more: one fp16 term each (11 significant bits), against an fp16
 *      copy of V that a kernel launched first writes into the workspace, on every
 *      64-key tile whose V values are all below 2^16 in magnitude (fp16 holds
 *      them exactly down to 2^-17, within 2^-25 below); e*s carries a power-of-
 *      two factor per row, from a bound on |r . k|, that keeps it in fp16's
 *      range. Other tiles, and every tile with a smaller workspace, take
 *      bf16 hi + lo pairs of the weights rounded to 17 significant bits.
 *  - workspace: at least 256 bytes, zeroed once; its first word is the device
 *    status word read by parallax_workspace_status. The rest (fp16 copy of V,
 *    per-block records) is rewritten by every call, so concurrent calls need
 *    separate workspaces.
 * Errors as parallax_decode.
 */
int parallax_prefill(const void* q, const void* r, const void* k, const void* v,
                     void* out, int B, int Hq, int Hkv, int L, int D, float scale,
                     int causal, void* stream, int out_dtype, void* workspace,
                     size_t workspace_bytes);

/*
 * Workspace bytes with which a bf16-output parallax_prefill (dense: B batch
 * rows of L keys) or parallax_varlen_prefill (B = 1, L = total_tokens) takes
 * the fp16 value products: the 256-byte header, an fp16 copy of V
 * (B * L * Hkv * D * 2 bytes from byte 1024) and 4 bytes per kv item and
 * 64-key block. Returns 0 for B, L or Hkv below 1 or D other than 64 or 128.
 */
size_t parallax_prefill_workspace_bytes(int B, int L, int Hkv, int D);

/*
 * The packed variable-length forward: parallax-kernel 0.1.0 README, "Helion
 * kernels (experimental)" and "Install" name parallax_varlen_func beside
 * parallax_func ("training (dense + varlen)"). The pages give no signature; this
 * takes the usual packed form: sequence b occupies rows cu_seqlens[b] ..
 * cu_seqlens[b+1]-1 of the token dimension and each row attends (causally,
 * unless causal == 0) to the keys of its own sequence only, with the
 * arithmetic of parallax_prefill.
 *  - q, r, out [total_tokens][Hq][D]; k, v [total_tokens][Hkv][D]; bf16 inputs
 *    (device pointers, 16-byte aligned); out bf16 or fp32 (out_dtype).
 *  - cu_seqlens: device int32 [B + 1], non-decreasing, cu_seqlens[0] = 0,
 *    cu_seqlens[B] = total_tokens. Values outside [0, total_tokens] or a
 *    decreasing pair are clamped on the device (no row outside the buffers is
 *    touched) and set PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED.
 *  - max_seqlen: the longest sequence (it sizes the grid; a longer sequence
 *    sets PARALLAX_DEVICE_STATUS_SEQLEN_CLAMPED and its first rows are not
 *    written). 1 <= max_seqlen <= total_tokens.
 *  - Rows of a neighbouring sequence may be read into a tile and masked out
 *    (weight 0), so inputs must be finite.
 *  - workspace and errors as parallax_prefill (the fp16 value products with
 *    parallax_prefill_workspace_bytes(1, total_tokens, Hkv, D) bytes or more).
 */
int parallax_varlen_prefill(const void* q, const void* r, const void* k, const void* v,
                            const int32_t* cu_seqlens, void* out, int B, int total_tokens,
                            int max_seqlen, int Hq, int Hkv, int D, float scale, int causal,
                            void* stream, int out_dtype, void* workspace,
                            size_t workspace_bytes);

/*
 * Synchronise the current device, then read (and, if clear != 0, zero) the
 * device status word at the start of a workspace. *device_status receives PARALLAX_DEVICE_STATUS_* bits;
 * the return value maps them to a status: PARALLAX_ERR_DEVICE_TIMEOUT if a
 * bounded wait inside a kernel gave up (the kernel then returned early and its
 * output is invalid), PARALLAX_ERR_SEQLEN_CLAMPED if a length was outside
 * [0, Lmax], else PARALLAX_OK.
 */
int parallax_workspace_status(void* workspace, int clear, uint32_t* device_status);

/* Human-readable text for a status code; never NULL. */
const char* parallax_status_string(int status);

/*
 * parallax_decode_noalloc - parallax_decode for callers that cannot allocate.
 *
 * The paper has no counterpart to this entry point; it exists for callers of
 * this library that have no way to obtain device memory for the workspace:
 * for example a plugin or C host program running next to a framework whose
 * memory pool has already reserved the GPU's memory, or a latency-critical
 * decode loop that must never call cudaMalloc (which can synchronise the
 * device and fail once a pool holds everything). Such callers pass only the
 * inputs and the output; the workspace is a fixed array of
 * PARALLAX_NOALLOC_SCRATCH_BYTES in the library's own device memory, which
 * every GPU that loads the library holds until the process exits.
 *
 *  - Arguments are those of parallax_decode without workspace and
 *    workspace_bytes; the same layouts, dtypes and errors apply.
 *  - Capacity: with D = 128 the array holds 1008 partitions for 2 query
 *    heads per kv head, 504 for 4, 252 for 8 and 126 for 16 (twice as many
 *    at D = 64). With num_splits = 0 the call takes the default count (one
 *    partition per SM, 148 on a B200) capped at that capacity, so a default
 *    call never fails for size. An explicit num_splits whose workspace
 *    (parallax_decode_workspace_bytes for the same shape and count) exceeds
 *    PARALLAX_NOALLOC_SCRATCH_BYTES is rejected with
 *    PARALLAX_ERR_SCRATCH_LIMIT before anything is launched.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and keeps it for the
 *    life of the process; make that first call before any stream capture,
 *    and do not use this entry point across a cudaDeviceReset (or any other
 *    teardown of the device's primary context), which frees the array and
 *    leaves the kept address stale.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears the status word at its start (a
 *    cudaMemsetAsync on `stream`). Calls that can overlap on the GPU (other
 *    streams, other host threads) race on the array: order them.
 *  - Device-side status (bounded-wait timeouts, clamped lengths) is kept in
 *    the array and not reported; use parallax_decode to read it.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define PARALLAX_NOALLOC_SCRATCH_BYTES (4u << 20)
#define PARALLAX_ERR_SCRATCH_LIMIT (-12)
int parallax_decode_noalloc(const void* q, const void* r, const void* k_cache,
                            const void* v_cache, const int32_t* cache_seqlens,
                            void* out, int B, int Hq, int Hkv, int D, float scale,
                            void* stream, int Lmax, int in_dtype, int out_dtype,
                            int num_splits);

/*
 * Stream-ordered copy of `bytes` bytes from src to dst done by a kernel, not
 * by a DMA engine: for the small per-step transfers of a decode loop (q, r
 * and the lengths in, the output back), where the fixed latency of a DMA copy
 * is several times the kernel's own. The pages have no counterpart; it exists
 * for callers that keep a step's inputs and outputs in host memory.
 *  - Each pointer is device memory, managed memory, or page-locked host
 *    memory mapped into the current device's address space (cudaHostAlloc or
 *    cudaHostRegister memory on a system with unified addressing); host
 *    pointers are translated to their device mapping (cudaPointerGetAttributes'
 *    devicePointer). Pageable host
 *    memory, or a host block not mapped for this device, gives
 *    PARALLAX_ERR_BAD_SHAPE before anything is launched.
 *  - Both pointers 16-byte aligned and bytes a multiple of 16
 *    (PARALLAX_ERR_MISALIGNED otherwise); bytes = 0 launches nothing. The
 *    ranges must not overlap.
 *  - Writes to host memory are fenced at system scope before the kernel
 *    ends, so a host thread that waits for the stream (or a later event on
 *    it) reads the copied bytes.
 */
int parallax_copy(void* dst, const void* src, size_t bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARALLAX_H */
