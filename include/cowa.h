/*
 * cowa.h -- C ABI of the CoWindow Attention (CoWA) library for B200 (sm_100a).
 *
 * CoWA is the position-defined, block-sparse causal attention of
 * "CoWindow Attention: Full Causal Coverage Is a Collective Property"
 * (abstract; paper digest, method key points).  Every KV head sees a shared
 * prefix-sink window and a shared near-diagonal window, plus its own
 * complementary long-range window; the long windows of the KV heads split the
 * remaining history into equal-width slices, so the union over heads is the
 * full causal prefix.  The windows are described by the quadruple
 * (sink width S, near width N, gap G, long-range width W) and by
 * bottom-right-aligned causal distance, used identically for training,
 * prefill and decoding.
 *
 * Exact rule (the pages give no breakpoint formula; this library fixes it):
 * for query row i of Lq and key j of Lk, p = i + Lk - Lq and d = p - j.
 * Key j is visible to KV head h (global index) iff d >= 0 and
 *     j < S   or   d < N   or   N+G+h*W <= d < N+G+(h+1)*W.
 * Query head hq uses KV head floor(hq / (Hq/Hkv)) (contiguous GQA groups).
 *
 * Conventions for every entry point
 *  - Tensors are bf16 in [B, L, H, d] order with the last dimension
 *    contiguous; the other three strides are given in ELEMENTS and must be
 *    multiples of 8 (16 bytes).  Base pointers must be 16-byte aligned.
 *  - LSE is fp32, contiguous [B, Hq, Lq], natural logarithm; a query row
 *    that sees no key gets O = 0 and LSE = -inf.
 *  - d (head dimension) is 64 or 128.
 *  - All device pointers are owned by the caller.  The library allocates no
 *    memory: scratch space is the caller's workspace buffer, sized by the
 *    matching *_workspace_size call, 256-byte aligned.
 *  - Calls are asynchronous on the given CUDA stream (a cudaStream_t passed as
 *    void*; NULL is the legacy default stream).  They return only
 *    launch-time errors; they never abort or throw.  Kernel-side errors
 *    (a bounded wait that ran out) are recorded in a device word that
 *    cowa_get_device_error() reads.
 *  - Thread safety: calls may be issued from several host threads; the
 *    detail string of the last error is per thread.
 */
#ifndef COWA_H
#define COWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define COWA_ABI_VERSION 1

#if defined(__GNUC__)
#define COWA_API __attribute__((visibility("default")))
#else
#define COWA_API
#endif

/* Window quadruple (sink width, near width, gap, long-range width), in keys. */
typedef struct {
    int32_t S, N, G, W;
} cowa_quad_t;

/*
 * Problem shape.  Hkv is the number of KV heads present in the tensors;
 * kv_head_offset is the global index of the first of them (0 on one GPU; a
 * rank of a KV-head tensor-parallel group passes the index of its first head
 * so the windows stay those of the global head, as the paper digest's
 * execution notes describe).  Strides are in elements for (b, l, h).
 */
typedef struct {
    int64_t B, Lq, Lk, Hq, Hkv, d;
    int64_t q_stride[3];  /* Q, and dQ in cowa_bwd */
    int64_t k_stride[3];  /* K, and dK in cowa_bwd */
    int64_t v_stride[3];  /* V, and dV in cowa_bwd */
    int64_t o_stride[3];  /* O, and dO in cowa_bwd */
    int64_t kv_head_offset;
} cowa_shape_t;

typedef enum {
    COWA_OK = 0,
    COWA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, negative window */
    COWA_ERR_UNSUPPORTED = 2,  /* head dim not 64/128, no sm_100 device */
    COWA_ERR_ALIGNMENT = 3,    /* pointer or stride not 16-byte aligned */
    COWA_ERR_WORKSPACE = 4,    /* workspace missing or too small */
    COWA_ERR_CUDA = 5,         /* a CUDA runtime call failed */
    COWA_ERR_TIMEOUT = 6,      /* a kernel's bounded wait ran out */
    COWA_ERR_DEVICE = 7        /* a kernel's own consistency check failed */
} cowa_status_t;

/* Human-readable name of a status code (static string). */
COWA_API const char *cowa_status_string(int status);

/* Detail of the last error raised on this host thread ("" if none). */
COWA_API const char *cowa_last_error_detail(void);

/* ABI version of the loaded library (COWA_ABI_VERSION). */
COWA_API int cowa_abi_version(void);

/* Number of CUDA kernels this library has launched in this process. */
COWA_API uint64_t cowa_launch_count(void);

/*
 * Packed (variable-length) batches for training (chunked prefill included):
 * sequence b owns query rows [cu_q[b], cu_q[b+1]) of q / o / dq / dO and key
 * rows [cu_k[b], cu_k[b+1]) of k / v / dk / dv, each tensor [total, H, d]
 * bf16 with the given (token, head) strides in elements (multiples of 8, last
 * dim contiguous, 16-byte aligned bases).  cu_q / cu_k are device int32
 * arrays of B + 1 ascending offsets; max_q / max_k bound every sequence's
 * length.  Each sequence is aligned bottom-right on its own (p = i + Lk_b -
 * Lq_b), exactly as a batch of one (paper digest, method key points: the
 * same position rule for training, prefill and decoding).  LSE is fp32
 * [Hq, total_q].  A sequence whose offsets do not fit the tensors or exceed
 * max_q / max_k is treated as empty and reported by cowa_get_device_error
 * (COWA_ERR_DEVICE); no access leaves the tensors.  Batches without any key
 * (or, for the backward, any query) are refused with COWA_ERR_UNSUPPORTED.
 */
typedef struct {
    int64_t B;                   /* sequences */
    int64_t total_q, total_k;    /* rows of the packed query / key tensors */
    int64_t max_q, max_k;        /* longest query / key sequence */
    int64_t Hq, Hkv, d;
    int64_t q_stride[2], k_stride[2], v_stride[2], o_stride[2]; /* token, head */
    int64_t kv_head_offset;
} cowa_varlen_shape_t;

COWA_API size_t cowa_fwd_varlen_workspace_size(const cowa_varlen_shape_t *shape, cowa_quad_t quad);
COWA_API size_t cowa_bwd_varlen_workspace_size(const cowa_varlen_shape_t *shape, cowa_quad_t quad);
COWA_API int cowa_fwd_varlen(const cowa_varlen_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                             const int32_t *cu_q, const int32_t *cu_k, const void *q, const void *k,
                             const void *v, void *o, float *lse, void *workspace, size_t workspace_bytes,
                             void *stream);
COWA_API int cowa_bwd_varlen(const cowa_varlen_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                             const int32_t *cu_q, const int32_t *cu_k, const void *q, const void *k,
                             const void *v, const void *o, const float *lse, const void *dout, void *dq,
                             void *dk, void *dv, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Windowed decode cache (paper: decoding reads only each head's windows;
 * Digest, execution notes, and the decode memory saving of the abstract).
 * For a horizon of R query positions [origin[b], origin[b] + R) of sequence
 * b, KV head h only ever sees the keys of sink [0, S), near
 * [origin-N+1, origin+R-1] and its long slice [origin-e+1, origin+R-1-c]
 * (c = N+G+hW, e = c+W).  The windowed cache stores exactly that key set per
 * (sequence, KV head), merged and in ascending key order, in a contiguous
 * bf16 tensor [B, rows, Hkv, d] with rows = cowa_wcache_rows(quad, R);
 * unused rows are zero.  h is the GLOBAL head (local + kv_head_offset).
 *
 * cowa_wcache_rows: S + N + W + 2R, an upper bound of every head's key set
 *   (0 for a negative field or R <= 0, or if the result reaches 2^30).
 * cowa_wcache_build: from a full cache k_full/v_full [B, Lk, Hkv, d]
 *   (shape->Lk, shape->k_stride, shape->v_stride; Lq, Hq, q/o strides are
 *   ignored) and device int32 origin[B] (origin[b] < Lk: the position of the
 *   query at build time, so keys 0..origin[b] exist), fills k_win/v_win.
 *   Keys above origin[b] are left zero for cowa_wcache_append.
 * cowa_wcache_append: writes the K/V of the token at device int32 pos[b]
 *   (k_new/v_new [B, Hkv, d]; shape->k_stride[0] / [2] and v_stride[0] / [2]
 *   are their batch and head strides) into the rows that hold it.
 * cowa_decode_windowed: as cowa_decode over a windowed cache (shape->Lk =
 *   rows, k/v strides those of the contiguous windowed tensors); the query
 *   of sequence b sits at seqlens[b] - 1, which must lie in
 *   [origin[b], origin[b] + R).  Workspace: cowa_decode_workspace_size.
 * Errors: as cowa_decode; a device-side position outside the horizon (or an
 * origin outside the source) sets COWA_ERR_DEVICE for cowa_get_device_error
 * and the sequence reads or writes nothing.
 */
COWA_API int64_t cowa_wcache_rows(cowa_quad_t quad, int32_t horizon);
COWA_API int cowa_wcache_build(const cowa_shape_t *shape, cowa_quad_t quad, int32_t horizon,
                               const int32_t *origin, const void *k_full, const void *v_full,
                               void *k_win, void *v_win, void *stream);
COWA_API int cowa_wcache_append(const cowa_shape_t *shape, cowa_quad_t quad, int32_t horizon,
                                const int32_t *origin, const int32_t *pos, const void *k_new,
                                const void *v_new, void *k_win, void *v_win, void *stream);
COWA_API int cowa_decode_windowed(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                                  int32_t horizon, const int32_t *origin, const void *q,
                                  const void *k_win, const void *v_win, const int32_t *seqlens,
                                  void *o, float *lse, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Kernel trace, a measurement aid with no counterpart in the paper.
 * cowa_trace_start(capacity, only) creates `capacity` CUDA event pairs on
 * the current device and turns tracing on (capacity 0 turns it off and frees
 * them); any earlier trace is discarded.  While on, each kernel the library
 * launches on that device -- only the kernel named `only`, unless `only` is
 * NULL or "" -- records one pair on its own stream, bracketing that launch
 * alone; launches past the capacity, or on another device, are counted by
 * cowa_trace_dropped() and not recorded.  cowa_trace_stop() stops
 * recording and keeps the records.  cowa_trace_entry(i, &name, &ms) waits for
 * record i (0 <= i < cowa_trace_size()) and gives the kernel's name (a
 * static string: "fwd_sm100", "dkdv_sm100", "dq_sm100", "bwd_prep",
 * "decode_split", "decode_combine", "schedule", ...) and its duration in
 * milliseconds.  Start/stop are not meant to race with launches from other
 * host threads; entries stay valid until the next cowa_trace_start.
 * Errors: COWA_ERR_INVALID_ARG (capacity outside 0..2^20, `only` of 64
 * characters or more, index out of range, NULL output), COWA_ERR_CUDA (event creation or timing failed).
 */
COWA_API int cowa_trace_start(int64_t capacity, const char *only);
COWA_API int cowa_trace_stop(void);
COWA_API int64_t cowa_trace_size(void);
COWA_API int64_t cowa_trace_dropped(void);
COWA_API int cowa_trace_entry(int64_t i, const char **name, float *ms);

/*
 * Default quadruple: G = 0 and W = ceil((Lk - N) / Hkv), clamped at 0, so
 * the Hkv long windows exactly cover distances N .. Lk-1.  Hkv here is the
 * GLOBAL number of KV heads.
 */
COWA_API cowa_quad_t cowa_default_quad(int64_t Lk, int64_t Hkv, int32_t S, int32_t N);

/* Workspace bytes for each call (0 is never returned for a valid shape). */
COWA_API size_t cowa_fwd_workspace_size(const cowa_shape_t *shape, cowa_quad_t quad);
COWA_API size_t cowa_bwd_workspace_size(const cowa_shape_t *shape, cowa_quad_t quad);
COWA_API size_t cowa_decode_workspace_size(const cowa_shape_t *shape, cowa_quad_t quad);

/*
 * Training / prefill forward (paper abstract: training forward pass).
 *   q [B, Lq, Hq, d], k/v [B, Lk, Hkv, d] in; o [B, Lq, Hq, d] bf16 and
 *   lse [B, Hq, Lq] fp32 out.  O_i = sum_j softmax_j(scale * q_i.k_j) v_j over
 *   the keys visible to row i.  softmax_scale <= 0 selects 1/sqrt(d).
 * Only key tiles that hold at least one visible pair are read ("block
 * traversal skips invisible KV blocks", paper digest, execution notes).
 */
COWA_API int cowa_fwd(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
             const void *q, const void *k, const void *v, void *o, float *lse,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Training backward (paper abstract: training backward pass).
 *   Inputs q, k, v, o (the forward output), lse (the forward's), dO (o's
 *   strides).  Outputs dq (q's strides), dk (k's strides), dv (v's strides),
 *   bf16.  dK and dV sum the contributions of the query heads of each group.
 *   Recomputes P = exp(scale*q.k - LSE) per visible tile; delta = rowsum(dO*O).
 */
COWA_API int cowa_bwd(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
             const void *q, const void *k, const void *v, const void *o,
             const float *lse, const void *dout, void *dq, void *dk, void *dv,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * MassAlloc Attention (MALA), the companion operator of the same pages
 * ("Two new attention models slash redundancy...", first section; "CoWindow
 * Attention: Full Causal Coverage Is a Collective Property", abstract): it
 * keeps full causal QK scoring and lets attention's own softmax statistics
 * decide where the remaining work of a block is skipped.  The pages give no
 * rule; this library fixes the plainest reading:
 *   - scores on every causal pair (bottom-right alignment, p = i + Lk - Lq;
 *     query head hq uses KV head hq / (Hq / Hkv)); LSE over all of them;
 *   - per block of 128 query rows x 64 keys of one head, the mass each row
 *     gives the block, M = sum_j P_ij with P = exp(s - LSE); the block is kept
 *     when some row of it has M >= tau, skipped otherwise;
 *   - O_i = sum over kept blocks of P_ij v_j: the dropped mass is not
 *     redistributed (LSE stays the full statistic);
 *   - the gradient is that of this O with the block decisions held fixed:
 *     dV and dP only over kept pairs, dS = P (dP - delta) over every causal
 *     pair (skipped pairs keep -P * delta through the LSE).
 * The decision compares an fp32 sum of the kernel's fp32 probabilities with
 * tau; a block whose mass lies within about 1e-5 (relative) of tau may be
 * decided either way.
 *
 * cowa_mala_keep_bytes: bytes of the decision array keep[B][Hq][ceil(Lq/128)]
 *   [ceil(Lk/64)] (uint8: 1 kept, 0 skipped or past the causal diagonal).
 * cowa_mala_fwd: q, k, v as for cowa_fwd (shape->kv_head_offset must be 0:
 *   MALA has no per-head windows); o [B, Lq, Hq, d] bf16, lse [B, Hq, Lq]
 *   fp32 (natural log) and keep (device, cowa_mala_keep_bytes) out.  tau is
 *   a finite value >= 0: tau = 0 keeps every causal block (dense causal
 *   attention), tau > 1 keeps none (O = 0, LSE still the full statistic).
 *   Needs no workspace.  Rows with no causal key give O = 0, LSE = -inf.
 * cowa_mala_bwd: q, k, v, o, lse and keep from cowa_mala_fwd, dout (o's
 *   strides); dq, dk, dv out as for cowa_bwd; workspace of
 *   cowa_mala_bwd_workspace_size bytes, 256-byte aligned.
 * Both are asynchronous on `stream`; errors as for cowa_fwd / cowa_bwd
 * (COWA_ERR_INVALID_ARG for a NULL keep, tau < 0 or not finite, or a
 * nonzero kv_head_offset).
 */
COWA_API size_t cowa_mala_keep_bytes(const cowa_shape_t *shape);
COWA_API int cowa_mala_fwd(const cowa_shape_t *shape, float tau, float softmax_scale,
             const void *q, const void *k, const void *v, void *o, float *lse, uint8_t *keep,
             void *stream);
COWA_API size_t cowa_mala_bwd_workspace_size(const cowa_shape_t *shape);
COWA_API int cowa_mala_bwd(const cowa_shape_t *shape, float softmax_scale,
             const void *q, const void *k, const void *v, const void *o, const float *lse,
             const uint8_t *keep, const void *dout, void *dq, void *dk, void *dv,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Single-token decode over a KV cache (paper abstract: decoding).
 *   shape->Lq must be 1 and shape->Lk is the cache capacity Lcap.
 *   q [B, 1, Hq, d]; k_cache / v_cache [B, Lcap, Hkv, d]; seqlens [B] int32
 *   on the device, 0 <= seqlens[b] <= Lcap: keys 0 .. seqlens[b]-1 are valid
 *   and the new token's own K/V is already stored at seqlens[b]-1, so the
 *   query sits at p = seqlens[b]-1.  The quadruple is the model's (it is not
 *   re-derived from the current length).  Out: o [B, 1, Hq, d] bf16 and
 *   lse [B, Hq] fp32.  Only visible keys are read (split over the KV
 *   sequence, then merged with LSE weights).
 */
COWA_API int cowa_decode(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                const void *q, const void *k_cache, const void *v_cache,
                const int32_t *seqlens, void *o, float *lse, void *workspace,
                size_t workspace_bytes, void *stream);

/*
 * Decode that allocates nothing (no counterpart in the paper: it exists for
 * callers that cannot allocate device memory, such as a plugin inside another
 * runtime that owns all device memory and passes only input and output
 * buffers, or a serving loop where cudaMalloc, which may synchronise the
 * device, is not allowed).
 *   Same arguments and results as cowa_decode, without the workspace: the
 *   split-KV partials live in a static device array of
 *   COWA_DECODE_NOALLOC_SCRATCH_BYTES bytes inside the library, which every
 *   GPU that loads the library holds until the process exits.  Shapes whose
 *   partials (cowa_decode_workspace_size) exceed it are refused with
 *   COWA_ERR_WORKSPACE and a detail message; nothing is launched then.  The
 *   split count, hence the size, depends on the device's SM count: a caller
 *   can check cowa_decode_workspace_size(shape, quad) <=
 *   COWA_DECODE_NOALLOC_SCRATCH_BYTES on the target device ahead of time.
 *   The first call in a CUDA context (the device's primary context, another
 *   context a host runtime makes current, or a new primary context after a
 *   device reset) looks up the array's device address in that context
 *   (cudaGetSymbolAddress) and keeps it under the context's ID; make that
 *   first call before any stream capture.  Every call on a device shares the one array:
 *   calls whose kernels overlap on the GPU (different streams, no ordering
 *   between them) race on it and must not be issued.  The array keeps the
 *   last call's partials; each call overwrites every partial it reads.
 *   No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define COWA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
COWA_API int cowa_decode_noalloc(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                                 const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *seqlens, void *o, float *lse, void *stream);

/*
 * Visible-tile classes of one KV head, as the training kernels see them, for
 * checking the schedule: writes out[qt * nkt + kt] (device, uint8) for the
 * tiling BM x BN, BM in {32, 64, 128} and BN in {64, 96, 128} (the forward
 * uses query tiles of 128 with key tiles of 128; the dQ pass query tiles of 128 with key tiles of 64; the dK/dV
 * pass, key-tile major, key tiles of 128 with query tiles of 64 for d = 64
 * and 32 for d = 128),
 * nqt = ceil(Lq/BM), nkt = ceil(Lk/BN):
 *   0 = tile skipped, 1 = visited with the element mask applied,
 *   2 = visited without a mask (every in-range pair visible).
 * kv_head is the global KV-head index.  transposed = 0 uses the
 * query-tile-major schedule (forward, dQ), 1 the key-tile-major schedule
 * (dK/dV).  workspace as from cowa_schedule_workspace_size.
 */
COWA_API size_t cowa_schedule_workspace_size(int64_t Lq, int64_t Lk, int32_t BM, int32_t BN);
COWA_API int cowa_tile_classes(int64_t Lq, int64_t Lk, int64_t kv_head, cowa_quad_t quad,
                      int32_t BM, int32_t BN, int transposed, uint8_t *out,
                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * Reads and clears the device error word (synchronises the stream).
 * Returns COWA_OK, COWA_ERR_TIMEOUT or COWA_ERR_DEVICE.
 */
COWA_API int cowa_get_device_error(void *stream);

/*
 * Self-test of the timeout path: launches one 32-thread block whose only
 * work is the kernels' bounded mbarrier wait on a barrier that nothing
 * completes.  After the wait limit (2 s) the block records COWA_ERR_TIMEOUT in
 * the device error word and returns, so the context stays usable, and
 * cowa_get_device_error(stream) then returns COWA_ERR_TIMEOUT.  Touches no
 * caller memory.  Returns launch-time errors only: COWA_ERR_UNSUPPORTED on a
 * device other than sm_100, COWA_ERR_CUDA if the launch fails.
 */
COWA_API int cowa_selftest_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* COWA_H */
