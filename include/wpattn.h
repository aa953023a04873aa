/*
 * wpattn — per-RoPE-wavelength windowed causal attention on NVIDIA B200 (sm_100a).
 *
 * The method ("ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract;
 * "WavePrune: One period is often enough for RoPE", Original abstract):
 * the RoPE attention score is a sum of one term per 2-D rotation pair p
 * (dims p and p + D/2), and the window drops pair p's term once the
 * query-key distance d = q_pos - k_pos exceeds T_p = floor(alpha * lambda_p),
 * lambda_p = 2*pi * base^(2p/D).  Dropped terms add 0 to the score; the
 * causal softmax over keys is unchanged:
 *
 *     s(i,j) = sum_p [d <= T_p] * (q[i,p] k[j,p] + q[i,p+D/2] k[j,p+D/2])
 *     out_i  = softmax_j(scale * s(i,j)) . v_j      over keys with k_pos <= q_pos
 *
 * With group_pairs = 8 the pairs {8m..8m+7} (16 head dims, the Tensor-Core
 * block size of WavePrune's kernels) share the threshold of the group's
 * longest wavelength, T_{8m+7}.  alpha = +INFINITY disables the window.
 *
 * Conventions for every entry point:
 *  - Return value: WPATTN_OK or an error code (wpattn_strerror names it).
 *    Argument errors are reported synchronously and nothing is launched.
 *  - Device pointers are plain CUDA device addresses of the current device;
 *    the caller owns every buffer.  Kernels run asynchronously on
 *    `cuda_stream` (a cudaStream_t; NULL = the legacy default stream); the
 *    call does not synchronise.  A kernel fault shows at the caller's next
 *    synchronisation.  A kernel that gives up waiting (a bounded spin ran out)
 *    records WPATTN_ETIMEOUT, which wpattn_device_status returns.
 *  - bf16 tensors are contiguous, row-major, in the layouts stated below, and
 *    16-byte aligned.
 *  - No entry point allocates device memory.  The library's device image holds
 *    a 4-byte status word and the scratch array of wpattn_decode_noalloc.
 */
#ifndef WPATTN_H
#define WPATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WPATTN_API __attribute__((visibility("default")))
#else
#define WPATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum {
    WPATTN_OK = 0,
    WPATTN_EINVAL = 1,        /* bad argument (null pointer, bad shape, alpha <= 0 or NaN, ...) */
    WPATTN_EUNSUPPORTED = 2,  /* valid but not supported here (head_dim, device arch, size limit) */
    WPATTN_ECUDA = 3,         /* a CUDA runtime call or a kernel launch failed */
    WPATTN_ETIMEOUT = 4,      /* a kernel's bounded wait ran out (see wpattn_device_status) */
    WPATTN_EWORKSPACE = 5,    /* workspace null or smaller than wpattn_decode_workspace_size */
    WPATTN_EINDEX = 6         /* a device-side index was out of range (block-table entry outside
                                 the pool, negative key position); see wpattn_device_status */
};

/*
 * The window: head dim D (64 or 128 on the GPU paths; any even D for the
 * host planner), RoPE base (> 1), factor alpha (> 0; +INFINITY = window off)
 * and pair granularity g (1 or 8; 8 needs D/2 divisible by 8).
 * T_p is evaluated on the host in IEEE double as
 *     floor(alpha * (6.283185307179586 * pow(base, (double)(2p) / D)))
 * and every device comparison is an integer one.
 */
typedef struct wpattn_window {
    int32_t head_dim;
    int32_t group_pairs;
    double rope_base;
    double alpha;
} wpattn_window;

/*
 * Per-pair thresholds T_eff[p], p = 0 .. D/2 - 1 (host only; ATFlash
 * Abstract: "wavelength-proportional distance").  With g = 8 each pair holds
 * its group's threshold.  A disabled window reports INT64_MAX.
 * T_eff: caller-owned host array of D/2 entries.
 */
WPATTN_API int wpattn_thresholds(const wpattn_window *w, int64_t *T_eff);

/*
 * Pruned pair-terms of one (batch, head) of a prefill (host only, O(D)
 * closed form; ATFlash Abstract: "closed form logarithmic in the sequence
 * length").  Queries t = 0..Nq-1 sit at q_pos0 + t, keys j = 0..Nk-1 at
 * k_pos0 + j; every causal (query, key) pair contributes D/2 pair-terms and
 * a term is pruned when its distance exceeds its pair's threshold.
 * Outputs (host pointers, any may be NULL): pruned and total term counts and
 * their ratio (0 when total is 0).
 */
WPATTN_API int wpattn_pruned_fraction(const wpattn_window *w, int64_t Nq, int64_t Nk,
                           int64_t q_pos0, int64_t k_pos0,
                           uint64_t *pruned_terms, uint64_t *total_terms,
                           double *fraction);

/*
 * Prefill (ATFlash Abstract: the window as a slice of the query-key
 * contraction axis inside a FlashAttention-style kernel; WavePrune: 16-dim
 * head-dim blocks for the Tensor Cores).
 *   q   : bf16 device [B, Nq, Hq, D]      query t at position q_pos0 + t
 *   k, v: bf16 device [B, Nk, Hkv, D]     key j at position k_pos0 + j
 *   out : bf16 device [B, Nq, Hq, D]      written
 *   lse : fp32 device [B, Hq, Nq] natural-log sum-exp of scale*s, or NULL
 * Query head h reads kv head h / (Hq / Hkv).  softmax_scale <= 0 means
 * 1/sqrt(D).  A query with no causal key gets out = 0 and lse = -inf.
 * Requires D in {64, 128}, Hq % Hkv == 0, an sm_100 device,
 * 0 <= Nq, Nk <= 2^30 and |q_pos0 - k_pos0| <= 2^30 (else WPATTN_EUNSUPPORTED).
 * Nq == 0 or B == 0 is a no-op.
 */
WPATTN_API int wpattn_prefill(const wpattn_window *w,
                   const void *q, const void *k, const void *v,
                   void *out, float *lse,
                   int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                   int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                   void *cuda_stream);

/*
 * Prefill with the key ranges of some work items split into parts (flash-
 * decoding's split along the keys, applied to prefill CTAs).  A work item is
 * one 256-row query block of one head of one sequence: one CTA of
 * wpattn_prefill's grid.  A split item runs as P CTAs, one per range of
 * ceil(nkt / P) key tiles of 128 keys (a range past the last key tile is
 * dropped); each writes its rows' fp32 result, normalised over its own keys,
 * and the log2-sum-exp of its scores into the workspace, and a merge kernel
 * combines the parts (weights 2^(l_s - max l)) into out and lse.  The items
 * that are not split run in wpattn_prefill's kernel, unchanged.
 *   kv_splits = 0: the library's plan (wpattn_prefill_split_plan) on the
 *                  current device; it splits only the items of the grid's last
 *                  partial wave, and only when every item does the same work;
 *   kv_splits = 1: nothing is split (wpattn_prefill);
 *   kv_splits = 2 .. 64: every item in kv_splits parts.
 * Same arguments and results as wpattn_prefill (equal to it up to float
 * rounding order), plus:
 *   workspace: device, 256-byte aligned, at least
 *              wpattn_prefill_split_workspace_size(...) bytes when the plan
 *              splits anything (else WPATTN_EWORKSPACE; WPATTN_EINVAL when
 *              NULL or misaligned); unused otherwise.
 * kv_splits outside 0 .. 64: WPATTN_EINVAL.
 */
WPATTN_API int wpattn_prefill_split(const wpattn_window *w,
                   const void *q, const void *k, const void *v,
                   void *out, float *lse,
                   int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                   int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                   int32_t kv_splits, void *workspace, size_t workspace_bytes,
                   void *cuda_stream);

/*
 * The split plan of wpattn_prefill_split on a device with num_sms SMs
 * (num_sms <= 0: the current device).  Host only.  Outputs (any may be NULL):
 * the items run unsplit (the first main_items in grid order), the items split
 * after them, and the parts of each split item (1 when none is split).
 * kv_splits = 0 plans as follows: when the last query sees at most 10% more
 * keys than the first (a chunk far into a long context), every item takes the
 * same time, and with one CTA per SM a grid of W full waves plus r < num_sms
 * items leaves most SMs idle while the last r run.  Those r items are split
 * into min(8, num_sms / r) parts of at least 64 key tiles, so they take a
 * fraction of a wave; nothing is split when r = 0 or fewer than 2 parts fit.
 */
WPATTN_API int wpattn_prefill_split_plan(int32_t B, int32_t Nq, int32_t Nk, int32_t Hq,
                   int64_t q_pos0, int64_t k_pos0, int32_t kv_splits, int32_t num_sms,
                   int64_t *main_items, int32_t *split_items, int32_t *parts);

/* Workspace bytes of wpattn_prefill_split for that plan: parts * split items *
 * 256 * (head_dim + 1) * 4; 0 when nothing is split or on bad sizes.  Host
 * only (num_sms <= 0: the current device). */
WPATTN_API size_t wpattn_prefill_split_workspace_size(int32_t B, int32_t Nq, int32_t Nk,
                   int32_t Hq, int32_t head_dim, int64_t q_pos0, int64_t k_pos0,
                   int32_t kv_splits, int32_t num_sms);

/*
 * Prefill with a block mask stacked on the window (token-level block
 * sparsity of the MInference kind; ATFlash Abstract: the window is orthogonal
 * to token selection and composes with it).  Same arguments and results as
 * wpattn_prefill, plus:
 *   block_mask: device uint32 [B, Hq, ceil(Nq / 128), mask_words], 4-byte
 *               aligned.  Query rows 128 qb .. 128 qb + 127 of head h attend
 *               keys 128 kb .. 128 kb + 127 only if bit kb % 32 of word
 *               kb / 32 of row (b, h, qb) is set; the window and causality
 *               then apply to the attended keys.  Bits past ceil(Nk / 128)
 *               are ignored.  Build it from a byte mask with
 *               wpattn_pack_block_mask.
 *   mask_words: words per row, >= ceil(ceil(Nk / 128) / 32) (else
 *               WPATTN_EINVAL).
 * Key tiles that no query tile of a CTA attends are neither loaded nor
 * computed.  A query left with no key gets out = 0 and lse = -inf.  An
 * all-ones mask gives wpattn_prefill's output bit for bit.
 */
WPATTN_API int wpattn_prefill_masked(const wpattn_window *w,
                  const void *q, const void *k, const void *v,
                  void *out, float *lse,
                  int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                  int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                  const uint32_t *block_mask, int32_t mask_words,
                  void *cuda_stream);

/*
 * Prefill with explicit per-token positions (ATFlash Abstract: the window is a
 * function of the query-key distance alone): query t of sequence b sits at
 * q_pos[b * q_pos_stride + t], key j at k_pos[b * k_pos_stride + j], for
 * caches that dropped tokens, chunks with gaps, or packed inputs whose
 * positions do not follow the index.  A key after its query is left out;
 * otherwise arguments and results as for wpattn_prefill.
 *   q_pos: device int32, 4-byte aligned, q_pos_stride >= Nq.
 *   k_pos: device int32, 16-byte aligned, k_pos_stride a multiple of 4 and
 *          >= Nk rounded up to a multiple of 128 (the kernel copies key
 *          positions 128 at a time; entries past Nk are read, never used).
 * Positions must be non-decreasing along each sequence and in
 * [0, 2^31 - 1); otherwise the output is undefined (no access leaves the
 * arrays).  Bad strides or alignment give WPATTN_EINVAL.
 */
WPATTN_API int wpattn_prefill_positions(const wpattn_window *w,
                  const void *q, const void *k, const void *v,
                  void *out, float *lse,
                  int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                  const int32_t *q_pos, int64_t q_pos_stride,
                  const int32_t *k_pos, int64_t k_pos_stride,
                  float softmax_scale, void *cuda_stream);

/*
 * Pack a byte block mask (device uint8 [rows, nkb], nonzero = attended) into
 * the bit rows wpattn_prefill_masked reads (device uint32 [rows, mask_words],
 * caller-allocated, 4-byte aligned; bit kb % 32 of word kb / 32, zero past
 * nkb).  mask_words >= ceil(nkb / 32) (else WPATTN_EINVAL).  Asynchronous on
 * `cuda_stream`; bit-exact.
 */
WPATTN_API int wpattn_pack_block_mask(const uint8_t *mask, uint32_t *words, int64_t rows,
                  int32_t nkb, int32_t mask_words, void *cuda_stream);

/*
 * Bytes of device workspace wpattn_decode needs for up to B sequences of up
 * to max_kv_len keys (0 on bad arguments).  The split of each sequence into
 * key ranges depends only on (B, Hkv, max_kv_len) and the device: its SM
 * count and how many decode CTAs one SM holds at once (the split fills at
 * most one such wave).  The size returned covers every device.
 */
WPATTN_API size_t wpattn_decode_workspace_size(const wpattn_window *w, int32_t B, int32_t Hq,
                                    int32_t Hkv, int64_t max_kv_len);

/*
 * Decode: one new query per sequence (ATFlash Abstract: the window ported
 * into a FlashInfer-style decode; K is read only over the active head-dim
 * slice of each key block).
 *   q          : bf16 device [B, Hq, D]; sequence b's query sits at position kv_len[b]-1
 *   k_cache,
 *   v_cache    : bf16 device [B, Lmax, Hkv, D]; key j at position j, j < kv_len[b] valid
 *   kv_len_host: host int32 [B], 1 <= kv_len[b] <= Lmax (read during the call)
 *   out        : bf16 device [B, Hq, D];  lse: fp32 device [B, Hq] or NULL
 *   workspace  : device, >= wpattn_decode_workspace_size(w, B, Hq, Hkv, Lmax)
 *                bytes, 256-byte aligned; its contents are scratch (fp32 partial
 *                results of each key range) and are overwritten.
 * Requires D in {64, 128}, Hq % Hkv == 0, Hq / Hkv <= 16, B <= 1024.
 */
WPATTN_API int wpattn_decode(const wpattn_window *w,
                  const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *kv_len_host, int64_t Lmax,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * Decode without any allocation: the same computation as wpattn_decode, with
 * its scratch (the per-split partial results) taken from a fixed array built
 * into the library instead of a caller-supplied workspace.  The paper has no
 * counterpart; it is for callers that cannot allocate device memory at the
 * point of the call: a serving runtime whose allocator already reserved the
 * GPU's memory, a plugin that only receives tensors from its host, or code on
 * a latency path where cudaMalloc (which can synchronise the device) is not
 * allowed.  Arguments as for wpattn_decode, minus the workspace.
 *  - The scratch array holds wpattn_decode_noalloc_max_bytes() bytes (4 MiB)
 *    on every GPU that loads the library, until the process exits.  A problem
 *    whose partial results need more (B * Hq * splits * (D + 2) * 4 bytes)
 *    is rejected with WPATTN_EWORKSPACE and nothing runs.
 *  - The first call on a device looks up the array's device address for that
 *    device (cudaGetSymbolAddress); make that first call before capturing a
 *    stream into a CUDA graph.
 *  - Every call on a device shares the one array: calls whose kernels can
 *    overlap on the GPU (different streams, no ordering) race on it.  Nothing
 *    in it needs clearing: each call writes every partial it later reads.
 */
WPATTN_API int wpattn_decode_noalloc(const wpattn_window *w,
                  const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *kv_len_host, int64_t Lmax,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse, void *cuda_stream);

/* Size in bytes of the built-in scratch array wpattn_decode_noalloc uses. */
WPATTN_API size_t wpattn_decode_noalloc_max_bytes(void);

/*
 * Decode with the K cache in the pair-major layout (a variant of this
 * library, not a layout of the pages; ATFlash Abstract: decode reads K only
 * over the active head-dim slice of each key block, and here that slice is
 * contiguous).
 *   k_slabs: bf16 device [B, Hkv, D/16, Lmax, 16].  Slab g of key j holds head
 *            dims 8g..8g+7 followed by D/2+8g..D/2+8g+7, i.e. the 8 RoPE pairs
 *            8g..8g+7 whose window group starts a contraction step.  Build it
 *            from a [B, Lmax, Hkv, D] cache with wpattn_kcache_to_pairmajor.
 * Every other argument, the result and the workspace are those of
 * wpattn_decode (same sizes, same errors); the two calls give the same
 * output.  A key block (32 keys) loads only the slabs of the groups kept at
 * some of its distances, so the window also cuts the bytes K moves from HBM.
 */
WPATTN_API int wpattn_decode_pairmajor(const wpattn_window *w,
                  const void *q, const void *k_slabs, const void *v_cache,
                  const int32_t *kv_len_host, int64_t Lmax,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * Rewrite a K cache [B, Lmax, Hkv, head_dim] (bf16, device) into the
 * pair-major slabs [B, Hkv, head_dim/16, Lmax, 16] that
 * wpattn_decode_pairmajor reads (bf16, device, caller-allocated,
 * B * Lmax * Hkv * head_dim * 2 bytes, must not overlap k_cache).  Both
 * pointers 16-byte aligned; head_dim in {64, 128} (else WPATTN_EUNSUPPORTED);
 * asynchronous on `cuda_stream`.  Bit-exact: only moves bytes.
 */
WPATTN_API int wpattn_kcache_to_pairmajor(const void *k_cache, void *k_slabs, int64_t Lmax,
                  int32_t B, int32_t Hkv, int32_t head_dim, void *cuda_stream);

/*
 * Decode with explicit positions: the keys of a sequence need not sit at
 * positions 0..kv_len-1 with the query right after them (a cache that evicted
 * or reordered tokens, a query at a position of its own).  ATFlash Abstract:
 * whether a pair is kept depends only on the relative position, so the
 * window is applied to d = q_pos[b] - k_pos[b, j].
 *   q_pos_host: host int32 [B], 0 <= q_pos < 2^31 - 1 (else WPATTN_EINVAL).
 *   k_pos:      device int32, k_pos[b * k_pos_stride + j] is the position of
 *               cache row j of sequence b (j < kv_len[b]); 4-byte aligned;
 *               k_pos_stride >= max kv_len (else WPATTN_EINVAL).  Positions
 *               need not be sorted or distinct.  A key whose position is
 *               after q_pos[b] is left out (causality).  A negative position
 *               is an error found on the device: the key is left out and
 *               WPATTN_EINDEX is recorded for wpattn_device_status.
 * Every other argument, the result and the workspace are those of
 * wpattn_decode.  A sequence with no key at or before its query gets out = 0
 * and lse = -inf.  With k_pos[b, j] = j and q_pos[b] = kv_len[b] - 1 the
 * call gives wpattn_decode's output bit for bit.
 */
WPATTN_API int wpattn_decode_positions(const wpattn_window *w,
                  const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *kv_len_host, int64_t Lmax,
                  const int32_t *q_pos_host, const int32_t *k_pos, int64_t k_pos_stride,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * Decode from a paged KV cache (the page-table layout serving engines use;
 * not a layout of the pages, whose decode reads a contiguous cache).
 *   k_pages, v_pages: bf16 device pools [num_pages, page_size, Hkv, D],
 *               16-byte aligned.
 *   page_size:  8, 16 or a multiple of 32 (else WPATTN_EUNSUPPORTED).
 *   block_table: device int32 [B, max_pages_per_seq], 4-byte aligned: cache
 *               row j of sequence b is row j % page_size of page
 *               block_table[b * max_pages_per_seq + j / page_size].  Only the
 *               entries that cover rows j < kv_len[b] are read.  An entry
 *               outside [0, num_pages) is an error found on the device: page
 *               0 is read in its place and WPATTN_EINDEX is recorded.
 *   kv_len_host: host int32 [B], 1 <= kv_len <= max_pages_per_seq * page_size.
 *   q_pos_host, k_pos, k_pos_stride: both null (keys at 0..kv_len-1, query at
 *               kv_len-1) or both given, as for wpattn_decode_positions
 *               (k_pos is indexed by the logical row j, not by page).
 * The workspace is sized by wpattn_decode_workspace_size with max_kv_len =
 * max_pages_per_seq * page_size.  Result and errors as for wpattn_decode; the
 * output equals, bit for bit, that of wpattn_decode (or
 * wpattn_decode_positions) on the [B, max_pages_per_seq * page_size, Hkv, D]
 * cache gathered through the block table.
 */
WPATTN_API int wpattn_decode_paged(const wpattn_window *w,
                  const void *q, const void *k_pages, const void *v_pages,
                  int32_t num_pages, int32_t page_size,
                  const int32_t *block_table, int32_t max_pages_per_seq,
                  const int32_t *kv_len_host, const int32_t *q_pos_host,
                  const int32_t *k_pos, int64_t k_pos_stride,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * RoPE rotation (WavePrune, Original abstract: each 2-D channel of a query or
 * key turns at a channel-specific frequency).  Pair p = dims (p, p + D/2)
 * turns by pos * theta_p, theta_p = rope_base^(-2p/D):
 *   y_p = x_p cos - x_{p+D/2} sin,   y_{p+D/2} = x_p sin + x_{p+D/2} cos.
 *   x, out: bf16 device [B, N, H, head_dim], 16-byte aligned; out may be x.
 *   positions: device int32 [B, N] (4-byte aligned), or NULL: token t of
 *              every sequence at pos0 + t (0 <= pos0 <= 2^40).
 * The angle is reduced modulo 2 pi in double precision, its cosine and sine
 * taken in float; each rotated value is rounded to bf16 (nearest even).
 * head_dim in {64, 128} (else WPATTN_EUNSUPPORTED); rope_base > 1.
 */
WPATTN_API int wpattn_rope(const void *x, void *out, int32_t B, int32_t N, int32_t H,
                  int32_t head_dim, int64_t pos0, const int32_t *positions, double rope_base,
                  void *cuda_stream);

/*
 * The RoPE rotation of a prefill's queries and keys in one launch: q
 * [B, Nq, Hq, head_dim] at positions q_pos0 + t into q_out, and k
 * [B, Nk, Hkv, head_dim] at k_pos0 + j into k_out, each exactly as
 * wpattn_rope would turn it (same rounding, same result bit for bit).
 *   q, q_out, k, k_out: bf16 device, 16-byte aligned; q_out may be q and
 *                       k_out may be k.  Nk = 0 turns q alone (k, k_out unused).
 *   0 <= q_pos0, k_pos0 <= 2^40.
 * head_dim in {64, 128} (else WPATTN_EUNSUPPORTED); rope_base > 1.
 */
WPATTN_API int wpattn_rope_qk(const void *q, void *q_out, const void *k, void *k_out,
                  int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                  int32_t head_dim, int64_t q_pos0, int64_t k_pos0, double rope_base,
                  void *cuda_stream);

/*
 * Prefill from queries and keys that arrive before their RoPE rotation
 * (v is never rotated).  Arguments and results as for wpattn_prefill; q and
 * k are rotated with w->rope_base at their positions q_pos0 + t and
 * k_pos0 + j (wpattn_rope_qk, one launch), into the workspace, then attended.  The rotation
 * is a pre-pass rather than part of the attention kernel's producer: there
 * each key tile would be turned again by every query block that reads it,
 * on the special-function pipe the attention's exponentials already fill.
 *   workspace: device, 256-byte aligned, at least
 *              wpattn_prefill_rope_workspace_size(...) bytes (else
 *              WPATTN_EWORKSPACE); holds the rotated q and k.
 */
WPATTN_API int wpattn_prefill_rope(const wpattn_window *w,
                  const void *q, const void *k, const void *v,
                  void *out, float *lse,
                  int32_t B, int32_t Nq, int32_t Nk, int32_t Hq, int32_t Hkv,
                  int64_t q_pos0, int64_t k_pos0, float softmax_scale,
                  void *workspace, size_t workspace_bytes, void *cuda_stream);

/* Workspace bytes wpattn_prefill_rope needs (0 on bad arguments). */
WPATTN_API size_t wpattn_prefill_rope_workspace_size(int32_t B, int32_t Nq, int32_t Nk,
                  int32_t Hq, int32_t Hkv, int32_t head_dim);

/*
 * Decode with the query before its RoPE rotation: the kernel turns q by its
 * position (q_pos, kv_len - 1 by default) with w->rope_base as it loads it,
 * rounding to bf16 exactly as wpattn_rope does, so the result equals
 * wpattn_rope followed by wpattn_decode (or wpattn_decode_positions) bit for
 * bit.  The cache holds rotated keys, as serving caches do.  q_pos_host,
 * k_pos, k_pos_stride: both NULL, or both given as for
 * wpattn_decode_positions.  Everything else as for wpattn_decode.
 */
WPATTN_API int wpattn_decode_rope(const wpattn_window *w,
                  const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *kv_len_host, int64_t Lmax,
                  const int32_t *q_pos_host, const int32_t *k_pos, int64_t k_pos_stride,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * One shard of a decode whose KV cache is split by length across devices
 * (each device holds a contiguous range of every sequence's keys).  The call
 * attends the query to the shard's keys only and returns the result
 * normalised over them, with its log-sum-exp; wpattn_merge_lse then combines
 * the shards' results into the decode over the whole cache (exactly, up to
 * rounding: each shard's part enters with weight exp(lse_shard - lse)).
 *   k_shard, v_shard: bf16 device [B, Lmax, Hkv, D], the shard's keys.
 *   kv_len_host: host int32 [B], keys of each sequence in this shard,
 *                0 <= kv_len <= Lmax (0: the shard has none of them).
 *   q_pos_host:  host int64 [B], position of each query in the whole cache.
 *   k_pos0_host: host int64 [B], position of the shard's first key of each
 *                sequence; its key j sits at k_pos0 + j.  Every key of the
 *                shard must be at or before the query (else WPATTN_EINVAL).
 *   lse: required.  A sequence with no key in the shard gets out = 0 and
 *        lse = -inf.  Workspace and the remaining arguments as for
 *        wpattn_decode (size it with the shard's Lmax).
 */
WPATTN_API int wpattn_decode_shard(const wpattn_window *w,
                  const void *q, const void *k_shard, const void *v_shard,
                  const int32_t *kv_len_host, int64_t Lmax,
                  const int64_t *q_pos_host, const int64_t *k_pos0_host,
                  int32_t B, int32_t Hq, int32_t Hkv, float softmax_scale,
                  void *out, float *lse,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/*
 * Combine R partial attention results of the same rows:
 *   outs: bf16 device [R, rows, head_dim], each normalised over its keys;
 *   lses: fp32 device [R, rows], natural-log sum-exp of each part (-inf: no key);
 *   out:  bf16 device [rows, head_dim];  lse: fp32 device [rows] or NULL.
 * out = sum_r w_r outs_r / sum_r w_r with w_r = exp(lses_r - max_r lses_r);
 * lse = max + ln(sum_r w_r).  A row whose parts are all empty gets 0 and
 * -inf.  head_dim in {64, 128}.  Asynchronous on `cuda_stream`.
 */
WPATTN_API int wpattn_merge_lse(const void *outs, const float *lses, int32_t R, int64_t rows,
                  int32_t head_dim, void *out, float *lse, void *cuda_stream);

/*
 * Synchronises `cuda_stream`, then reads and clears the current device's
 * kernel status word.  Returns WPATTN_OK, WPATTN_ETIMEOUT (a kernel gave up a
 * bounded wait; its outputs are undefined), WPATTN_EINDEX (a kernel met an
 * out-of-range device-side index; its outputs are undefined) or WPATTN_ECUDA.
 */
WPATTN_API int wpattn_device_status(void *cuda_stream);

/*
 * Self-check of the failure path that every kernel's waits share (the pages
 * have no counterpart).  Launches one CTA on `cuda_stream` whose only waiting
 * thread waits on a shared-memory mbarrier that nothing ever arrives at.  The
 * wait is bounded like every wait in the library's kernels (2 s on the
 * device's global timer); when the bound runs out the thread records
 * WPATTN_ETIMEOUT in the device status word and the kernel returns normally,
 * so the CUDA context stays usable.  The next wpattn_device_status on the
 * device returns WPATTN_ETIMEOUT (and clears it).  Returns WPATTN_OK once
 * launched, WPATTN_EUNSUPPORTED off sm_100, WPATTN_ECUDA on a launch error.
 */
WPATTN_API int wpattn_selftest_wait_timeout(void *cuda_stream);

/* Static English text for a status code. */
WPATTN_API const char *wpattn_strerror(int code);

/* Library version as "major.minor.patch". */
WPATTN_API const char *wpattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WPATTN_H */
