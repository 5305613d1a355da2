/*
 * attn.h -- C ABI of libattn_b200.so: fused grouped-KV scaled-dot-product
 * attention forward on NVIDIA B200 (sm_100a).
 *
 * The operation (all entry points):
 *   For batch b, query head h, query row i, with G = n_q / n_kv and the
 *   key/value head g = floor(h / G):
 *     s_j = scale * <q[b,h,i,:], k[b,g,j,:]>   for the visible keys j
 *     O[b,h,i,:] = sum_j softmax_j(s) v[b,g,j,:]
 *     LSE[b,h,i] = ln sum_j exp(s_j)          (natural log, scaled scores)
 *   Sources: "Attention, Worked Out by Hand (Part 2)" (j33.ai), "The recap"
 *   (score, scale, mask, softmax, mix); "Attention Engineering: From MHA to
 *   GQA, MLA & FlashAttention" (arman1o1.github.io), section 2 (Grouped-Query
 *   Attention Formulation: G query heads share one K/V head) and section 4
 *   (the online-softmax recurrence and the per-row log-sum-exp L = m + log l);
 *   "2.4 Multi-Head Attention, MQA, GQA & MLA" (llm-stack-book), "Implementing
 *   the MHA -> GQA conversion" (query head j reads KV head j // n_rep).
 *   MQA is n_kv = 1; MHA is n_kv = n_q.
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers of the current CUDA device; the caller
 *     owns and allocates every buffer (the library never allocates, frees or
 *     keeps a pointer after the call returns).
 *   - bf16 tensors are IEEE bfloat16 stored as 16-bit words; LSE is fp32.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; 0 is
 *     the legacy default stream). Nothing on the hot path synchronises.
 *   - Argument errors are returned synchronously and nothing is launched.
 *     Errors found on the device (a bounded wait that expired, a seqlen out
 *     of range) are recorded in a per-device status word that
 *     attn_device_status() reads.
 *   - Every base pointer must be 16-byte aligned and every row stride a
 *     multiple of 8 elements (16 bytes): the kernels move tiles with the
 *     Tensor Memory Accelerator, which requires it.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared here without the CUDA headers. */
typedef struct CUstream_st *attn_stream_t;

/* Status codes. */
enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1,   /* null pointer, bad size, n_q % n_kv != 0, bad scale/causal */
    ATTN_ERR_UNSUPPORTED = -2,   /* head dims outside the compiled set; causal with Sq > Skv */
    ATTN_ERR_MISALIGNED = -3,    /* pointer not 16-byte aligned or stride not a multiple of 8 */
    ATTN_ERR_WORKSPACE = -4,     /* workspace missing or smaller than attn_decode_workspace_bytes */
    ATTN_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed (e.g. launch error) */
    ATTN_ERR_DEVICE_TIMEOUT = -6,/* a kernel's bounded wait expired (reported by attn_device_status) */
    ATTN_ERR_DEVICE_RANGE = -7   /* a device-side value (seqlens[b]) was out of range and clamped */
};

/*
 * attn_fwd -- prefill / full forward.
 *
 *   q   [B, n_q,  Sq,  d_qk] bf16, contiguous (BHSD)
 *   k   [B, n_kv, Skv, d_qk] bf16, contiguous
 *   v   [B, n_kv, Skv, d_v ] bf16, contiguous
 *   o   [B, n_q,  Sq,  d_v ] bf16, contiguous (written)
 *   lse [B, n_q,  Sq]        fp32, contiguous (written; may be NULL to skip)
 *   causal: 0 = every key visible; 1 = key j visible to query row i iff
 *     j <= i + (Skv - Sq) (the query rows are the last Sq positions; for
 *     Sq == Skv this is the usual lower-triangular mask).
 *   scale: multiplies q.k before the softmax (finite, > 0; 1/sqrt(d_qk) is
 *     the usual choice).
 * Supported: d_qk == d_v in {32, 64, 128}; any B >= 0, Sq >= 0, Skv >= 1,
 * any n_kv dividing n_q with n_q / n_kv a power of two <= 256; causal needs
 * Sq <= Skv. Output rows are bf16 rounded to nearest even.
 * Returns ATTN_OK or an error code (nothing launched on error).
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int Sq, int Skv, int n_q, int n_kv, int d_qk, int d_v,
             int causal, float scale, attn_stream_t stream);

/*
 * attn_fwd_fp8 -- attn_fwd on FP8 (e4m3) queries, keys and values with one
 * scale per 128-row tile.
 * Source: "Flash Attention 3 and Multi-Headed Latent Attention", FP8 section
 * (e4m3 operands, largest finite 448, with scaling factors per tile).
 *
 *   q8  [B, n_q,  Sq,  d] e4m3 bytes, contiguous (BHSD)
 *   k8  [B, n_kv, Skv, d] e4m3 bytes, contiguous
 *   v8  [B, n_kv, Skv, d] e4m3 bytes, contiguous
 *   q_scale [B, n_q,  ceil(Sq / 128)]  fp32: row i of (b, h) means
 *           e4m3(q8[b][h][i]) * q_scale[b][h][i / 128]
 *   k_scale, v_scale [B, n_kv, ceil(Skv / 128)] fp32, likewise for keys and
 *           values (finite and > 0; other values give undefined results)
 *   o, lse, causal, scale: as attn_fwd (o bf16, lse fp32 natural log)
 *   workspace: device scratch of at least attn_fwd_fp8_workspace_bytes(...)
 *           bytes, 256-byte aligned, contents on entry irrelevant; calls that
 *           share it must be ordered on one stream.
 * The result is attn_fwd of the dequantised operands. Computed as: the
 * e4m3 keys and values widened to bf16 into the workspace (exact: every
 * e4m3 value is a bf16 value), then the attention kernel, which loads the
 * e4m3 query tiles and widens them in shared memory, folds the query and
 * key tile scales into each score tile's exponent scale and the value
 * tile's scale into P (the row sums take P unscaled). Two launches on
 * `stream`, the second a programmatic dependent of the first (its prologue
 * and query tiles overlap the widening of the keys and values).
 * Supported: d == 128, and the rest as attn_fwd.
 * Returns ATTN_OK or an error code (nothing launched on error).
 */
int attn_fwd_fp8_workspace_bytes(int B, int Sq, int Skv, int n_q, int n_kv, int d, size_t *bytes);
int attn_fwd_fp8(const void *q8, const void *k8, const void *v8,
                 const float *q_scale, const float *k_scale, const float *v_scale,
                 void *o, float *lse, int B, int Sq, int Skv, int n_q, int n_kv, int d,
                 int causal, float scale, void *workspace, size_t workspace_bytes,
                 attn_stream_t stream);

/*
 * attn_fwd_window -- causal attn_fwd with a sliding window and sink keys.
 * Source: "Attention deep dive" (askaiml.pages.dev), section 6 (sliding-window
 * attention: token i attends to the last W tokens, mask (j <= i) AND
 * (i - j < W)); "Attention Engineering: From MHA to GQA, MLA &
 * FlashAttention", section 5, failure mode 2 (keep the first tokens as
 * permanent attention sinks in a rolling window).
 * Layouts, outputs and errors as attn_fwd, with causal fixed: a query at
 * position p = i + (Skv - Sq) sees key j iff j <= p and (p - j < window or
 * j < n_sink). Key tiles that hold neither window nor sink keys of a query
 * tile are never loaded.
 * Supported: as attn_fwd with causal = 1 (Sq <= Skv); window >= 1,
 * n_sink >= 0 (0: no sinks).
 */
int attn_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                    int B, int Sq, int Skv, int n_q, int n_kv, int d_qk, int d_v,
                    int window, int n_sink, float scale, attn_stream_t stream);

/*
 * attn_fwd_varlen -- attn_fwd over a packed batch of sequences of different
 * lengths (no padding). Source: "Attention deep dive" (askaiml.pages.dev),
 * section 5 (engines batch sequences of different lengths); each sequence is
 * attended exactly as attn_fwd attends one batch element.
 *
 *   q   [total_q, n_q,  d_qk] bf16, contiguous (tokens of all sequences, packed)
 *   k   [total_k, n_kv, d_qk] bf16, contiguous
 *   v   [total_k, n_kv, d_v ] bf16, contiguous
 *   o   [total_q, n_q,  d_v ] bf16 (written)
 *   lse [n_q, total_q] fp32 (written; may be NULL)
 *   cu_seqlens_q, cu_seqlens_k: [B + 1] int32 on the device, non-decreasing
 *     offsets: sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *     and key rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1.
 *   max_seqlen_q: an upper bound of every sequence's query count (sizes the
 *     grid).
 *   causal: per sequence, query i sees key j iff j <= i + (Skv_b - Sq_b); a
 *     row that sees no key (Sq_b > Skv_b, or Skv_b = 0) gets O = 0, LSE = -inf.
 * A sequence whose offsets are negative, decreasing, past total_q / total_k or
 * longer than max_seqlen_q is skipped (its outputs are left as they were) and
 * reported as ATTN_ERR_DEVICE_RANGE by attn_device_status.
 * Supported: d_qk == d_v in {32, 64, 128}; n_q / n_kv a power of two <= 256;
 * B <= 65535. Returns ATTN_OK or an error code (nothing launched on error).
 */
int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                    int B, int max_seqlen_q, int total_q, int total_k,
                    int n_q, int n_kv, int d_qk, int d_v, int causal, float scale, attn_stream_t stream);

/*
 * attn_decode_workspace_bytes -- scratch size attn_decode needs for these
 * sizes (split-KV partial outputs and their softmax statistics). Writes the
 * byte count to *bytes. The split of the cached keys into chunks is planned
 * from the sizes and the SM count of the CURRENT device (a small batch is
 * cut into more chunks so that it spreads over every SM), so the answer is
 * the same for the same sizes on the same device; ask with the device
 * current that the decode will run on. (d_qk selects the shape family: the
 * (576, 512) MLA form needs no workspace.)
 */
int attn_decode_workspace_bytes(int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                                size_t *bytes);

/*
 * attn_decode -- one query token per sequence against a KV cache.
 * Source: "Attention deep dive" (askaiml.pages.dev), section 5 (the KV cache:
 * the new token's query against every cached key and value); "2.4 Multi-Head
 * Attention, MQA, GQA & MLA", exercise decode_step (is_causal=False for the
 * lone query: every cached key is visible).
 *
 *   q       [B, n_q, d_qk] bf16, contiguous
 *   kcache  element (b, g, j, c) at kcache[b*k_stride_b + g*k_stride_h + j*k_stride_s + c]
 *   vcache  element (b, g, j, c) at vcache[b*v_stride_b + g*v_stride_h + j*v_stride_s + c]
 *           (strides in ELEMENTS; kcache and vcache may alias: the MLA latent
 *           cache passes the same pointer, the 576-wide row as key and its
 *           first 512 columns as value)
 *   seqlens [B] int32: keys 0 .. seqlens[b]-1 of sequence b are visible
 *           (values above S_max are clamped and reported as
 *           ATTN_ERR_DEVICE_RANGE; 0 gives O = 0 and LSE = -inf)
 *   o       [B, n_q, d_v] bf16 (written); lse [B, n_q] fp32 (written; may be NULL)
 *   workspace: device scratch of at least attn_decode_workspace_bytes(...)
 *           bytes, 256-byte aligned; its contents on entry do not matter.
 *           Calls that share a workspace must be ordered on one stream.
 *           (128, 128): split-KV partial outputs and statistics; (576, 512):
 *           the same for the key chunks when the batch is too small to fill
 *           the GPU by whole sequences, and none otherwise (0 bytes; the
 *           pointer may then be NULL).
 * Supported: (d_qk, d_v) = (128, 128) with n_q / n_kv in {1, 2, 4, 8, 16, ...}
 * (any power of two); (576, 512) with n_kv = 1 (MLA absorbed decode, the
 * scale usually 1/sqrt(128 + 64)). Cache rows at or past a sequence's length
 * may hold anything (NaN and Inf included): they never reach the result.
 */
int attn_decode(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                void *o, float *lse,
                int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                float scale, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_window -- attn_decode with a sliding window and sink keys.
 * Source: "Attention deep dive" (askaiml.pages.dev), section 6 (each token
 * attends only to the last W tokens); "Attention Engineering" section 5,
 * failure mode 2 (the first tokens stay as attention sinks). For a sequence
 * of length L the visible keys are L-window .. L-1 and 0 .. n_sink-1; key
 * chunks holding neither are not read. Arguments, layouts, workspace and
 * errors as attn_decode; window >= 1, n_sink >= 0. Supported: (d_qk, d_v) =
 * (128, 128).
 */
int attn_decode_window(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                       void *o, float *lse,
                       int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                       int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                       int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                       int window, int n_sink, float scale,
                       void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_fp8 -- attn_decode against an FP8 (e4m3) KV cache with one
 * scale per KV head. Source: "Flash Attention 3 and Multi-Headed Latent
 * Attention" (misar.blog), FP8 section (8-bit e4m3 operands with scaling
 * factors), and "Attention deep dive" (askaiml.pages.dev), section 5
 * (quantized FP8 / INT8 KV caches halve KV memory).
 *
 *   q        [B, n_q, 128] bf16, contiguous (|q| < 65504: the scores are
 *            computed in f16 x f16 products with fp32 accumulation)
 *   kcache, vcache: one byte per element (e4m3: 1 sign, 4 exponent, 3
 *            mantissa bits, bias 7, no infinities); element (b, g, j, c) at
 *            byte offset b*stride_b + g*stride_h + j*stride_s + c (strides in
 *            ELEMENTS = bytes, multiples of 16, stride_s >= 128)
 *   k_scale, v_scale: [n_kv] fp32 on the device; key (b, g, j) is
 *            e4m3(bytes) * k_scale[g], value likewise with v_scale[g]
 *   seqlens, o, lse, scale: as attn_decode
 *   workspace: at least attn_decode_fp8_workspace_bytes(...) bytes, 256-byte
 *            aligned, caller-owned.
 * The result is attention over the dequantized cache (the e4m3 values times
 * their scales), computed exactly as attn_decode computes it for a bf16
 * cache; half the bytes cross HBM. Supported: head dim 128, n_q / n_kv a
 * power of two. Returns ATTN_OK or an error code (nothing launched on
 * error). attn_decode_fp8_workspace_bytes plans the key chunks as
 * attn_decode_workspace_bytes does (sizes and the current device's SM count).
 */
int attn_decode_fp8_workspace_bytes(int B, int n_q, int n_kv, int S_max, size_t *bytes);
int attn_decode_fp8(const void *q, const void *kcache, const void *vcache, const float *k_scale,
                    const float *v_scale, const int32_t *seqlens, void *o, float *lse,
                    int B, int n_q, int n_kv, int S_max,
                    int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                    int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                    float scale, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_fp8_tiles -- attn_decode_fp8 with one key scale and one value
 * scale per 128-key tile of each (sequence, KV head) instead of per KV head.
 * Source: "Flash Attention 3 and Multi-Headed Latent Attention"
 * (misar.blog), FP8 section (e4m3 operands with per-tile scaling factors).
 *
 *   k_scales, v_scales: [B, n_kv, ceil(S_max / 128)] fp32 on the device,
 *            contiguous; key j of (b, g) is e4m3(bytes) * k_scales[b, g, j / 128],
 *            value likewise with v_scales (finite, > 0)
 *   every other argument, the workspace (attn_decode_fp8_workspace_bytes)
 *   and the error behaviour as attn_decode_fp8.
 * The key scale of a tile multiplies its scores, the value scale the
 * softmax weights of its keys before they meet the values (so the weights
 * stay below the value scale in f16); the row sums take the unscaled
 * weights.
 */
int attn_decode_fp8_tiles(const void *q, const void *kcache, const void *vcache, const float *k_scales,
                          const float *v_scales, const int32_t *seqlens, void *o, float *lse,
                          int B, int n_q, int n_kv, int S_max,
                          int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                          int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                          float scale, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_paged -- attn_decode against a paged KV cache.
 * Source: "Attention deep dive" (askaiml.pages.dev), section 5 (production
 * engines keep the KV cache in fixed-size pages addressed through a page
 * table, so sequences of different lengths share one pool); "2.4 Multi-Head
 * Attention, MQA, GQA & MLA", GQA in libraries (serving engines size their
 * paged KV blocks by the number of KV heads). The attention computed is that
 * of attn_decode; only where cached token j of sequence b lives changes.
 *
 *   q        [B, n_q, 128] bf16, contiguous
 *   k_pages  element (page p, token t of the page, kv head g, dim c) at
 *            k_pages[p*k_stride_page + t*k_stride_token + g*k_stride_head + c]
 *            (strides in ELEMENTS, multiples of 8, token stride >= 128; the
 *            common pool layout [num_pages][page_size][n_kv][128] has strides
 *            (page_size*n_kv*128, n_kv*128, 128))
 *   v_pages  the same for values (may alias k_pages with other strides)
 *   block_table [B, pages_per_seq] int32, device: logical token j of
 *            sequence b is token j % page_size of page
 *            block_table[b*pages_per_seq + j / page_size]. Only the entries
 *            covering tokens 0 .. seqlens[b]-1 are read. A page id outside
 *            [0, num_pages) reads as zeros and is reported as
 *            ATTN_ERR_DEVICE_RANGE (by attn_device_status).
 *   seqlens  [B] int32, device; values above pages_per_seq*page_size are
 *            clamped (reported as ATTN_ERR_DEVICE_RANGE); 0 gives O = 0,
 *            LSE = -inf
 *   o, lse   as attn_decode
 *   workspace: at least attn_decode_workspace_bytes(B, n_q, n_kv, 128, 128,
 *            pages_per_seq * page_size) bytes, 256-byte aligned, caller-owned.
 * Supported: d_qk = d_v = 128, n_q / n_kv a power of two, page_size in
 * {16, 32, 64} or a power of two that is a multiple of 128. Cache rows past a
 * sequence's length may hold anything (NaN and Inf included): they never
 * reach the result. Returns ATTN_OK or an error code (nothing launched on
 * error).
 */
int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *block_table,
                      const int32_t *seqlens, void *o, float *lse,
                      int B, int n_q, int n_kv, int d_qk, int d_v,
                      int page_size, int pages_per_seq, int num_pages,
                      int64_t k_stride_page, int64_t k_stride_token, int64_t k_stride_head,
                      int64_t v_stride_page, int64_t v_stride_token, int64_t v_stride_head,
                      float scale, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_fwd_paged -- prefill (or chunked prefill) of a packed batch whose keys
 * and values live in a paged KV cache. Source: "Attention deep dive"
 * (askaiml.pages.dev), section 5 (production engines keep the KV cache in
 * fixed-size pages addressed through a page table, and batch sequences of
 * different lengths); the attention of each sequence is that of attn_fwd_varlen
 * over its first seqlens_k[b] cached tokens, only where those tokens live
 * changes. The cached tokens include the new ones (the caller writes the new
 * keys and values into the cache before the call), so a chunk of Sq_b new
 * queries sits at the end of its sequence: query i of sequence b is position
 * seqlens_k[b] - Sq_b + i.
 *
 *   q            [total_q, n_q, d_qk] bf16, contiguous (the queries of all
 *                sequences, packed); o [total_q, n_q, d_v] bf16 (written);
 *                lse [n_q, total_q] fp32 (written; may be NULL)
 *   cu_seqlens_q [B + 1] int32 on the device: sequence b owns query rows
 *                cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 (non-decreasing)
 *   seqlens_k    [B] int32 on the device: cached tokens of sequence b
 *                (values above pages_per_seq * page_size are clamped and
 *                reported as ATTN_ERR_DEVICE_RANGE by attn_device_status)
 *   k_pages, v_pages, block_table, page_size, pages_per_seq, num_pages and
 *                the page / token / head strides (in ELEMENTS): as for
 *                attn_decode_paged (head dim d_qk = d_v instead of 128; token
 *                stride >= d). Only table entries of tokens below seqlens_k[b]
 *                are read; a page id outside [0, num_pages) reads as zeros
 *                and is reported as ATTN_ERR_DEVICE_RANGE.
 *   max_seqlen_q an upper bound of every Sq_b (sizes the grid).
 *   causal       query i sees key j iff j <= i + (seqlens_k[b] - Sq_b); a row
 *                that sees no key gets O = 0, LSE = -inf.
 * Supported: d_qk == d_v in {32, 64, 128}; n_q / n_kv a power of two <= 256;
 * page_size 16, 32, 64 or a power of two >= 128; B <= 65535. Malformed
 * cu_seqlens_q entries skip the sequence and are reported as
 * ATTN_ERR_DEVICE_RANGE. Returns ATTN_OK or an error code (nothing launched
 * on error).
 */
int attn_fwd_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *block_table,
                   const int32_t *cu_seqlens_q, const int32_t *seqlens_k, void *o, float *lse,
                   int B, int max_seqlen_q, int total_q, int n_q, int n_kv, int d_qk, int d_v,
                   int page_size, int pages_per_seq, int num_pages,
                   int64_t k_stride_page, int64_t k_stride_token, int64_t k_stride_head,
                   int64_t v_stride_page, int64_t v_stride_token, int64_t v_stride_head,
                   int causal, float scale, attn_stream_t stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device
 * memory.
 *
 * This entry point has no counterpart in the pages the method comes from; it
 * exists for the library's users. Some callers of a decode step cannot call
 * cudaMalloc or any allocator: a plugin running inside another framework that
 * owns every device allocation, a real-time serving loop that must not take
 * the allocator's locks or implicit synchronisation, or host code that has no
 * device allocator at all. They cannot provide attn_decode's workspace, so this
 * variant uses a scratch array that the library itself holds in device memory
 * (a file-scope __device__ array of ATTN_NOALLOC_SCRATCH_BYTES bytes, present
 * on every GPU that loads the library until the process exits).
 *
 * Arguments and results are those of attn_decode without the workspace.
 * Sizes whose scratch need (attn_decode_workspace_bytes) exceeds
 * ATTN_NOALLOC_SCRATCH_BYTES are rejected with ATTN_ERR_WORKSPACE, before
 * anything is launched. Supported shapes: the (128, 128) head dims of
 * attn_decode.
 *
 * The first call on a device looks up that device's address of the scratch
 * array (cudaGetSymbolAddress); make that first call before any stream
 * capture on the device. Nothing is allocated or freed, then or later.
 * The address is kept per device together with the CUDA context it belongs
 * to; after a cudaDeviceReset (a new primary context, in which the library's
 * module and the array are loaded again) the next call looks it up anew, so
 * that first call after a reset should also come before any capture.
 * All calls share the one array and it keeps the previous call's contents;
 * no part of it needs to start at zero (every value read is written earlier
 * in the same call). Calls that overlap on the GPU (on different streams, or
 * from several host threads without ordering) race on the array: order them
 * on one stream.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (36u * 1024u * 1024u)

int attn_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                        void *o, float *lse,
                        int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                        int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                        int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                        float scale, attn_stream_t stream);

/*
 * Rotary position embedding (RoPE).
 * Source: "Attention Engineering: From MHA to GQA, MLA & FlashAttention",
 * section 1 (Rotary Position Embeddings: the head dimension is split into
 * d/2 planes (x_{2j}, x_{2j+1}); at position m plane j is turned by the
 * angle m * theta_j, theta_j = base^(-2j/d), i.e. multiplied by the 2x2
 * rotation [[cos, -sin], [sin, cos]]; the angles are kept in cos/sin tables
 * of shape [positions, d/2]) and section 2 (the GQA formulation applies it
 * to the queries and the keys before the scores; values are not rotated).
 *
 * Tables: cos, sin [n_pos, d/2] fp32 on the device, 16-byte aligned, row m
 * holding cos(m theta_j) and sin(m theta_j).
 */

/*
 * attn_rope_tables -- fill cos/sin [n_pos, d/2] for the given base (10000 in
 * the original RoPE, 500000 in Llama-3). Angles in fp64, rounded once to
 * fp32. d even, n_pos >= 0, base finite and > 0. Asynchronous on `stream`.
 */
int attn_rope_tables(float *cos, float *sin, int n_pos, int d, double base, attn_stream_t stream);

/*
 * attn_rope_apply -- y = RoPE(x): x, y [B, H, S, d] bf16 contiguous (y may be
 * x: rotated in place); row (b, h, s) sits at position pos0 + s, and
 * pos0 + S <= n_pos. Computed in fp32, rounded once to bf16 (nearest even).
 * This is how keys enter a KV cache in rotated form. d a multiple of 8.
 */
int attn_rope_apply(const void *x, void *y, int B, int H, int S, int d, int pos0,
                    const float *cos, const float *sin, int n_pos, attn_stream_t stream);

/*
 * attn_fwd_rope -- attn_fwd on rotated queries and keys:
 *   O = softmax(scale * RoPE(Q) RoPE(K)^T + mask) V
 * with key j at position j and query row i at position i + (Skv - Sq) (the
 * alignment of the causal mask). q, k, v, o, lse, causal, scale as attn_fwd
 * (q and k are given unrotated). The keys are rotated once into k_rot
 * ([B, n_kv, Skv, d_qk] bf16, caller-owned, written; it may be k itself,
 * which is then overwritten): each key tile is read by every query tile of
 * its group, so it is rotated by one bandwidth-bound pass rather than in
 * each of them. The queries are rotated inside the attention kernel, in
 * shared memory, before their first score MMA. Rotated values are rounded
 * to bf16 before the MMAs (the precision of the tensor-core operands).
 * Supported: as attn_fwd, plus Sq <= Skv <= n_pos. Two launches on `stream`.
 */
int attn_fwd_rope(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int Sq, int Skv, int n_q, int n_kv, int d_qk, int d_v,
                  int causal, float scale, const float *cos, const float *sin, int n_pos,
                  void *k_rot, attn_stream_t stream);

/*
 * attn_decode_rope -- attn_decode (head dim 128) with the query rotated at
 * position seqlens[b] - 1 (the new token is the last one in the cache),
 * inside the kernel before its score MMAs. The cache holds keys that were
 * rotated when they were written (attn_rope_apply), as the KV cache of a
 * RoPE model does. Arguments as attn_decode plus the tables; a length above
 * n_pos uses the last table row and raises ATTN_ERR_DEVICE_RANGE in
 * attn_device_status. The MLA shape is not supported here.
 */
int attn_decode_rope(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                     void *o, float *lse, int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                     int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                     int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s,
                     const float *cos, const float *sin, int n_pos, float scale,
                     void *workspace, size_t workspace_bytes, attn_stream_t stream);

/* Human-readable text of a status code (static storage). */
const char *attn_status_string(int status);

/*
 * attn_device_status -- synchronise `stream`, then read and clear the status
 * word of the current device. Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT (a
 * kernel's bounded wait expired; its outputs are invalid), ATTN_ERR_DEVICE_RANGE,
 * or ATTN_ERR_CUDA if the synchronisation itself failed.
 * The status word is one per DEVICE, not per stream: it collects the errors of
 * every kernel of this library on the device, whatever stream launched it,
 * and only `stream` is synchronised first. With work in flight on other
 * streams, an error of one of their kernels may be reported to (and cleared
 * by) this call, or land after it; callers that need per-stream attribution
 * must synchronise those streams too before calling.
 */
int attn_device_status(attn_stream_t stream);

/*
 * attn_selftest_timeout -- launch one small kernel that waits, with the
 * library's bounded-wait routine, on a barrier nothing will complete, giving
 * up after `timeout_us` microseconds (1 .. 1000000). It must end with the
 * status word set to ATTN_ERR_DEVICE_TIMEOUT: a test of the failure path that
 * faults and hangs nothing.
 */
int attn_selftest_timeout(int timeout_us, attn_stream_t stream);

/*
 * attn_selftest_ex2 -- evaluate, for n device floats x, the two base-2
 * exponentials the prefill softmax uses: y_poly = the FMA-pipe evaluation
 * (range reduction + a cubic fitted for relative error, inputs clamped at
 * -125) and y_sfu = the special-function unit's ex2.approx. For tests of the
 * kernels' exponential accuracy.
 */
int attn_selftest_ex2(const float *x, float *y_poly, float *y_sfu, int n, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
