/*
 * pkvq — attention over a paged, 8-bit-quantized KV cache, for NVIDIA B200
 * (sm_100a).  C ABI of libpkvq.so.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless a comment says otherwise.  The
 *     caller owns every buffer; the library allocates nothing, frees
 *     nothing, creates no stream and never synchronizes the host with the
 *     device.  All work is enqueued on `stream` (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).
 *   - Arguments are checked on the host before anything is launched; a
 *     failed check returns a status and launches nothing.  No C++ exception
 *     crosses this boundary.
 *   - Contract violations that only the device could see (a block id outside
 *     the pool, overlapping slots) are undefined behaviour unless the
 *     library was built with PKVQ_BOUNDS_CHECK, in which case the kernels
 *     skip the access and record it in a device status word read by
 *     pkvq_device_status().
 *   - Cache layout (a design choice; the pages only say that pages hold
 *     fixed-size token groups addressed by a page id): K and V codes are
 *     [num_blocks][num_kv_heads][block_size][head_dim] bytes, so one
 *     (block, KV head) is a contiguous block_size * head_dim byte tile.
 *     INT8 scales are fp16 [num_blocks][num_kv_heads][block_size].
 *   - Token j of sequence s lives at slot block_table[s][j / block_size] *
 *     block_size + j % block_size.
 *   - A query row (token t of q_len new tokens of a sequence whose context,
 *     new tokens included, is c) sits at position c - q_len + t and attends
 *     to keys 0..position.  A row that sees no key gets zeros and lse -inf.
 *   - GQA: query head h reads KV head h / (num_q_heads / num_kv_heads).
 */
#ifndef PKVQ_H
#define PKVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKVQ_API __attribute__((visibility("default")))
#else
#define PKVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKVQ_OK = 0,
    PKVQ_ERR_INVALID_ARG = 1,        /* null pointer, bad size or count */
    PKVQ_ERR_UNSUPPORTED = 2,        /* head_dim, block size or dtype not built */
    PKVQ_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
    PKVQ_ERR_WORKSPACE_TOO_SMALL = 4,
    PKVQ_ERR_DEVICE = 5,             /* a device-side check fired (see pkvq_device_status) */
    PKVQ_ERR_CUDA = 6                /* a CUDA runtime call failed */
} pkvq_status;

typedef enum {
    /* FP8 E4M3 (OCP "FN" variant: bias 7, no inf, S.1111.111 = NaN, max 448)
     * with one static fp32 scale per KV head for K and one for V.  Source:
     * "ReVolta" PyPI page, "E4M3 KV" (calibrated K/V scales; a missing scale
     * means 1.0, which the caller passes explicitly). */
    PKVQ_KV_FP8_E4M3 = 0,
    /* INT8 with one fp16 scale per (token, KV head), computed when the token
     * is written.  Source: "ReVolta" PyPI page, "INT8 KV" (scales computed per
     * token and head at run time, no calibration). */
    PKVQ_KV_INT8 = 1,
    /* FP8 E5M2 (bias 15, S.11111.00 = inf, S.11111.xx = NaN, max 57344) with
     * the same static fp32 scales as E4M3.  Source: "1Cat-LLM" README,
     * current SM70 work list ("FP8 E4M3 / E5M2 KV storage"). */
    PKVQ_KV_FP8_E5M2 = 2,
    /* The fp16 values themselves, no scale (2 bytes per element).  Source:
     * "ReVolta" PyPI page, first section ("KV formats: FP8 E4M3, FP16, and
     * INT8"). */
    PKVQ_KV_FP16 = 3
} pkvq_kv_dtype;

/* Describes caller-owned cache memory.  All pointers device, 16-byte aligned. */
typedef struct {
    int32_t dtype;          /* pkvq_kv_dtype */
    int32_t num_blocks;     /* blocks in the pool */
    int32_t block_size;     /* tokens per block: 16, 32 or 64 */
    int32_t num_kv_heads;
    int32_t head_dim;       /* must be 128 */
    void *k_cache;          /* [num_blocks][num_kv_heads][block_size][head_dim] elements:
                               1 byte (E4M3, E5M2, INT8) or 2 (FP16) */
    void *v_cache;
    const float *k_scale;   /* FP8 formats: fp32 [num_kv_heads] (or [1], see
                               scale_per_layer); INT8, FP16: unused (NULL) */
    const float *v_scale;
    void *k_scale_tok;      /* INT8: fp16 [num_blocks][num_kv_heads][block_size]; else NULL */
    void *v_scale_tok;
    int32_t scale_per_layer; /* FP8 formats: nonzero = k_scale and v_scale hold one value
                                each, shared by every KV head ("ReVolta" PyPI page, "E4M3
                                KV": one calibrated K and V scale per layer) */
} pkvq_cache;

/*
 * KV write + quantize.
 * Source: "ReVolta" PyPI page, "Weight and KV formats" (KV stored as 8-bit
 * codes), "E4M3 KV" (static per-layer scales; here per KV head) and "INT8 KV"
 * (per-token, per-head scales computed at run time).
 *
 * For every token i < num_tokens with slot_mapping[i] >= 0 and every KV head
 * h, writes row (slot / block_size, h, slot % block_size):
 *   E4M3: code[d] = E4M3_rn_satfinite(fp32(x[d]) / k_scale[h]) (scale 0 -> 0);
 *         NaN keeps its sign as S.1111.111, +-inf saturates to +-448.
 *   E5M2: the same with E5M2: NaN -> S.11111.11, +-inf saturates to +-57344.
 *   FP16: the fp16 bits of x as given.
 *   INT8: s = fp16_rn(fp32(max_d |x[d]|) / 127);
 *         code[d] = clamp(rint(fp32(x[d]) / fp32(s)), -127, 127), s == 0 -> 0;
 *         s is stored in k_scale_tok / v_scale_tok.  Inputs must be finite.
 * fp32 divisions are IEEE round-to-nearest; rint is ties-to-even.
 *   k, v          fp16 [num_tokens][num_kv_heads][head_dim], 16-byte aligned.
 *   slot_mapping  int32 [num_tokens]; negative entries are skipped.  Slots
 *                 must be < num_blocks * block_size and distinct.
 * num_tokens == 0 is a no-op.  Codes are bit-exact with the CPU oracle.
 */
PKVQ_API pkvq_status pkvq_kv_write_quant(const pkvq_cache *cache, const void *k, const void *v,
                                const int32_t *slot_mapping, int32_t num_tokens,
                                void *stream);

/*
 * Workspace bytes pkvq_paged_attn_decode needs for this shape on the
 * current device (split-KV partial states: fp32 O, max and sum per split).
 * Returns 0 on invalid arguments.  The same arguments give the same size and
 * the same split plan in pkvq_paged_attn_decode.
 */
PKVQ_API size_t pkvq_decode_workspace_bytes(int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, const pkvq_cache *cache);

/*
 * Decode / draft-verify attention: q_len (1..16) new tokens per sequence,
 * causal among themselves, over each sequence's paged context.
 * Source: "1Cat-LLM" README, "Layer 1" (paged KV read through page ids with
 * wide loads), "Layer 2" (GQA multi-head packing, online softmax with FP32
 * state, Split-KV with an FP32 merge of partial states); "ReVolta" PyPI page
 * (MTP4: 1 + 4 verify positions).
 *   q             fp16 [batch][q_len][num_q_heads][head_dim]
 *   out           fp16 [batch][q_len][num_q_heads][head_dim]
 *   lse_out       nullable fp32 [batch][q_len][num_q_heads]: natural-log
 *                 sum-exp of the scaled scores (-inf for an empty row)
 *   block_table   int32 [batch][max_blocks_per_seq]
 *   context_lens  int32 [batch]: cached tokens including the q_len new
 *                 ones, which must already be in the cache.  Each must be
 *                 <= max_context_len and <= max_blocks_per_seq * block_size.
 *   max_context_len  host-side upper bound of context_lens; sizes the split
 *                 plan (must match the value given to the workspace query).
 *                 The kernels split each sequence's tokens over CTAs in
 *                 proportion to its own context length, read on the device.
 *   softmax_scale scores are softmax_scale * q . k_dequantized.
 *   workspace     device scratch of at least pkvq_decode_workspace_bytes();
 *                 contents need not be initialised.  Calls that overlap on
 *                 the device must not share a workspace.
 * num_q_heads must be a multiple of num_kv_heads with a group of at most 16.
 * Up to 16 query rows per KV head (q_len x group) run on mma.sync tiles;
 * 17 to 128 rows run all rows of a KV head in one tcgen05 CTA.
 */
PKVQ_API pkvq_status pkvq_paged_attn_decode(const pkvq_cache *cache, const void *q, void *out,
                                   float *lse_out, const int32_t *block_table,
                                   int32_t max_blocks_per_seq, const int32_t *context_lens,
                                   int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, float softmax_scale,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode without a caller-provided workspace.  The pages have no counterpart:
 * this is an addition for callers that cannot allocate device memory (for
 * example an engine whose caching allocator already holds nearly all of HBM,
 * or a plugin whose host framework owns every allocation).
 * Same arguments, results and errors as pkvq_paged_attn_decode, minus the
 * workspace: the split-KV scratch is a fixed 8 MiB array compiled into the
 * library (held on every GPU that loads it, until exit).  Nothing is
 * allocated.  Shapes whose workspace (pkvq_decode_workspace_bytes) exceeds
 * 8 MiB return PKVQ_ERR_WORKSPACE_TOO_SMALL.  The first call on each device
 * looks up the array's device address; make that first call before any
 * stream capture.  All calls on a device share the array: calls that may
 * overlap on the device race and must be ordered by the caller.  The array
 * needs no clearing between calls.
 */
PKVQ_API pkvq_status pkvq_paged_attn_decode_noalloc(const pkvq_cache *cache, const void *q,
                                   void *out, float *lse_out, const int32_t *block_table,
                                   int32_t max_blocks_per_seq, const int32_t *context_lens,
                                   int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, float softmax_scale, void *stream);

/*
 * Causal (chunked) prefill over a cached prefix, varlen batch.
 * Source: "1Cat-LLM" README, "Layer 2" (causal online softmax with FP32
 * accumulation, prefix / causal-tail separation, wide QK/PV tensor-core
 * tiles); "ReVolta" PyPI page (chunked prefill with an 8,192-token budget).
 *   q             fp16 [total_q][num_q_heads][head_dim], sequences packed
 *   out           fp16 [total_q][num_q_heads][head_dim]
 *   lse_out       nullable fp32 [total_q][num_q_heads]
 *   cu_seqlens_q  int32 [batch + 1], cu[0] = 0, nondecreasing
 *   block_table   int32 [batch][max_blocks_per_seq]
 *   context_lens  int32 [batch]: cached prefix + this chunk (already written)
 *   max_q_len     host-side upper bound of the per-sequence chunk length
 *   workspace     may be NULL with workspace_bytes 0 (none needed).
 */
PKVQ_API pkvq_status pkvq_paged_attn_prefill(const pkvq_cache *cache, const void *q, void *out,
                                    float *lse_out, const int32_t *cu_seqlens_q,
                                    const int32_t *block_table, int32_t max_blocks_per_seq,
                                    const int32_t *context_lens, int32_t batch,
                                    int32_t max_q_len, int32_t num_q_heads,
                                    float softmax_scale, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * Options of the _ex attention entry points.  A zeroed struct, or NULL, gives
 * exactly pkvq_paged_attn_decode / pkvq_paged_attn_prefill.
 */
typedef struct {
    /* > 0: a query at position p sees only keys max(0, p - w + 1) .. p, and
     * the kernels read no block below the window.  0: keys 0 .. p.  Source:
     * "1Cat-LLM" README, "DFlash2 Long-Context Decay" (draft attention over
     * a sliding window of recent keys, the paged loop starting at the
     * window's first tile). */
    int32_t sliding_window;
    /* Decode only (NULL for prefill).  Nullable device int32 [batch][q_len]:
     * the position of every query among this call's keys, so that key j of
     * sequence b is visible to query t iff j <= query_pos[b][t] (and
     * j < context_lens[b]).  NULL means context_lens[b] - q_len + t.  For a
     * rank holding part of every sequence's keys (sequence-sharded decode,
     * "ReVolta" PyPI page, "Hardware": TP4 + DCP2): its keys in order, and
     * for each query the index of the last of them at or before the query's
     * global position (-1 if none). */
    const int32_t *query_pos;
} pkvq_attn_opts;

/*
 * pkvq_paged_attn_decode with options (sliding window, explicit query
 * positions).  Same arguments, results and errors otherwise; the workspace
 * is sized by pkvq_decode_workspace_bytes as before.  sliding_window < 0
 * returns PKVQ_ERR_INVALID_ARG.
 */
PKVQ_API pkvq_status pkvq_paged_attn_decode_ex(const pkvq_cache *cache, const void *q, void *out,
                                   float *lse_out, const int32_t *block_table,
                                   int32_t max_blocks_per_seq, const int32_t *context_lens,
                                   int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, float softmax_scale,
                                   const pkvq_attn_opts *opts, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * One decode step with its KV write: the step's new keys and values are
 * quantised into the cache exactly as pkvq_kv_write_quant does, then the
 * attention of pkvq_paged_attn_decode_ex runs over the whole context.
 * Source: "ReVolta" PyPI page, "Weight and KV formats" (new K/V quantised
 * into the 8-bit cache) and "1Cat-LLM" README, "Layer 1" / "Layer 2" (the
 * decode attention); the pages run the two as separate steps, this call
 * fuses them where it can.
 *   k_new, v_new  fp16 [batch][q_len][num_kv_heads][head_dim]: the keys and
 *                 values of each sequence's last q_len positions
 *                 (context_lens[b] - q_len + t), which land in the slots the
 *                 block table gives those positions (positions below 0 are
 *                 skipped).  16-byte aligned.
 * Every other argument as pkvq_paged_attn_decode_ex; opts->query_pos must
 * be NULL (PKVQ_ERR_INVALID_ARG otherwise).  Up to 16 query rows per KV head
 * the split-KV kernel writes the new tokens itself (the CTA that reads a
 * token's block quantises and stores it first), so a step is one launch plus
 * the merge; with more rows the KV write kernel runs first on the stream.
 * The cache afterwards is bit-identical to pkvq_kv_write_quant of the same
 * tokens, and the results to pkvq_paged_attn_decode_ex after it.
 */
PKVQ_API pkvq_status pkvq_paged_attn_decode_append(const pkvq_cache *cache, const void *k_new,
                                   const void *v_new, const void *q, void *out, float *lse_out,
                                   const int32_t *block_table, int32_t max_blocks_per_seq,
                                   const int32_t *context_lens, int32_t batch, int32_t q_len,
                                   int32_t num_q_heads, int32_t max_context_len,
                                   float softmax_scale, const pkvq_attn_opts *opts,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * pkvq_paged_attn_prefill with options (sliding window; query_pos must be
 * NULL, else PKVQ_ERR_UNSUPPORTED).
 */
PKVQ_API pkvq_status pkvq_paged_attn_prefill_ex(const pkvq_cache *cache, const void *q,
                                    void *out, float *lse_out, const int32_t *cu_seqlens_q,
                                    const int32_t *block_table, int32_t max_blocks_per_seq,
                                    const int32_t *context_lens, int32_t batch,
                                    int32_t max_q_len, int32_t num_q_heads,
                                    float softmax_scale, const pkvq_attn_opts *opts,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Combines attention results of the same queries computed over disjoint key
 * sets, e.g. by ranks that each hold part of every sequence's keys, after an
 * all-gather of their results.  Source: "ReVolta" PyPI page, "Hardware"
 * (TP4 + DCP2); "1Cat-LLM" README, "Layer 2" (FP32 merge of partial softmax
 * states).  With lse_r the natural-log sum-exp of part r's scores:
 *   lse = ln sum_r e^lse_r,  out = sum_r e^(lse_r - lse) out_r  (FP32),
 * parts with lse_r = -inf (no key) weigh nothing; a row no part saw gets zeros
 * and lse -inf.
 *   parts_out  fp16 [num_parts][n_rows][head_dim], each part's normalised output
 *   parts_lse  fp32 [num_parts][n_rows]
 *   out        fp16 [n_rows][head_dim];  lse_out nullable fp32 [n_rows]
 * head_dim must be 128; num_parts 1..64; n_rows == 0 is a no-op.
 */
PKVQ_API pkvq_status pkvq_merge_attn_states(const void *parts_out, const float *parts_lse,
                                   int32_t num_parts, int64_t n_rows, int32_t head_dim,
                                   void *out, float *lse_out, void *stream);

/*
 * Copies whole cache blocks between two caches of the same format and block
 * geometry (dtype, block_size, num_kv_heads, head_dim; the block counts may
 * differ), e.g. between the GPU pool and a host tier in pinned host memory the
 * device can address (cudaHostAlloc with mapping, or cudaHostRegister; with
 * unified addressing the host pointer serves as is).  Source: "ReVolta" PyPI
 * page, "KV offload modes" (cached pages kept in CPU memory and brought
 * back).  For i < n, block pairs[2i] of src becomes block pairs[2i + 1] of
 * dst: its K and V elements and, for INT8, its per-token scales.  The
 * per-head FP8 scales belong to the cache, not to a block, and are not
 * copied.  pairs: int32 [n][2], device-addressable.  Destination blocks must
 * be distinct and none may be a source block of the same call; ids outside
 * either pool are undefined behaviour (skipped and recorded in a
 * PKVQ_BOUNDS_CHECK build).  n == 0 is a no-op.
 */
PKVQ_API pkvq_status pkvq_kv_copy_blocks(const pkvq_cache *dst, const pkvq_cache *src,
                                const int32_t *pairs, int32_t n, void *stream);

/* Static description of a status code (never NULL). */
PKVQ_API const char *pkvq_status_string(pkvq_status status);

/*
 * Reads (and, if clear != 0, resets) the device status word of the current
 * device: 0 when no device-side check has fired.  Bit 0: an mbarrier wait
 * gave up after its iteration limit; bit 1: a block id outside the pool was
 * skipped (PKVQ_BOUNDS_CHECK builds).  Synchronizes with the device (it is a
 * diagnostic, not part of the hot path).  Returns PKVQ_ERR_CUDA if the copy
 * fails.
 */
PKVQ_API pkvq_status pkvq_device_status(uint32_t *status_out, int32_t clear);

/*
 * Text of the last CUDA runtime failure seen by this thread inside the library
 * (the call that failed and cudaGetErrorString of its code), or "" if none.
 * The pointer stays valid until this thread's next library call.
 */
PKVQ_API const char *pkvq_last_error(void);

/* Library version as "major.minor.patch". */
PKVQ_API const char *pkvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKVQ_H */
