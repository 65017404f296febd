/*
 * CPU oracle for attention over a paged, 8-bit-quantized KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this file's library.  The GPU
 * product path never calls it and shares no code, header, table or constant
 * with it.
 *
 * Everything here is plain and slow on purpose: FP64 arithmetic, one output
 * row at a time, no tiling, no online softmax, no split/merge.  OpenMP only
 * distributes independent output rows over host cores; it does not change the
 * order of any sum.
 *
 * What it follows (page title, section):
 *   - "ReVolta" (PyPI page), "Weight and KV formats": the cache stores 8-bit
 *     codes and converts them to FP16 for compute, i.e. attention is computed
 *     on the dequantized values code * scale.
 *   - same page, "E4M3 KV": static calibrated K/V scales, fallback 1.0; the
 *     oracle takes one fp32 scale per KV head (a per-layer scale is the case
 *     where all heads share one value).
 *   - same page, "INT8 KV": INT8 scales computed at run time per token and
 *     head; no calibration.
 *   - "1Cat-LLM" README, "Layer 1": paged KV maps logical tokens to physical
 *     pages through a page id; the oracle reads every key through the block
 *     table.
 *   - same README, "Layer 2" (N32 online softmax, Split-KV3, prefix/causal
 *     tail separation): these reach exactly the softmax attention result, so
 *     the oracle is that definition written out, softmax with max
 *     subtraction, in FP64.
 *   - "ReVolta" PyPI page, first section ("KV formats: FP8 E4M3, FP16, and
 *     INT8") and "1Cat-LLM" README, current SM70 work list ("FP8 E4M3 / E5M2
 *     KV storage"): the E5M2 and FP16 cache formats.
 *   - "ReVolta" PyPI page, "Hardware" and launch flags (TP4 + DCP2, decode
 *     context parallel size 2): a sequence's keys split over ranks, each rank
 *     attending over its own keys; or_merge_states combines the per-rank
 *     results by the definition of the softmax over the union of the keys.
 *   - "1Cat-LLM" README, "DFlash2 Long-Context Decay" (draft attention over a
 *     sliding window of recent keys): a query at position p sees keys
 *     p - window + 1 .. p.
 *   - "ReVolta" PyPI page, "KV offload modes" (CPU memory offload of cached
 *     pages): or_copy_blocks moves whole cache blocks between two pools.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes of this repository):
 *   - E4M3 is the OCP "E4M3FN" variant: bias 7, no infinities, S.1111.111 is
 *     NaN, largest finite 448.
 *   - Encoding divides in fp32 (correctly rounded), then rounds the fp32
 *     quotient to nearest-even E4M3 and saturates finite overflow to +-448
 *     (infinities too).  NaN keeps its sign: S.1111.111.  Scale 0 gives code
 *     0.
 *   - INT8: s = fp16_rn(fp32(absmax) / 127), code = clamp(rint(x / s), -127,
 *     127) with fp32 division and ties-to-even; s == 0 gives all-zero codes.
 *   - Query t of a sequence with context c and q_len new tokens sits at
 *     position c - q_len + t and sees keys 0..pos.  A row with no visible key
 *     returns zeros and lse = -inf.
 *   - GQA: query head h reads KV head h / (Hq / Hkv).
 *   - E5M2 is the OCP/IEEE-style 8-bit format: bias 15, S.11111.00 is
 *     infinity, S.11111.xx (xx != 0) NaN, largest finite 57344.  Encoding is
 *     the same as for E4M3: fp32 quotient, nearest-even, finite overflow and
 *     infinities saturate to +-57344, NaN keeps its sign as S.11111.11.
 *   - FP16 cache: the fp16 values themselves, no scale.
 *   - Per-layer scale: one fp32 K scale and one V scale shared by every KV
 *     head (the per-head arrays with all entries equal).
 *   - Sliding window w > 0: keys max(0, p - w + 1) .. p; w <= 0: all keys
 *     0 .. p.  Keys exist only below the context length.
 *   - Query positions given explicitly (a rank holding part of a sequence's
 *     keys): key j is visible to a query at position p iff j <= p; the
 *     default position is context - q_len + t.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * fp32 division must be IEEE round-to-nearest (x86-64 SSE does this).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_FP8_E4M3 0
#define OR_INT8 1
#define OR_FP8_E5M2 2
#define OR_FP16 3

/* bytes per stored element of a cache format */
static int or_elem_bytes(int dtype)
{
    return dtype == OR_FP16 ? 2 : 1;
}

/* ------------------------------------------------------------------ */
/* binary16                                                             */
/* ------------------------------------------------------------------ */

/* fp16 bit pattern -> double (exact). */
double or_half_to_double(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);             /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

/* fp32 -> fp16 bits, IEEE round to nearest, ties to even; overflow -> inf. */
uint16_t or_float_to_half_rn(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    if (isnan(f))
        return sign | 0x7e00u;
    if (isinf(f))
        return sign | 0x7c00u;
    double v = fabs((double)f);
    if (v == 0.0)
        return sign;
    int e2;
    frexp(v, &e2);          /* v = frac * 2^e2, frac in [0.5, 1) */
    int E = e2 - 1;         /* v in [2^E, 2^(E+1)) */
    if (E > 15)
        return sign | 0x7c00u;
    if (E < -14)
        E = -14;            /* subnormals share the spacing of the first binade */
    double ulp = ldexp(1.0, E - 10);
    double r = rint(v / ulp); /* exact quotient; rint = nearest, ties to even */
    if (r >= 2048.0) {        /* rounding carried into the next binade */
        E += 1;
        r = 1024.0;
    }
    if (E > 15)
        return sign | 0x7c00u;
    uint32_t ir = (uint32_t)r;
    if (ir < 1024u)           /* subnormal (only when E == -14) */
        return sign | (uint16_t)ir;
    return sign | (uint16_t)(((uint32_t)(E + 15) << 10) + (ir - 1024u));
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (FN variant)                                               */
/* ------------------------------------------------------------------ */

double or_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);           /* (m/8) * 2^(1-7) */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Round an fp32 value to E4M3: nearest, ties to even, saturating. */
uint8_t or_e4m3_encode(float q)
{
    uint32_t x;
    memcpy(&x, &q, 4);
    uint8_t sign = (uint8_t)((x >> 24) & 0x80u);
    if (isnan(q))
        return sign | 0x7fu;
    double v = fabs((double)q);
    if (v >= 448.0)             /* includes +-inf: saturate to the max finite */
        return sign | 0x7eu;
    if (v == 0.0)
        return sign;
    int e2;
    frexp(v, &e2);
    int E = e2 - 1;             /* v in [2^E, 2^(E+1)) */
    if (E < -6)
        E = -6;                 /* subnormals: spacing 2^-9 */
    double ulp = ldexp(1.0, E - 3);
    double r = rint(v / ulp);
    if (r >= 16.0) {
        E += 1;
        r = 8.0;
    }
    uint32_t ir = (uint32_t)r;
    if (ir < 8u)                /* subnormal (only when E == -6) */
        return sign | (uint8_t)ir;
    /* v < 448 guarantees E <= 8 and, at E == 8, r <= 14 (448 = 1.75 * 2^8) */
    return sign | (uint8_t)(((uint32_t)(E + 7) << 3) | (ir - 8u));
}

/* ------------------------------------------------------------------ */
/* FP8 E5M2                                                            */
/* ------------------------------------------------------------------ */

double or_e5m2_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 2) & 31;
    int m = c & 3;
    double v;
    if (e == 31)
        return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0)
        v = ldexp((double)m, -16);          /* (m/4) * 2^(1-15) */
    else
        v = ldexp((double)(4 + m), e - 17); /* (1 + m/4) * 2^(e-15) */
    return s ? -v : v;
}

/* Round an fp32 value to E5M2: nearest, ties to even, saturating. */
uint8_t or_e5m2_encode(float q)
{
    uint32_t x;
    memcpy(&x, &q, 4);
    uint8_t sign = (uint8_t)((x >> 24) & 0x80u);
    if (isnan(q))
        return sign | 0x7fu;
    double v = fabs((double)q);
    if (v >= 57344.0)           /* includes +-inf: saturate to the max finite */
        return sign | 0x7bu;
    if (v == 0.0)
        return sign;
    int e2;
    frexp(v, &e2);
    int E = e2 - 1;             /* v in [2^E, 2^(E+1)) */
    if (E < -14)
        E = -14;                /* subnormals: spacing 2^-16 */
    double ulp = ldexp(1.0, E - 2);
    double r = rint(v / ulp);
    if (r >= 8.0) {
        E += 1;
        r = 4.0;
    }
    uint32_t ir = (uint32_t)r;
    if (ir < 4u)                /* subnormal (only when E == -14) */
        return sign | (uint8_t)ir;
    /* v < 57344 = 1.75 * 2^15 keeps E <= 15 and, at E == 15, r <= 7 */
    return sign | (uint8_t)(((uint32_t)(E + 15) << 2) | (ir - 4u));
}

/* ------------------------------------------------------------------ */
/* Quantize one (token, head) row                                      */
/* ------------------------------------------------------------------ */

/* FP8: code[d] = E4M3(fp32(x[d]) / scale) (E5M2 when e5m2 != 0), scale 0 ->
 * code 0. */
void or_quant_row_fp8(const uint16_t *x, int D, float scale, uint8_t *codes, int e5m2)
{
    for (int d = 0; d < D; ++d) {
        if (scale == 0.0f) {
            codes[d] = 0;
            continue;
        }
        float xf = (float)or_half_to_double(x[d]); /* exact */
        float qf = xf / scale;                     /* fp32 IEEE division */
        codes[d] = e5m2 ? or_e5m2_encode(qf) : or_e4m3_encode(qf);
    }
}

/* INT8: s = fp16(absmax / 127); code = clamp(rint(x / s), -127, 127). */
void or_quant_row_int8(const uint16_t *x, int D, int8_t *codes, uint16_t *scale_bits)
{
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
        float a = fabsf((float)or_half_to_double(x[d]));
        if (a > amax)
            amax = a;
    }
    float s32 = amax / 127.0f;
    uint16_t s16 = or_float_to_half_rn(s32);
    *scale_bits = s16;
    float s = (float)or_half_to_double(s16);
    for (int d = 0; d < D; ++d) {
        if (s == 0.0f) {
            codes[d] = 0;
            continue;
        }
        float xf = (float)or_half_to_double(x[d]);
        float qf = xf / s;
        float r = rintf(qf);
        if (r > 127.0f)
            r = 127.0f;
        if (r < -127.0f)
            r = -127.0f;
        codes[d] = (int8_t)r;
    }
}

/* ------------------------------------------------------------------ */
/* KV write + quantize into the paged cache                             */
/* ------------------------------------------------------------------ */

/*
 * Cache layout: [num_blocks][Hkv][block_size][D] elements (1 byte for the
 * 8-bit formats, the fp16 bits for FP16); INT8 scales [num_blocks][Hkv]
 * [block_size] fp16.  Token i goes to slot slot_mapping[i] = block *
 * block_size + offset; a negative slot is skipped.  k, v: fp16 [T][Hkv][D].
 * FP8 scales: fp32 [Hkv], or one value for every head when scale_per_layer.
 */
void or_kv_write_quant(int dtype, int num_blocks, int block_size, int Hkv, int D,
                       uint8_t *k_cache, uint8_t *v_cache,
                       const float *k_scale, const float *v_scale, int scale_per_layer,
                       uint16_t *k_scale_tok, uint16_t *v_scale_tok,
                       const uint16_t *k, const uint16_t *v,
                       const int32_t *slot_mapping, int T)
{
    (void)num_blocks;
    for (int i = 0; i < T; ++i) {
        int32_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int blk = slot / block_size;
        int off = slot % block_size;
        for (int h = 0; h < Hkv; ++h) {
            size_t row = ((size_t)blk * Hkv + h) * block_size + off;
            const uint16_t *kx = k + ((size_t)i * Hkv + h) * D;
            const uint16_t *vx = v + ((size_t)i * Hkv + h) * D;
            int hs = scale_per_layer ? 0 : h;
            if (dtype == OR_FP8_E4M3 || dtype == OR_FP8_E5M2) {
                int e5 = dtype == OR_FP8_E5M2;
                or_quant_row_fp8(kx, D, k_scale[hs], k_cache + row * D, e5);
                or_quant_row_fp8(vx, D, v_scale[hs], v_cache + row * D, e5);
            } else if (dtype == OR_FP16) {
                memcpy(k_cache + row * D * 2, kx, (size_t)D * 2);
                memcpy(v_cache + row * D * 2, vx, (size_t)D * 2);
            } else {
                or_quant_row_int8(kx, D, (int8_t *)(k_cache + row * D), k_scale_tok + row);
                or_quant_row_int8(vx, D, (int8_t *)(v_cache + row * D), v_scale_tok + row);
            }
        }
    }
}

/*
 * Whole-block copy between two pools of the same geometry: for i < n, block
 * pairs[2i] of the source becomes block pairs[2i+1] of the destination
 * (K and V elements, and the INT8 per-token scales when present).
 */
void or_copy_blocks(int dtype, int block_size, int Hkv, int D,
                    const uint8_t *src_k, const uint8_t *src_v,
                    const uint16_t *src_ks, const uint16_t *src_vs,
                    uint8_t *dst_k, uint8_t *dst_v, uint16_t *dst_ks, uint16_t *dst_vs,
                    const int32_t *pairs, int n)
{
    size_t blk_bytes = (size_t)Hkv * block_size * D * or_elem_bytes(dtype);
    size_t blk_scales = (size_t)Hkv * block_size;
    for (int i = 0; i < n; ++i) {
        size_t s = (size_t)pairs[2 * i], d = (size_t)pairs[2 * i + 1];
        memcpy(dst_k + d * blk_bytes, src_k + s * blk_bytes, blk_bytes);
        memcpy(dst_v + d * blk_bytes, src_v + s * blk_bytes, blk_bytes);
        if (dtype == OR_INT8) {
            memcpy(dst_ks + d * blk_scales, src_ks + s * blk_scales, blk_scales * 2);
            memcpy(dst_vs + d * blk_scales, src_vs + s * blk_scales, blk_scales * 2);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Attention over the paged cache                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    int dtype, num_blocks, block_size, Hkv, D;
    const uint8_t *k_cache, *v_cache;
    const float *k_scale, *v_scale;
    int scale_per_layer;
    const uint16_t *k_scale_tok, *v_scale_tok;
} or_cache;

/* Dequantized element d of key/value token j of sequence s, KV head g. */
static double dq(const or_cache *c, const uint8_t *codes, const float *head_scale,
                 const uint16_t *tok_scale, const int32_t *bt_row, int j, int g, int d)
{
    int blk = bt_row[j / c->block_size];
    int off = j % c->block_size;
    size_t row = ((size_t)blk * c->Hkv + g) * c->block_size + off;
    int hs = c->scale_per_layer ? 0 : g;
    if (c->dtype == OR_FP16) {
        uint16_t h;
        memcpy(&h, codes + (row * c->D + d) * 2, 2);
        return or_half_to_double(h);
    }
    uint8_t code = codes[row * c->D + d];
    if (c->dtype == OR_FP8_E4M3)
        return or_e4m3_decode(code) * (double)head_scale[hs];
    if (c->dtype == OR_FP8_E5M2)
        return or_e5m2_decode(code) * (double)head_scale[hs];
    return (double)(int8_t)code * or_half_to_double(tok_scale[row]);
}

/*
 * One output row: query token index i (into the packed q), query head h.
 * Keys lo..hi are visible (none when hi < lo).
 * scores: scratch of at least hi+1 doubles.
 */
static void attend_row(const or_cache *c, const uint16_t *q, int Hq, int i, int h,
                       const int32_t *bt_row, int lo, int hi, double softmax_scale,
                       double *scores, double *out_row, double *lse)
{
    int D = c->D;
    int G = Hq / c->Hkv;
    int g = h / G;
    const uint16_t *qr = q + ((size_t)i * Hq + h) * D;
    for (int d = 0; d < D; ++d)
        out_row[d] = 0.0;
    if (hi < lo) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int j = lo; j <= hi; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += or_half_to_double(qr[d]) *
                   dq(c, c->k_cache, c->k_scale, c->k_scale_tok, bt_row, j, g, d);
        scores[j] = softmax_scale * acc;
        if (scores[j] > m)
            m = scores[j];
    }
    double l = 0.0;
    for (int j = lo; j <= hi; ++j) {
        double p = exp(scores[j] - m);
        l += p;
        for (int d = 0; d < D; ++d)
            out_row[d] += p * dq(c, c->v_cache, c->v_scale, c->v_scale_tok, bt_row, j, g, d);
    }
    for (int d = 0; d < D; ++d)
        out_row[d] /= l;
    *lse = m + log(l);
}

/*
 * Paged attention for a varlen batch.
 *   q            fp16 [total_q][Hq][D]; sequence s owns rows cu_seqlens_q[s] ..
 *                cu_seqlens_q[s+1]-1 (decode with a fixed q_len is the case
 *                cu_seqlens_q[s] = s * q_len).
 *   context_lens [B]: cached tokens including this step's new ones.
 *   block_table  [B][max_blocks_per_seq].
 *   rows         optional list of n_rows (token index, head) pairs; NULL means
 *                every (token, head).  out/lse are indexed like the full
 *                output when rows == NULL, and by list position otherwise.
 *   out          double [.][D], lse double [.].
 *   nthreads     OpenMP threads (<= 0: runtime default).
 * Returns the number of threads used.
 */
int or_paged_attention(int dtype, int num_blocks, int block_size, int Hkv, int D,
                       const uint8_t *k_cache, const uint8_t *v_cache,
                       const float *k_scale, const float *v_scale, int scale_per_layer,
                       const uint16_t *k_scale_tok, const uint16_t *v_scale_tok,
                       const uint16_t *q, int Hq,
                       const int32_t *cu_seqlens_q, const int32_t *context_lens,
                       const int32_t *block_table, int max_blocks_per_seq, int B,
                       float softmax_scale, int window, const int32_t *query_pos,
                       const int32_t *rows, int n_rows,
                       double *out, double *lse, int nthreads)
{
    or_cache c = {dtype, num_blocks, block_size, Hkv, D, k_cache, v_cache,
                  k_scale, v_scale, scale_per_layer, k_scale_tok, v_scale_tok};
    int total_q = cu_seqlens_q[B];
    long n = rows ? n_rows : (long)total_q * Hq;
    int max_ctx = 0;
    for (int s = 0; s < B; ++s)
        if (context_lens[s] > max_ctx)
            max_ctx = context_lens[s];
    int used = 1;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
#pragma omp parallel num_threads(nthreads)
    {
#ifdef _OPENMP
#pragma omp single
        used = omp_get_num_threads();
#endif
        double *scores = (double *)malloc(sizeof(double) * (size_t)(max_ctx > 0 ? max_ctx : 1));
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n; ++r) {
            int i, h;
            if (rows) {
                i = rows[2 * r];
                h = rows[2 * r + 1];
            } else {
                i = (int)(r / Hq);
                h = (int)(r % Hq);
            }
            int s = 0;
            while (s < B - 1 && !(cu_seqlens_q[s] <= i && i < cu_seqlens_q[s + 1]))
                ++s;
            int q_len = cu_seqlens_q[s + 1] - cu_seqlens_q[s];
            int t = i - cu_seqlens_q[s];
            int pos = query_pos ? query_pos[i] : context_lens[s] - q_len + t;
            int hi = pos < context_lens[s] - 1 ? pos : context_lens[s] - 1;
            int lo = window > 0 ? pos - window + 1 : 0;
            if (lo < 0)
                lo = 0;
            attend_row(&c, q, Hq, i, h, block_table + (size_t)s * max_blocks_per_seq, lo, hi,
                       (double)softmax_scale, scores, out + (size_t)r * D, lse + r);
        }
        free(scores);
    }
    return used;
}

/*
 * Softmax over the union of disjoint key sets, from each set's own result:
 * part r holds out_r = sum_j p_j v_j / sum_j p_j and lse_r = ln sum_j e^s_j
 * over its keys.  Then lse = ln sum_r e^lse_r and out = sum_r e^(lse_r - lse)
 * out_r.  A part with no key has lse_r = -inf and weight 0; no part with a
 * key gives out = 0, lse = -inf.
 *   outs [R][n][D], lses [R][n]; out [n][D], lse [n].
 */
void or_merge_states(int R, long n, int D, const double *outs, const double *lses,
                     double *out, double *lse)
{
    for (long i = 0; i < n; ++i) {
        double m = -INFINITY;
        for (int r = 0; r < R; ++r)
            if (lses[(size_t)r * n + i] > m)
                m = lses[(size_t)r * n + i];
        for (int d = 0; d < D; ++d)
            out[(size_t)i * D + d] = 0.0;
        if (m == -INFINITY) {
            lse[i] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int r = 0; r < R; ++r)
            sum += exp(lses[(size_t)r * n + i] - m);
        lse[i] = m + log(sum);
        for (int r = 0; r < R; ++r) {
            double w = exp(lses[(size_t)r * n + i] - lse[i]);
            if (w == 0.0)
                continue;
            for (int d = 0; d < D; ++d)
                out[(size_t)i * D + d] += w * outs[((size_t)r * n + i) * D + d];
        }
    }
}

/* ------------------------------------------------------------------ */
/* Element-wise batch helpers (plain loops over the scalar routines)    */
/* ------------------------------------------------------------------ */

void or_half_to_double_n(const uint16_t *h, double *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_half_to_double(h[i]);
}

void or_float_to_half_rn_n(const float *f, uint16_t *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_float_to_half_rn(f[i]);
}

void or_e4m3_decode_n(const uint8_t *c, double *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_e4m3_decode(c[i]);
}

void or_e4m3_encode_n(const float *q, uint8_t *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_e4m3_encode(q[i]);
}

void or_e5m2_decode_n(const uint8_t *c, double *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_e5m2_decode(c[i]);
}

void or_e5m2_encode_n(const float *q, uint8_t *out, long n)
{
    for (long i = 0; i < n; ++i)
        out[i] = or_e5m2_encode(q[i]);
}
