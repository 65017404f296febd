// Host-side declarations shared by the pkvq translation units (not part of
// the public C ABI; see include/pkvq.h for that).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pkvq {

constexpr int kKvFp8 = 0;     // E4M3
constexpr int kKvInt8 = 1;
constexpr int kKvE5m2 = 2;
constexpr int kKvFp16 = 3;
constexpr int kHeadDim = 128;

// Bytes per stored cache element of a format.
__host__ __device__ constexpr int kv_elem_bytes(int kvt) { return kvt == kKvFp16 ? 2 : 1; }
// Formats with a static fp32 scale per KV head (or per layer).
__host__ __device__ constexpr bool kv_has_head_scale(int kvt)
{
    return kvt == kKvFp8 || kvt == kKvE5m2;
}

struct KvWriteParams {
    uint8_t *k_cache, *v_cache;
    const float *k_scale, *v_scale;        // FP8 formats
    int scale_stride;                      // 1: per KV head; 0: one scale per layer
    uint16_t *k_scale_tok, *v_scale_tok;   // INT8 (fp16 bits)
    const __half *k, *v;
    const int32_t *slot_mapping;   // or null: the slots of each sequence's last q_len
                                   // positions, from block_table and context_lens
    const int32_t *block_table, *context_lens;
    int max_blocks_per_seq, q_len;
    int num_tokens, num_kv_heads, num_blocks, block_size;
    uint32_t *status;
};

cudaError_t launch_kv_write_quant(const KvWriteParams &p, int kv_dtype, cudaStream_t stream);

struct DecodeParams {
    const uint8_t *k_cache, *v_cache;            // [blocks][Hkv][block_size][row bytes]
    const __half *k_new, *v_new;                 // nullable [batch][q_len][Hkv][128]: the
                                                 // split kernel writes these new tokens
                                                 // (the last q_len positions) first
    const float *k_scale, *v_scale;              // FP8 formats: per KV head (or layer)
    int scale_stride;                            // 1: per KV head; 0: one per layer
    const uint16_t *k_scale_tok, *v_scale_tok;   // INT8: per (block, head, token)
    int window;                                  // > 0: sliding window of keys
    const int32_t *query_pos;                    // nullable [batch][q_len]
    const __half *q;
    __half *out;
    float *lse;
    const int32_t *block_table;
    const int32_t *context_lens;
    int max_blocks_per_seq;
    int batch, q_len, num_q_heads, num_kv_heads, group, num_blocks, block_size;
    int rows;            // q_len * group rows per (sequence, KV head)
    int rows_per_cta;    // 8 * NT
    int row_groups;      // ceil(rows / rows_per_cta)
    int num_splits;      // C: CTA slots per (row group, KV head), mapped to
                         // (sequence, split) on the device from the lengths
    int uniform_splits;  // splits per sequence when all hold max_context_len
    int uniform_bpc;     // blocks per split in that case
    int split_min_blocks, split_gran;   // shortest split; split sizes are multiples of gran
    float scale_log2;    // softmax_scale * log2(e)
    float *ws_o;         // [row groups x Hkv][C][rows_per_cta][128] fp32, unnormalised
    float *ws_ml;        // [row groups x Hkv][C][rows_per_cta][2] fp32 (log2 max, sum)
    uint32_t *status;
};

struct DecodePlan {
    int nt;              // n8 row tiles per CTA (1 or 2)
    int rows_per_cta, row_groups;
    int num_splits;                     // C slots per (row group, KV head)
    int uniform_splits, uniform_bpc;    // the assignment with equal lengths
    int split_min_blocks, split_gran;
    bool tc;                            // tensor-core kernel: all rows of a KV head in one CTA
    size_t workspace_bytes;
};

// Split plan for a decode shape on the current device (kv_dtype: kKvFp8 or
// kKvInt8, whose kernels differ in registers and so in occupancy).
bool decode_plan(int kv_dtype, int batch, int q_len, int num_q_heads, int num_kv_heads,
                 int block_size, int max_context_len, DecodePlan *plan);

// The tensor-core decode kernel (17..128 rows: all rows of a KV head in one
// CTA, query rows on the MMA's M).
cudaError_t launch_decode_tc(const DecodeParams &p, int kv_dtype, const CUtensorMap &kmap,
                             const CUtensorMap &vmap, cudaStream_t stream);

cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, int kv_dtype,
                          const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream);

struct PrefillParams {
    const uint8_t *k_cache, *v_cache;            // [blocks][Hkv][block_size][row bytes]
    const float *k_scale, *v_scale;
    int scale_stride;                            // 1: per KV head; 0: one per layer
    const uint16_t *k_scale_tok, *v_scale_tok;
    int window;                                  // > 0: sliding window of keys
    const __half *q;
    __half *out;
    float *lse;
    const int32_t *cu_seqlens_q;
    const int32_t *block_table;
    const int32_t *context_lens;
    int max_blocks_per_seq;
    int batch, max_q_len, num_q_heads, num_kv_heads, group, num_blocks, block_size;
    int tokens_per_tile;   // query tokens per CTA tile
    int q_tiles;           // ceil(max_q_len / tokens_per_tile)
    float scale_log2;
    uint32_t *status;
};

cudaError_t launch_prefill_tc(const PrefillParams &p, int kv_dtype, const CUtensorMap &kmap,
                              const CUtensorMap &vmap, cudaStream_t stream);

// Encodes a 2-D uint8 tensor map over a cache: rows of row_bytes (128 or
// 256) bytes, boxes of 128 bytes x box_rows rows, 128-byte swizzle.
bool make_cache_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, int box_rows,
                           int row_bytes);

struct MergeParams {
    const __half *parts_out;   // [parts][rows][128]
    const float *parts_lse;    // [parts][rows]
    __half *out;
    float *lse;
    int parts;
    long long rows;
};

cudaError_t launch_merge_states(const MergeParams &p, cudaStream_t stream);

struct CopyParams {
    const uint8_t *src_k, *src_v;
    uint8_t *dst_k, *dst_v;
    const uint16_t *src_ks, *src_vs;   // INT8 scales (or null)
    uint16_t *dst_ks, *dst_vs;
    const int32_t *pairs;
    int n;
    long long block_bytes;             // elements of one block (all heads), bytes
    int block_scales;                  // INT8 scales of one block (all heads)
    int src_blocks, dst_blocks;
    uint32_t *status;
};

cudaError_t launch_copy_blocks(const CopyParams &p, cudaStream_t stream);

int device_sm_count();

}  // namespace pkvq
