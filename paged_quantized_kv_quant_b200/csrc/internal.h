// Host-side declarations shared by the pkvq translation units (not part of
// the public C ABI; see include/pkvq.h for that).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pkvq {

constexpr int kKvFp8 = 0;
constexpr int kKvInt8 = 1;
constexpr int kHeadDim = 128;

struct KvWriteParams {
    uint8_t *k_cache, *v_cache;
    const float *k_scale, *v_scale;        // FP8
    uint16_t *k_scale_tok, *v_scale_tok;   // INT8 (fp16 bits)
    const __half *k, *v;
    const int32_t *slot_mapping;
    int num_tokens, num_kv_heads, num_blocks, block_size;
    uint32_t *status;
};

cudaError_t launch_kv_write_quant(const KvWriteParams &p, int kv_dtype, cudaStream_t stream);

struct DecodeParams {
    const float *k_scale, *v_scale;              // FP8: per KV head
    const uint16_t *k_scale_tok, *v_scale_tok;   // INT8: per (block, head, token)
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

// The tensor-core decode kernel (all rows of a KV head in one CTA).
cudaError_t launch_decode_tc(const DecodeParams &p, int kv_dtype, const CUtensorMap &kmap,
                             const CUtensorMap &vmap, cudaStream_t stream);

cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, int kv_dtype,
                          const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream);

struct PrefillParams {
    const float *k_scale, *v_scale;
    const uint16_t *k_scale_tok, *v_scale_tok;
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

// Encodes a 2-D uint8 tensor map over a cache: rows of 128 bytes, boxes of
// box_rows rows, 128-byte swizzle.
bool make_cache_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, int box_rows);

int device_sm_count();

}  // namespace pkvq
