// C ABI of libpkvq.so: argument validation, tensor-map setup and dispatch.
// Every check happens on the host before any launch; nothing here allocates
// device memory or synchronizes the host with the device (except
// pkvq_device_status, a diagnostic).
#include "../../include/pkvq.h"
#include "common.cuh"
#include "internal.h"

#include <cudaTypedefs.h>
#include <math.h>
#include <mutex>
#include <stdio.h>
#include <stdlib.h>

namespace pkvq {

__device__ uint32_t g_status_word;

namespace {

constexpr int kMaxDevices = 64;

uint32_t *status_ptr()
{
    static uint32_t *ptrs[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess)
            return nullptr;
        ptrs[dev] = static_cast<uint32_t *>(p);
    }
    return ptrs[dev];
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

pkvq_status check_cache(const pkvq_cache *c)
{
    if (!c || !c->k_cache || !c->v_cache)
        return PKVQ_ERR_INVALID_ARG;
    if (c->dtype != PKVQ_KV_FP8_E4M3 && c->dtype != PKVQ_KV_INT8 &&
        c->dtype != PKVQ_KV_FP8_E5M2 && c->dtype != PKVQ_KV_FP16)
        return PKVQ_ERR_UNSUPPORTED;
    if (c->head_dim != kHeadDim)
        return PKVQ_ERR_UNSUPPORTED;
    if (c->block_size != 16 && c->block_size != 32 && c->block_size != 64)
        return PKVQ_ERR_UNSUPPORTED;
    if (c->num_blocks <= 0 || c->num_kv_heads <= 0)
        return PKVQ_ERR_INVALID_ARG;
    // tensor-map row coordinates are int32
    if ((long long)c->num_blocks * c->num_kv_heads * c->block_size >= (1LL << 31))
        return PKVQ_ERR_UNSUPPORTED;
    if (kv_has_head_scale(c->dtype)) {
        if (!c->k_scale || !c->v_scale)
            return PKVQ_ERR_INVALID_ARG;
    } else if (c->dtype == PKVQ_KV_INT8) {
        if (!c->k_scale_tok || !c->v_scale_tok)
            return PKVQ_ERR_INVALID_ARG;
        if (!aligned16(c->k_scale_tok) || !aligned16(c->v_scale_tok))
            return PKVQ_ERR_MISALIGNED;
    }
    if (!aligned16(c->k_cache) || !aligned16(c->v_cache))
        return PKVQ_ERR_MISALIGNED;
    return PKVQ_OK;
}

pkvq_status cache_maps(const pkvq_cache *c, CUtensorMap *km, CUtensorMap *vm)
{
    const uint64_t rows = (uint64_t)c->num_blocks * c->num_kv_heads * c->block_size;
    const int row_bytes = kHeadDim * kv_elem_bytes(c->dtype);
    if (!make_cache_tensor_map(km, c->k_cache, rows, c->block_size, row_bytes) ||
        !make_cache_tensor_map(vm, c->v_cache, rows, c->block_size, row_bytes))
        return PKVQ_ERR_CUDA;
    return PKVQ_OK;
}

int scale_stride(const pkvq_cache *c)
{
    return c->scale_per_layer ? 0 : 1;
}

thread_local char t_last_error[256] = "";

pkvq_status from_cuda(cudaError_t e, const char *what = "launch")
{
    if (e == cudaSuccess)
        return PKVQ_OK;
    snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", what, cudaGetErrorString(e),
             (int)e);
    return PKVQ_ERR_CUDA;
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

bool make_cache_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, int box_rows,
                           int row_bytes)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int device_sm_count()
{
    static int counts[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 148;
    if (!counts[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

}  // namespace pkvq

using namespace pkvq;

extern "C" {

const char *pkvq_last_error(void)
{
    return t_last_error;
}

const char *pkvq_version(void)
{
    return "0.1.0";
}

const char *pkvq_status_string(pkvq_status s)
{
    switch (s) {
    case PKVQ_OK: return "ok";
    case PKVQ_ERR_INVALID_ARG: return "invalid argument";
    case PKVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKVQ_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case PKVQ_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case PKVQ_ERR_DEVICE: return "device-side check failed";
    case PKVQ_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

pkvq_status pkvq_device_status(uint32_t *status_out, int32_t clear)
{
    if (!status_out)
        return PKVQ_ERR_INVALID_ARG;
    uint32_t *p = status_ptr();
    if (!p)
        return PKVQ_ERR_CUDA;
    if (cudaMemcpy(status_out, p, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return PKVQ_ERR_CUDA;
    if (clear && cudaMemset(p, 0, sizeof(uint32_t)) != cudaSuccess)
        return PKVQ_ERR_CUDA;
    return PKVQ_OK;
}

pkvq_status pkvq_kv_write_quant(const pkvq_cache *cache, const void *k, const void *v,
                                const int32_t *slot_mapping, int32_t num_tokens, void *stream)
{
    pkvq_status st = check_cache(cache);
    if (st != PKVQ_OK)
        return st;
    if (num_tokens < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (num_tokens == 0)
        return PKVQ_OK;
    if (!k || !v || !slot_mapping)
        return PKVQ_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v))
        return PKVQ_ERR_MISALIGNED;
    KvWriteParams p{};
    p.k_cache = static_cast<uint8_t *>(cache->k_cache);
    p.v_cache = static_cast<uint8_t *>(cache->v_cache);
    p.k_scale = cache->k_scale;
    p.v_scale = cache->v_scale;
    p.scale_stride = scale_stride(cache);
    p.k_scale_tok = static_cast<uint16_t *>(cache->k_scale_tok);
    p.v_scale_tok = static_cast<uint16_t *>(cache->v_scale_tok);
    p.k = static_cast<const __half *>(k);
    p.v = static_cast<const __half *>(v);
    p.slot_mapping = slot_mapping;
    p.num_tokens = num_tokens;
    p.num_kv_heads = cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.block_size = cache->block_size;
    p.status = status_ptr();
    if (!p.status)
        return PKVQ_ERR_CUDA;
    return from_cuda(launch_kv_write_quant(p, cache->dtype, static_cast<cudaStream_t>(stream)));
}

size_t pkvq_decode_workspace_bytes(int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, const pkvq_cache *cache)
{
    if (check_cache(cache) != PKVQ_OK || batch <= 0 || q_len <= 0 || q_len > 16 ||
        max_context_len < 0 || num_q_heads <= 0 || num_q_heads % cache->num_kv_heads)
        return 0;
    DecodePlan plan;
    if (!decode_plan(cache->dtype, batch, q_len, num_q_heads, cache->num_kv_heads, cache->block_size,
                     max_context_len, &plan))
        return 0;
    return plan.workspace_bytes;
}

pkvq_status pkvq_paged_attn_decode(const pkvq_cache *cache, const void *q, void *out,
                                   float *lse_out, const int32_t *block_table,
                                   int32_t max_blocks_per_seq, const int32_t *context_lens,
                                   int32_t batch, int32_t q_len, int32_t num_q_heads,
                                   int32_t max_context_len, float softmax_scale,
                                   void *workspace, size_t workspace_bytes, void *stream)
{
    return pkvq_paged_attn_decode_ex(cache, q, out, lse_out, block_table, max_blocks_per_seq,
                                     context_lens, batch, q_len, num_q_heads, max_context_len,
                                     softmax_scale, nullptr, workspace, workspace_bytes, stream);
}

namespace {

// Decode, optionally appending the step's new tokens (k_new / v_new: the
// keys and values of each sequence's last q_len positions) first.
pkvq_status decode_impl(const pkvq_cache *cache, const void *k_new, const void *v_new,
                        const void *q, void *out, float *lse_out, const int32_t *block_table,
                        int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t batch,
                        int32_t q_len, int32_t num_q_heads, int32_t max_context_len,
                        float softmax_scale, const pkvq_attn_opts *opts, void *workspace,
                        size_t workspace_bytes, void *stream)
{
    if (opts && opts->sliding_window < 0)
        return PKVQ_ERR_INVALID_ARG;
    pkvq_status st = check_cache(cache);
    if (st != PKVQ_OK)
        return st;
    if (batch < 0 || q_len < 1 || q_len > 16 || num_q_heads <= 0 || max_context_len < 0 ||
        max_blocks_per_seq < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (num_q_heads % cache->num_kv_heads)
        return PKVQ_ERR_INVALID_ARG;
    const int group = num_q_heads / cache->num_kv_heads;
    if (group > 16)
        return PKVQ_ERR_UNSUPPORTED;
    if (!isfinite(softmax_scale))
        return PKVQ_ERR_INVALID_ARG;
    if (batch == 0)
        return PKVQ_OK;
    if (!q || !out || !block_table || !context_lens)
        return PKVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out))
        return PKVQ_ERR_MISALIGNED;
    if ((long long)max_blocks_per_seq * cache->block_size < max_context_len)
        return PKVQ_ERR_INVALID_ARG;
    DecodePlan plan;
    if (!decode_plan(cache->dtype, batch, q_len, num_q_heads, cache->num_kv_heads, cache->block_size,
                     max_context_len, &plan))
        return PKVQ_ERR_INVALID_ARG;
    if (plan.workspace_bytes > 0) {
        if (!workspace || workspace_bytes < plan.workspace_bytes)
            return PKVQ_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(workspace))
            return PKVQ_ERR_MISALIGNED;
    }
    CUtensorMap km, vm;
    st = cache_maps(cache, &km, &vm);
    if (st != PKVQ_OK)
        return st;
    DecodeParams p{};
    p.k_cache = static_cast<const uint8_t *>(cache->k_cache);
    p.v_cache = static_cast<const uint8_t *>(cache->v_cache);
    const bool head_scale = kv_has_head_scale(cache->dtype);
    p.k_scale = head_scale ? cache->k_scale : nullptr;
    p.v_scale = head_scale ? cache->v_scale : nullptr;
    p.scale_stride = scale_stride(cache);
    p.k_scale_tok = static_cast<const uint16_t *>(cache->k_scale_tok);
    p.v_scale_tok = static_cast<const uint16_t *>(cache->v_scale_tok);
    p.window = opts ? opts->sliding_window : 0;
    p.query_pos = opts ? opts->query_pos : nullptr;
    p.q = static_cast<const __half *>(q);
    p.out = static_cast<__half *>(out);
    p.lse = lse_out;
    p.block_table = block_table;
    p.context_lens = context_lens;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.batch = batch;
    p.q_len = q_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.group = group;
    p.num_blocks = cache->num_blocks;
    p.block_size = cache->block_size;
    p.rows = q_len * group;
    p.rows_per_cta = plan.rows_per_cta;
    p.row_groups = plan.row_groups;
    p.num_splits = plan.num_splits;
    p.uniform_splits = plan.uniform_splits;
    p.uniform_bpc = plan.uniform_bpc;
    p.split_min_blocks = plan.split_min_blocks;
    p.split_gran = plan.split_gran;
    p.scale_log2 = softmax_scale * kLog2e;
    // workspace: [partial O][partial (m, l)]
    float *ws = static_cast<float *>(workspace);
    const size_t n_rows_ws = (size_t)cache->num_kv_heads * plan.row_groups * plan.num_splits *
                             plan.rows_per_cta;
    p.ws_o = plan.workspace_bytes ? ws : nullptr;
    p.ws_ml = plan.workspace_bytes ? ws + n_rows_ws * kHeadDim : nullptr;
    p.status = status_ptr();
    if (!p.status)
        return PKVQ_ERR_CUDA;
    cudaStream_t st_ = static_cast<cudaStream_t>(stream);
    if (k_new) {
        if (plan.tc) {
            // the tensor-core kernel reads whole tiles through one copy ring:
            // the new tokens are written by the KV write kernel just before
            KvWriteParams w{};
            w.k_cache = static_cast<uint8_t *>(cache->k_cache);
            w.v_cache = static_cast<uint8_t *>(cache->v_cache);
            w.k_scale = cache->k_scale;
            w.v_scale = cache->v_scale;
            w.scale_stride = scale_stride(cache);
            w.k_scale_tok = static_cast<uint16_t *>(cache->k_scale_tok);
            w.v_scale_tok = static_cast<uint16_t *>(cache->v_scale_tok);
            w.k = static_cast<const __half *>(k_new);
            w.v = static_cast<const __half *>(v_new);
            w.slot_mapping = nullptr;
            w.block_table = block_table;
            w.context_lens = context_lens;
            w.max_blocks_per_seq = max_blocks_per_seq;
            w.q_len = q_len;
            w.num_tokens = batch * q_len;
            w.num_kv_heads = cache->num_kv_heads;
            w.num_blocks = cache->num_blocks;
            w.block_size = cache->block_size;
            w.status = p.status;
            const cudaError_t e = launch_kv_write_quant(w, cache->dtype, st_);
            if (e != cudaSuccess)
                return from_cuda(e);
        } else {
            // the split kernel: each CTA writes the new tokens of its blocks
            p.k_new = static_cast<const __half *>(k_new);
            p.v_new = static_cast<const __half *>(v_new);
        }
    }
    return from_cuda(launch_decode(p, plan, cache->dtype, km, vm, st_));
}

}  // namespace

pkvq_status pkvq_paged_attn_decode_ex(const pkvq_cache *cache, const void *q, void *out,
                                      float *lse_out, const int32_t *block_table,
                                      int32_t max_blocks_per_seq, const int32_t *context_lens,
                                      int32_t batch, int32_t q_len, int32_t num_q_heads,
                                      int32_t max_context_len, float softmax_scale,
                                      const pkvq_attn_opts *opts, void *workspace,
                                      size_t workspace_bytes, void *stream)
{
    return decode_impl(cache, nullptr, nullptr, q, out, lse_out, block_table,
                       max_blocks_per_seq, context_lens, batch, q_len, num_q_heads,
                       max_context_len, softmax_scale, opts, workspace, workspace_bytes, stream);
}

pkvq_status pkvq_paged_attn_decode_append(const pkvq_cache *cache, const void *k_new,
                                          const void *v_new, const void *q, void *out,
                                          float *lse_out, const int32_t *block_table,
                                          int32_t max_blocks_per_seq,
                                          const int32_t *context_lens, int32_t batch,
                                          int32_t q_len, int32_t num_q_heads,
                                          int32_t max_context_len, float softmax_scale,
                                          const pkvq_attn_opts *opts, void *workspace,
                                          size_t workspace_bytes, void *stream)
{
    if (opts && opts->query_pos)
        return PKVQ_ERR_INVALID_ARG;   // the new tokens are the last q_len positions
    if (batch > 0) {
        if (!k_new || !v_new)
            return PKVQ_ERR_INVALID_ARG;
        if (!aligned16(k_new) || !aligned16(v_new))
            return PKVQ_ERR_MISALIGNED;
    }
    return decode_impl(cache, k_new, v_new, q, out, lse_out, block_table, max_blocks_per_seq,
                       context_lens, batch, q_len, num_q_heads, max_context_len, softmax_scale,
                       opts, workspace, workspace_bytes, stream);
}

pkvq_status pkvq_paged_attn_prefill(const pkvq_cache *cache, const void *q, void *out,
                                    float *lse_out, const int32_t *cu_seqlens_q,
                                    const int32_t *block_table, int32_t max_blocks_per_seq,
                                    const int32_t *context_lens, int32_t batch,
                                    int32_t max_q_len, int32_t num_q_heads,
                                    float softmax_scale, void *workspace,
                                    size_t workspace_bytes, void *stream)
{
    return pkvq_paged_attn_prefill_ex(cache, q, out, lse_out, cu_seqlens_q, block_table,
                                      max_blocks_per_seq, context_lens, batch, max_q_len,
                                      num_q_heads, softmax_scale, nullptr, workspace,
                                      workspace_bytes, stream);
}

pkvq_status pkvq_paged_attn_prefill_ex(const pkvq_cache *cache, const void *q, void *out,
                                       float *lse_out, const int32_t *cu_seqlens_q,
                                       const int32_t *block_table, int32_t max_blocks_per_seq,
                                       const int32_t *context_lens, int32_t batch,
                                       int32_t max_q_len, int32_t num_q_heads,
                                       float softmax_scale, const pkvq_attn_opts *opts,
                                       void *workspace, size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    if (opts && opts->sliding_window < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (opts && opts->query_pos)
        return PKVQ_ERR_UNSUPPORTED;
    pkvq_status st = check_cache(cache);
    if (st != PKVQ_OK)
        return st;
    if (batch < 0 || max_q_len < 0 || num_q_heads <= 0 || max_blocks_per_seq < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (num_q_heads % cache->num_kv_heads)
        return PKVQ_ERR_INVALID_ARG;
    const int group = num_q_heads / cache->num_kv_heads;
    if (group > 128)
        return PKVQ_ERR_UNSUPPORTED;
    if (!isfinite(softmax_scale))
        return PKVQ_ERR_INVALID_ARG;
    if (batch == 0 || max_q_len == 0)
        return PKVQ_OK;
    if (!q || !out || !cu_seqlens_q || !block_table || !context_lens)
        return PKVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out))
        return PKVQ_ERR_MISALIGNED;
    CUtensorMap km, vm;
    st = cache_maps(cache, &km, &vm);
    if (st != PKVQ_OK)
        return st;
    PrefillParams p{};
    p.k_cache = static_cast<const uint8_t *>(cache->k_cache);
    p.v_cache = static_cast<const uint8_t *>(cache->v_cache);
    const bool head_scale = kv_has_head_scale(cache->dtype);
    p.k_scale = head_scale ? cache->k_scale : nullptr;
    p.v_scale = head_scale ? cache->v_scale : nullptr;
    p.scale_stride = scale_stride(cache);
    p.window = opts ? opts->sliding_window : 0;
    p.k_scale_tok = static_cast<const uint16_t *>(cache->k_scale_tok);
    p.v_scale_tok = static_cast<const uint16_t *>(cache->v_scale_tok);
    p.q = static_cast<const __half *>(q);
    p.out = static_cast<__half *>(out);
    p.lse = lse_out;
    p.cu_seqlens_q = cu_seqlens_q;
    p.block_table = block_table;
    p.context_lens = context_lens;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.batch = batch;
    p.max_q_len = max_q_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.group = group;
    p.num_blocks = cache->num_blocks;
    p.block_size = cache->block_size;
    p.tokens_per_tile = 128 / group;   // 128 query rows per CTA
    p.q_tiles = (max_q_len + p.tokens_per_tile - 1) / p.tokens_per_tile;
    p.scale_log2 = softmax_scale * kLog2e;
    p.status = status_ptr();
    if (!p.status)
        return PKVQ_ERR_CUDA;
    return from_cuda(launch_prefill_tc(p, cache->dtype, km, vm, static_cast<cudaStream_t>(stream)));
}

pkvq_status pkvq_merge_attn_states(const void *parts_out, const float *parts_lse,
                                   int32_t num_parts, int64_t n_rows, int32_t head_dim,
                                   void *out, float *lse_out, void *stream)
{
    if (head_dim != kHeadDim)
        return PKVQ_ERR_UNSUPPORTED;
    if (num_parts < 1 || num_parts > 64 || n_rows < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (n_rows == 0)
        return PKVQ_OK;
    if (!parts_out || !parts_lse || !out)
        return PKVQ_ERR_INVALID_ARG;
    if (!aligned16(parts_out) || !aligned16(out))
        return PKVQ_ERR_MISALIGNED;
    MergeParams p{};
    p.parts_out = static_cast<const __half *>(parts_out);
    p.parts_lse = parts_lse;
    p.out = static_cast<__half *>(out);
    p.lse = lse_out;
    p.parts = num_parts;
    p.rows = n_rows;
    return from_cuda(launch_merge_states(p, static_cast<cudaStream_t>(stream)));
}

pkvq_status pkvq_kv_copy_blocks(const pkvq_cache *dst, const pkvq_cache *src,
                                const int32_t *pairs, int32_t n, void *stream)
{
    pkvq_status st = check_cache(dst);
    if (st != PKVQ_OK)
        return st;
    st = check_cache(src);
    if (st != PKVQ_OK)
        return st;
    if (dst->dtype != src->dtype || dst->block_size != src->block_size ||
        dst->num_kv_heads != src->num_kv_heads || dst->head_dim != src->head_dim)
        return PKVQ_ERR_INVALID_ARG;
    if (n < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (n == 0)
        return PKVQ_OK;
    if (!pairs)
        return PKVQ_ERR_INVALID_ARG;
    CopyParams p{};
    p.src_k = static_cast<const uint8_t *>(src->k_cache);
    p.src_v = static_cast<const uint8_t *>(src->v_cache);
    p.dst_k = static_cast<uint8_t *>(dst->k_cache);
    p.dst_v = static_cast<uint8_t *>(dst->v_cache);
    const bool int8 = src->dtype == PKVQ_KV_INT8;
    p.src_ks = int8 ? static_cast<const uint16_t *>(src->k_scale_tok) : nullptr;
    p.src_vs = int8 ? static_cast<const uint16_t *>(src->v_scale_tok) : nullptr;
    p.dst_ks = int8 ? static_cast<uint16_t *>(dst->k_scale_tok) : nullptr;
    p.dst_vs = int8 ? static_cast<uint16_t *>(dst->v_scale_tok) : nullptr;
    p.pairs = pairs;
    p.n = n;
    p.block_bytes = (long long)src->num_kv_heads * src->block_size * kHeadDim *
                    kv_elem_bytes(src->dtype);
    p.block_scales = int8 ? src->num_kv_heads * src->block_size : 0;
    p.src_blocks = src->num_blocks;
    p.dst_blocks = dst->num_blocks;
    p.status = status_ptr();
    if (!p.status)
        return PKVQ_ERR_CUDA;
    return from_cuda(launch_copy_blocks(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
