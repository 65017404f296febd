// KV write + quantize into the paged cache.
//
// Source: "ReVolta" PyPI page, "Weight and KV formats" (KV kept as 8-bit
// codes), "E4M3 KV" (static calibrated scales), "INT8 KV" (scales per token
// and head, computed at run time) and the first section's list of KV formats
// (E4M3, FP16, INT8); "1Cat-LLM" README ("FP8 E4M3 / E5M2 KV storage").
//
// One (token, KV head) row of head_dim = 128 fp16 values is handled by a
// group of 16 threads; each thread owns 8 consecutive elements, i.e. one
// 16-byte load of K and one of V.  The kernel is a single pass: 512 bytes
// read and 256 bytes of codes (512 for FP16, +4 bytes of INT8 scales)
// written per row.
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace pkvq {
namespace {

constexpr int kD = 128;
constexpr int kThreadsPerRow = 16;
constexpr int kElemsPerThread = 8;
constexpr int kBlockThreads = 256;
constexpr int kTokensPerBlock = kBlockThreads / kThreadsPerRow;

// Grid: x = token groups of 16, y = KV head, so that no thread divides by a
// run-time value (the block size is a template parameter).
template <int KVT, int BS>
__global__ void __launch_bounds__(kBlockThreads)
kv_write_quant_kernel(KvWriteParams p)
{
    // The next kernel (e.g. decode, launched with programmatic dependent
    // launch) may start its input-free prologue now; it waits for this grid to
    // finish before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int sub = threadIdx.x % kThreadsPerRow;
    const int h = blockIdx.y;
    const long long tl = (long long)blockIdx.x * kTokensPerBlock + threadIdx.x / kThreadsPerRow;
    const bool active = tl < p.num_tokens;
    const int tok = active ? (int)tl : 0;
    int slot = -1;
    if (active) {
        if (p.slot_mapping) {
            slot = __ldg(p.slot_mapping + tok);
        } else {
            // the step's new tokens: token t of sequence b is the sequence's
            // position ctx - q_len + t, in the block the table gives it
            const int b = tok / p.q_len, t = tok % p.q_len;
            const int pos = __ldg(p.context_lens + b) - p.q_len + t;
            if (pos >= 0 && pos / BS < p.max_blocks_per_seq)
                slot = __ldg(p.block_table + (size_t)b * p.max_blocks_per_seq + pos / BS) * BS +
                       pos % BS;
        }
    }
    bool write = slot >= 0;
#ifdef PKVQ_BOUNDS_CHECK
    if (write && (long long)slot >= (long long)p.num_blocks * BS) {
        if (sub == 0)
            atomicOr(p.status, kStatusBadBlock);
        write = false;
    }
#endif
    // Every lane of a half-warp reaches the shuffle of the INT8 row scale,
    // so the loads are predicated rather than returned from early.
    uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
    const size_t src = ((size_t)tok * p.num_kv_heads + h) * kD + sub * kElemsPerThread;
    if (write) {
        kx = __ldcs(reinterpret_cast<const uint4 *>(p.k + src));
        vx = __ldcs(reinterpret_cast<const uint4 *>(p.v + src));
    }
    const int blk = write ? slot / BS : 0;
    const int off = write ? slot % BS : 0;
    const size_t drow = ((size_t)blk * p.num_kv_heads + h) * BS + off;
    float ks = 0.0f, vs = 0.0f;
    if constexpr (kv_has_head_scale(KVT)) {
        if (write) {
            ks = __ldg(p.k_scale + h * p.scale_stride);
            vs = __ldg(p.v_scale + h * p.scale_stride);
        }
    }
    quant_store_piece<KVT>(p.k_cache, p.k_scale_tok, ks, drow, sub, kx, write);
    quant_store_piece<KVT>(p.v_cache, p.v_scale_tok, vs, drow, sub, vx, write);
}

template <int KVT>
cudaError_t launch_kw(const KvWriteParams &p, dim3 grid, cudaStream_t stream)
{
    switch (p.block_size) {
    case 16: kv_write_quant_kernel<KVT, 16><<<grid, kBlockThreads, 0, stream>>>(p); break;
    case 32: kv_write_quant_kernel<KVT, 32><<<grid, kBlockThreads, 0, stream>>>(p); break;
    case 64: kv_write_quant_kernel<KVT, 64><<<grid, kBlockThreads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_write_quant(const KvWriteParams &p, int kv_dtype, cudaStream_t stream)
{
    if (p.num_tokens == 0 || p.num_kv_heads == 0)
        return cudaSuccess;
    const dim3 grid((unsigned)((p.num_tokens + kTokensPerBlock - 1) / kTokensPerBlock),
                    (unsigned)p.num_kv_heads);
    switch (kv_dtype) {
    case kKvFp8: return launch_kw<kKvFp8>(p, grid, stream);
    case kKvInt8: return launch_kw<kKvInt8>(p, grid, stream);
    case kKvE5m2: return launch_kw<kKvE5m2>(p, grid, stream);
    case kKvFp16: return launch_kw<kKvFp16>(p, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
