// Whole-block copies between two paged caches (pkvq_kv_copy_blocks): the
// gather/scatter of a KV offload tier.
//
// Source: "ReVolta" PyPI page, "KV offload modes" (cached pages kept in CPU
// memory or on disk and brought back instead of recomputed).  A block is
// contiguous in each pool ([num_blocks][Hkv][block_size][128] elements, and
// INT8 scales [num_blocks][Hkv][block_size]), so a block copy is three or
// five contiguous runs.  One CTA per (source, destination) pair streams them
// with 16-byte loads and stores; either pool may be device memory or host
// memory the device can address (pinned and mapped), so the same kernel
// gathers pages out to a host tier and scatters them back.
#include "common.cuh"
#include "internal.h"

namespace pkvq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // 16-byte loads in flight per thread

__device__ __forceinline__ void copy_run(uint8_t *dst, const uint8_t *src, long long bytes)
{
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    const long long n = bytes / 16;
    for (long long i0 = threadIdx.x; i0 < n; i0 += (long long)kThreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long i = i0 + (long long)u * kThreads;
            if (i < n)
                v[u] = s[i];
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const long long i = i0 + (long long)u * kThreads;
            if (i < n)
                d[i] = v[u];
        }
    }
}

__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(const CopyParams p)
{
    const int i = blockIdx.x;
    const int src = p.pairs[2 * i], dst = p.pairs[2 * i + 1];
#ifdef PKVQ_BOUNDS_CHECK
    if (src < 0 || src >= p.src_blocks || dst < 0 || dst >= p.dst_blocks) {
        if (threadIdx.x == 0)
            atomicOr(p.status, kStatusBadBlock);
        return;
    }
#endif
    copy_run(p.dst_k + (size_t)dst * p.block_bytes, p.src_k + (size_t)src * p.block_bytes,
             p.block_bytes);
    copy_run(p.dst_v + (size_t)dst * p.block_bytes, p.src_v + (size_t)src * p.block_bytes,
             p.block_bytes);
    if (p.block_scales) {
        const long long sb = (long long)p.block_scales * 2;
        copy_run(reinterpret_cast<uint8_t *>(p.dst_ks) + (size_t)dst * sb,
                 reinterpret_cast<const uint8_t *>(p.src_ks) + (size_t)src * sb, sb);
        copy_run(reinterpret_cast<uint8_t *>(p.dst_vs) + (size_t)dst * sb,
                 reinterpret_cast<const uint8_t *>(p.src_vs) + (size_t)src * sb, sb);
    }
}

}  // namespace

cudaError_t launch_copy_blocks(const CopyParams &p, cudaStream_t stream)
{
    if (p.n <= 0)
        return cudaSuccess;
    copy_blocks_kernel<<<p.n, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pkvq
