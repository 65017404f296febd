// Decode attention for callers that cannot allocate device memory.
//
// pkvq_paged_attn_decode needs a scratch workspace for its split-KV partial
// results, and the caller normally allocates it.  Some callers cannot: a
// serving engine that has handed almost all of HBM to its KV pool and its
// caching allocator (a fresh cudaMalloc would fail or fragment the pool), a
// plugin inside a host framework that owns every allocation, or code that must
// not allocate on its steady-state path because an allocation can block or
// synchronize the device.  This entry point uses a fixed scratch array that is
// compiled into the library instead.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes; every
// GPU that loads the library holds it until the process exits.  In host code
// its name is only a host-side handle, so its device address is looked up once
// per device with cudaGetSymbolAddress (with that device current) and passed
// to the kernels like any other workspace pointer.
//
// Sharing: all calls on a device use the same array.  Calls that could run at
// the same time on the device (different streams without ordering between
// them) race on it and must be serialized by the caller.  The decode kernels
// write every scratch word they later read within the same call, so the array
// needs no clearing between calls.
#include "../../include/pkvq.h"
#include "internal.h"

#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device, looked up on the
// first call per device.  Returns nullptr if the lookup fails.
void *scratch_on_current_device()
{
    static void *addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p)
            return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" PKVQ_API pkvq_status pkvq_paged_attn_decode_noalloc(
    const pkvq_cache *cache, const void *q, void *out, float *lse_out,
    const int32_t *block_table, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t max_context_len,
    float softmax_scale, void *stream)
{
    if (batch < 0)
        return PKVQ_ERR_INVALID_ARG;
    if (batch > 0) {
        const size_t need =
            pkvq_decode_workspace_bytes(batch, q_len, num_q_heads, max_context_len, cache);
        if (need > kNoAllocScratchBytes)
            return PKVQ_ERR_WORKSPACE_TOO_SMALL;   // shape needs more than the fixed array
    }
    void *scratch = scratch_on_current_device();
    if (!scratch)
        return PKVQ_ERR_CUDA;
    return pkvq_paged_attn_decode(cache, q, out, lse_out, block_table, max_blocks_per_seq,
                                  context_lens, batch, q_len, num_q_heads, max_context_len,
                                  softmax_scale, scratch, kNoAllocScratchBytes, stream);
}
