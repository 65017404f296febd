// KV write + quantize into the paged cache.
//
// Source: "ReVolta" PyPI page, "Weight and KV formats" (KV kept as 8-bit
// codes), "E4M3 KV" (static calibrated scales), "INT8 KV" (scales per token
// and head, computed at run time) and the first section's list of KV formats
// (E4M3, FP16, INT8); "1Cat-LLM" README ("FP8 E4M3 / E5M2 KV storage").
//
// One (token, KV head) row of head_dim = 128 fp16 values is handled by a
// group of 16 threads; each thread owns 8 consecutive elements, i.e. one
// 16-byte load of K and one of V.  (A group can take kRowsPerGroup rows and
// issue all of their loads before converting any; more than one row per group
// measured slower: the IEEE divisions of the FP8 formats then serialize per
// thread, and the one-token writes of a decode step lose most of their
// parallelism.)  The kernel is a single pass: 512 bytes read and 256 bytes
// of codes (512 for FP16, +4 bytes of INT8 scales) written per row.
#include "common.cuh"
#include "internal.h"

#include <cuda_fp8.h>

namespace pkvq {
namespace {

constexpr int kD = 128;
constexpr int kThreadsPerRow = 16;
constexpr int kElemsPerThread = 8;
constexpr int kBlockThreads = 256;
constexpr int kGroupsPerBlock = kBlockThreads / kThreadsPerRow;
constexpr int kRowsPerGroup = 1;
constexpr int kRowsPerBlock = kGroupsPerBlock * kRowsPerGroup;

// fp32 quotient -> E4M3 / E5M2 with round-to-nearest-even and saturation to
// the largest finite value (the hardware conversion with .satfinite).
template <int KVT>
__device__ __forceinline__ uint32_t quant_fp8x2(float a, float b)
{
    __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(
        make_float2(a, b), __NV_SATFINITE, KVT == kKvE5m2 ? __NV_E5M2 : __NV_E4M3);
    return (uint32_t)p;
}

// fp16 NaN -> the format's all-ones NaN (S.1111.111 / S.11111.11) with the
// input's own sign.  Decided on the fp16 bits: fp32 arithmetic on the GPU does
// not keep the sign of a NaN.
__device__ __forceinline__ uint32_t fix_nan(uint32_t code, uint16_t hbits)
{
    if ((hbits & 0x7c00u) == 0x7c00u && (hbits & 0x03ffu))
        return ((hbits >> 8) & 0x80u) | 0x7fu;
    return code;
}

// 8 fp16 values -> 8 FP8 codes of x / scale (scale == 0 -> codes 0).
template <int KVT>
__device__ __forceinline__ uint2 quant_fp8_8(const uint4 &x, float scale)
{
    if (scale == 0.0f)
        return make_uint2(0u, 0u);
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
    const uint16_t *hb = reinterpret_cast<const uint16_t *>(&x);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        const uint32_t pr = quant_fp8x2<KVT>(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
        c[i] = fix_nan(pr & 0xffu, hb[2 * i]) | (fix_nan((pr >> 8) & 0xffu, hb[2 * i + 1]) << 8);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ float absmax8(const uint4 &x)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

// Row scale s = fp16_rn(absmax / 127) over the 16-thread group (lanes of one
// half-warp); returns s as fp16 bits.
__device__ __forceinline__ uint16_t int8_row_scale(float local_absmax)
{
    float m = local_absmax;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return __half_as_ushort(__float2half_rn(__fdiv_rn(m, 127.0f)));
}

__device__ __forceinline__ uint2 quant_int8_8(const uint4 &x, uint16_t scale_bits)
{
    float s = __half2float(__ushort_as_half(scale_bits));
    if (s == 0.0f)
        return make_uint2(0u, 0u);
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        int a = __float2int_rn(__fdiv_rn(f.x, s));   // nearest, ties to even
        int b = __float2int_rn(__fdiv_rn(f.y, s));
        a = max(-127, min(127, a));
        b = max(-127, min(127, b));
        uint32_t pair = (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8);
        w[i >> 1] |= pair << (16 * (i & 1));
    }
    return make_uint2(w[0], w[1]);
}

template <int KVT>
__global__ void __launch_bounds__(kBlockThreads)
kv_write_quant_kernel(KvWriteParams p)
{
    // The next kernel (e.g. decode, launched with programmatic dependent
    // launch) may start its input-free prologue now; it waits for this grid to
    // finish before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int R = kRowsPerGroup;
    const int sub = threadIdx.x % kThreadsPerRow;
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    // rows of this group: row0 + i * kGroupsPerBlock (coalesced across groups)
    const long long row0 = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kThreadsPerRow;
    int slot[R], h[R];
    bool write[R];
    uint4 kx[R], vx[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const long long row = row0 + (long long)i * kGroupsPerBlock;
        const bool active = row < nrows;
        const int tok = active ? (int)(row / p.num_kv_heads) : 0;
        h[i] = active ? (int)(row % p.num_kv_heads) : 0;
        slot[i] = active ? __ldg(p.slot_mapping + tok) : -1;
        write[i] = slot[i] >= 0;
#ifdef PKVQ_BOUNDS_CHECK
        if (write[i] && (long long)slot[i] >= (long long)p.num_blocks * p.block_size) {
            if (sub == 0)
                atomicOr(p.status, kStatusBadBlock);
            write[i] = false;
        }
#endif
        // Every lane of a half-warp reaches the shuffle of the INT8 row scale,
        // so the loads are predicated rather than returned from early.
        kx[i] = make_uint4(0, 0, 0, 0);
        vx[i] = make_uint4(0, 0, 0, 0);
        const size_t src = ((size_t)tok * p.num_kv_heads + h[i]) * kD + sub * kElemsPerThread;
        if (write[i]) {
            kx[i] = __ldcs(reinterpret_cast<const uint4 *>(p.k + src));
            vx[i] = __ldcs(reinterpret_cast<const uint4 *>(p.v + src));
        }
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int blk = write[i] ? slot[i] / p.block_size : 0;
        const int off = write[i] ? slot[i] % p.block_size : 0;
        const size_t drow = ((size_t)blk * p.num_kv_heads + h[i]) * p.block_size + off;
        const size_t dst = drow * kD + sub * kElemsPerThread;
        if constexpr (KVT == kKvFp16) {
            if (write[i]) {
                *reinterpret_cast<uint4 *>(p.k_cache + dst * 2) = kx[i];
                *reinterpret_cast<uint4 *>(p.v_cache + dst * 2) = vx[i];
            }
        } else {
            uint2 kc, vc;
            if constexpr (kv_has_head_scale(KVT)) {
                const int hs = h[i] * p.scale_stride;
                kc = quant_fp8_8<KVT>(kx[i], write[i] ? __ldg(p.k_scale + hs) : 0.0f);
                vc = quant_fp8_8<KVT>(vx[i], write[i] ? __ldg(p.v_scale + hs) : 0.0f);
            } else {
                uint16_t ks = int8_row_scale(absmax8(kx[i]));
                uint16_t vs = int8_row_scale(absmax8(vx[i]));
                kc = quant_int8_8(kx[i], ks);
                vc = quant_int8_8(vx[i], vs);
                if (write[i] && sub == 0) {
                    p.k_scale_tok[drow] = ks;
                    p.v_scale_tok[drow] = vs;
                }
            }
            if (write[i]) {
                *reinterpret_cast<uint2 *>(p.k_cache + dst) = kc;
                *reinterpret_cast<uint2 *>(p.v_cache + dst) = vc;
            }
        }
    }
}

}  // namespace

cudaError_t launch_kv_write_quant(const KvWriteParams &p, int kv_dtype, cudaStream_t stream)
{
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    if (nrows == 0)
        return cudaSuccess;
    const unsigned grid = (unsigned)((nrows + kRowsPerBlock - 1) / kRowsPerBlock);
    switch (kv_dtype) {
    case kKvFp8: kv_write_quant_kernel<kKvFp8><<<grid, kBlockThreads, 0, stream>>>(p); break;
    case kKvInt8: kv_write_quant_kernel<kKvInt8><<<grid, kBlockThreads, 0, stream>>>(p); break;
    case kKvE5m2: kv_write_quant_kernel<kKvE5m2><<<grid, kBlockThreads, 0, stream>>>(p); break;
    case kKvFp16: kv_write_quant_kernel<kKvFp16><<<grid, kBlockThreads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace pkvq
