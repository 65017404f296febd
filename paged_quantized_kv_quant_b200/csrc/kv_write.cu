// KV write + quantize into the paged cache.
//
// Source: "ReVolta" PyPI page, "Weight and KV formats" (KV kept as 8-bit
// codes), "E4M3 KV" (static calibrated scales) and "INT8 KV" (scales per
// token and head, computed at run time).
//
// One (token, KV head) row of head_dim = 128 fp16 values is handled by a
// group of 16 threads; each thread owns 8 consecutive elements, i.e. one
// 16-byte load of K and one of V and one 8-byte store of codes each.  The
// kernel is a single bandwidth-bound pass: 512 bytes read and 256 bytes of
// codes (+4 bytes of INT8 scales) written per row.
#include "common.cuh"
#include "internal.h"

#include <cuda_fp8.h>

namespace pkvq {
namespace {

constexpr int kD = 128;
constexpr int kThreadsPerRow = 16;
constexpr int kElemsPerThread = 8;
constexpr int kBlockThreads = 256;
constexpr int kRowsPerBlock = kBlockThreads / kThreadsPerRow;

// fp32 quotient -> E4M3 with round-to-nearest-even and saturation to +-448
// (the hardware conversion with .satfinite).
__device__ __forceinline__ uint32_t quant_e4m3x2(float a, float b)
{
    __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)p;
}

// fp16 NaN -> S.1111.111 with the input's own sign.  Decided on the fp16 bits:
// fp32 arithmetic on the GPU does not keep the sign of a NaN.
__device__ __forceinline__ uint32_t fix_nan(uint32_t code, uint16_t hbits)
{
    if ((hbits & 0x7c00u) == 0x7c00u && (hbits & 0x03ffu))
        return ((hbits >> 8) & 0x80u) | 0x7fu;
    return code;
}

// 8 fp16 values -> 8 E4M3 codes of x / scale (scale == 0 -> codes 0).
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
        const uint32_t pr = quant_e4m3x2(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
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
    const int row = blockIdx.x * kRowsPerBlock + threadIdx.x / kThreadsPerRow;
    const int sub = threadIdx.x % kThreadsPerRow;
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    const bool active = row < nrows;
    const int tok = active ? row / p.num_kv_heads : 0;
    const int h = active ? row % p.num_kv_heads : 0;
    int slot = active ? __ldg(p.slot_mapping + tok) : -1;
    bool write = slot >= 0;
#ifdef PKVQ_BOUNDS_CHECK
    if (write && (long long)slot >= (long long)p.num_blocks * p.block_size) {
        if (sub == 0)
            atomicOr(p.status, kStatusBadBlock);
        write = false;
    }
#endif
    // Every lane of a half-warp reaches the shuffle in int8_row_scale, so the
    // loads are predicated rather than returned from early.
    uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
    const size_t src = ((size_t)tok * p.num_kv_heads + h) * kD + sub * kElemsPerThread;
    if (write) {
        kx = __ldcs(reinterpret_cast<const uint4 *>(p.k + src));
        vx = __ldcs(reinterpret_cast<const uint4 *>(p.v + src));
    }
    const int blk = write ? slot / p.block_size : 0;
    const int off = write ? slot % p.block_size : 0;
    const size_t drow = ((size_t)blk * p.num_kv_heads + h) * p.block_size + off;
    const size_t dst = drow * kD + sub * kElemsPerThread;
    uint2 kc, vc;
    if constexpr (KVT == kKvFp8) {
        kc = quant_fp8_8(kx, write ? __ldg(p.k_scale + h) : 0.0f);
        vc = quant_fp8_8(vx, write ? __ldg(p.v_scale + h) : 0.0f);
    } else {
        uint16_t ks = int8_row_scale(absmax8(kx));
        uint16_t vs = int8_row_scale(absmax8(vx));
        kc = quant_int8_8(kx, ks);
        vc = quant_int8_8(vx, vs);
        if (write && sub == 0) {
            p.k_scale_tok[drow] = ks;
            p.v_scale_tok[drow] = vs;
        }
    }
    if (write) {
        *reinterpret_cast<uint2 *>(p.k_cache + dst) = kc;
        *reinterpret_cast<uint2 *>(p.v_cache + dst) = vc;
    }
}

}  // namespace

cudaError_t launch_kv_write_quant(const KvWriteParams &p, int kv_dtype, cudaStream_t stream)
{
    const long long nrows = (long long)p.num_tokens * p.num_kv_heads;
    if (nrows == 0)
        return cudaSuccess;
    const unsigned grid = (unsigned)((nrows + kRowsPerBlock - 1) / kRowsPerBlock);
    if (kv_dtype == kKvFp8)
        kv_write_quant_kernel<kKvFp8><<<grid, kBlockThreads, 0, stream>>>(p);
    else
        kv_write_quant_kernel<kKvInt8><<<grid, kBlockThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pkvq
