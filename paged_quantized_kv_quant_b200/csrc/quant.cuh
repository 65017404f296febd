// Quantisation of fp16 K/V rows to the cache formats, shared by the KV write
// kernel and the decode kernel's appending form (which writes the step's new
// tokens itself).
//
// Source: "ReVolta" PyPI page, "Weight and KV formats" ("E4M3 KV": static
// calibrated scales; "INT8 KV": scales per token and head computed at run
// time); "1Cat-LLM" README ("FP8 E4M3 / E5M2 KV storage").
//
// Codes without a division per element.  A code is the format's rounding of
// the correctly rounded fp32 quotient RN(x / s).  With r = RN(1 / s),
// r_lo = RN(r (1 - 2^-20)) and r_hi = RN(r (1 + 2^-20)), the products
// RN(x r_lo) and RN(x r_hi) lie strictly below and above RN(x / s) in
// magnitude (each factor is off by at most 2^-24 relatively, far less than
// the 2^-20 margin), and rounding to a code is monotonic: when both products
// give the same code, so does the quotient.  Otherwise -- a quotient within
// about 2^-20 of a rounding boundary, a few in a million -- the thread
// divides.  Products below the fp32 normal range round to a zero code on
// both sides, as does the quotient; scales whose reciprocal leaves the
// normal range always divide.
#pragma once

#include "common.cuh"
#include "internal.h"

#include <cuda_fp8.h>

namespace pkvq {

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

// True if one of the 8 fp16 values is a NaN (exponent all ones, mantissa
// non-zero): ((h & 0x7fff) + 0x3ff) carries into bit 15 exactly then.
__device__ __forceinline__ bool any_nan8(const uint4 &x)
{
    const uint32_t m = 0x7fff7fffu, k = 0x03ff03ffu;
    const uint32_t t = ((x.x & m) + k) | ((x.y & m) + k) | ((x.z & m) + k) | ((x.w & m) + k);
    return (t & 0x80008000u) != 0u;
}

// Reciprocal brackets of a positive scale (see the file comment); false if
// the products cannot be trusted (the reciprocal is not a normal number with
// room to spare), in which case the caller divides.
__device__ __forceinline__ bool recip_bracket(float s, float &r_lo, float &r_hi)
{
    const float r = __frcp_rn(s);
    r_lo = __fmul_rn(r, 1.0f - 0x1p-20f);
    r_hi = __fmul_rn(r, 1.0f + 0x1p-20f);
    return s > 0x1p-120f && s < 0x1p120f;
}

// 8 fp16 values -> 8 FP8 codes of x / scale (scale == 0 -> codes 0).
template <int KVT>
__device__ __forceinline__ uint2 quant_fp8_8(const uint4 &x, float scale, float r_lo, float r_hi,
                                             bool fast)
{
    if (scale == 0.0f)
        return make_uint2(0u, 0u);
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
    uint32_t c[4];
    bool same = fast;
    if (fast) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            const uint32_t lo = quant_fp8x2<KVT>(__fmul_rn(f.x, r_lo), __fmul_rn(f.y, r_lo));
            const uint32_t hi = quant_fp8x2<KVT>(__fmul_rn(f.x, r_hi), __fmul_rn(f.y, r_hi));
            same &= lo == hi;
            c[i] = lo;
        }
    }
    if (!same) {   // a quotient next to a rounding boundary (or no brackets)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            c[i] = quant_fp8x2<KVT>(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
        }
    }
    if (any_nan8(x)) {
        const uint16_t *hb = reinterpret_cast<const uint16_t *>(&x);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            c[i] = fix_nan(c[i] & 0xffu, hb[2 * i]) | (fix_nan((c[i] >> 8) & 0xffu, hb[2 * i + 1]) << 8);
    }
    return make_uint2((c[0] & 0xffffu) | (c[1] << 16), (c[2] & 0xffffu) | (c[3] << 16));
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

// rint(q) for |q| < 2^22 as the bits of RN(q + 1.5 * 2^23): the integer sits
// in the low mantissa bits (ties to even, as rint).
__device__ __forceinline__ uint32_t rint_bits(float q)
{
    return __float_as_uint(__fadd_rn(q, 12582912.0f));
}

__device__ __forceinline__ uint32_t int8_code(uint32_t rbits)
{
    const int v = (int)rbits - (int)0x4B400000;   // bits of 1.5 * 2^23
    return (uint32_t)(max(-127, min(127, v)) & 0xff);
}

// 8 fp16 values -> 8 INT8 codes clamp(rint(x / s), -127, 127) (s == 0 ->
// codes 0).  |x / s| stays near 127 at most, far inside rint_bits' range.
__device__ __forceinline__ uint2 quant_int8_8(const uint4 &x, uint16_t scale_bits)
{
    const float s = __half2float(__ushort_as_half(scale_bits));
    if (s == 0.0f)
        return make_uint2(0u, 0u);
    float r_lo, r_hi;
    recip_bracket(s, r_lo, r_hi);   // an fp16 scale's reciprocal is always normal
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
    uint32_t w[2] = {0u, 0u};
    bool same = true;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        const uint32_t la = rint_bits(__fmul_rn(f.x, r_lo)), ha = rint_bits(__fmul_rn(f.x, r_hi));
        const uint32_t lb = rint_bits(__fmul_rn(f.y, r_lo)), hb = rint_bits(__fmul_rn(f.y, r_hi));
        same &= (la == ha) & (lb == hb);
        w[i >> 1] |= (int8_code(la) | (int8_code(lb) << 8)) << (16 * (i & 1));
    }
    if (!same) {   // a quotient next to a half-integer: divide
        w[0] = w[1] = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            const uint32_t a = int8_code(rint_bits(__fdiv_rn(f.x, s)));
            const uint32_t b = int8_code(rint_bits(__fdiv_rn(f.y, s)));
            w[i >> 1] |= (a | (b << 8)) << (16 * (i & 1));
        }
    }
    return make_uint2(w[0], w[1]);
}

// One thread's 8 elements (16-byte piece `sub` of 16) of a (token, KV head)
// row of K or V: the codes go to element offset drow * 128 + 8 sub of
// `cache` and, for INT8, the row scale to scale_tok[drow] (by piece 0).
// FP8 formats divide by head_scale (a per-head or per-layer value).  All 16
// threads of the row (one half-warp) take part, `write` or not: the INT8 row
// scale is a half-warp reduction.
template <int KVT>
__device__ __forceinline__ void quant_store_piece(uint8_t *cache, uint16_t *scale_tok,
                                                  float head_scale, size_t drow, int sub,
                                                  const uint4 &x, bool write)
{
    const size_t dst = drow * 128 + (size_t)sub * 8;
    if constexpr (KVT == kKvFp16) {
        if (write)
            *reinterpret_cast<uint4 *>(cache + dst * 2) = x;
    } else {
        uint2 c;
        if constexpr (kv_has_head_scale(KVT)) {
            const float sc = write ? head_scale : 0.0f;
            float lo, hi;
            const bool fast = recip_bracket(sc, lo, hi);
            c = quant_fp8_8<KVT>(x, sc, lo, hi, fast);
        } else {
            const uint16_t sb = int8_row_scale(absmax8(x));
            c = quant_int8_8(x, sb);
            if (write && sub == 0)
                scale_tok[drow] = sb;
        }
        if (write)
            *reinterpret_cast<uint2 *>(cache + dst) = c;
    }
}

}  // namespace pkvq
