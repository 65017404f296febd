// Merge of attention results computed over disjoint key sets of the same
// queries (pkvq_merge_attn_states).
//
// Source: "ReVolta" PyPI page, "Hardware" and launch flags (TP4 + DCP2: each
// rank of a decode-context-parallel group holds part of every sequence's
// keys); "1Cat-LLM" README, "Layer 2" (partial softmax states merged in
// FP32).  With lse_r the natural-log sum-exp of part r's scores and out_r its
// normalised output, the softmax over the union of the keys is
//   lse = ln sum_r e^lse_r,   out = sum_r e^(lse_r - lse) out_r.
//
// One warp per output row; lane i owns elements 4i .. 4i+3 (8 bytes of the
// fp16 row).  The warp reads every part's lse first (two per lane), reduces
// the maximum with shuffles, then issues the row loads of 8 parts at a time
// before accumulating any of them.
#include "common.cuh"
#include "internal.h"

#include <math.h>

namespace pkvq {
namespace {

constexpr int kParts = 64;        // parts per call (two per lane)
constexpr int kRowLoads = 8;      // part rows in flight per lane

__global__ void __launch_bounds__(256) merge_states_kernel(const MergeParams p)
{
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= p.rows)
        return;
    // every part's lse: lane i holds parts i and i + 32
    const float l0 = lane < p.parts ? p.parts_lse[(size_t)lane * p.rows + row] : -INFINITY;
    const float l1 = lane + 32 < p.parts ? p.parts_lse[(size_t)(lane + 32) * p.rows + row]
                                         : -INFINITY;
    float m = fmaxf(l0, l1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    uint2 *dst = reinterpret_cast<uint2 *>(p.out + row * kHeadDim) + lane;
    if (m == -INFINITY) {   // no part saw a key
        *dst = make_uint2(0u, 0u);
        if (lane == 0 && p.lse)
            p.lse[row] = -INFINITY;
        return;
    }
    // weights relative to the maximum, and their sum
    const float e0 = expf(l0 - m), e1 = expf(l1 - m);
    float sum = e0 + e1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r0 = 0; r0 < p.parts; r0 += kRowLoads) {
        uint2 x[kRowLoads];
        float w[kRowLoads];
#pragma unroll
        for (int k = 0; k < kRowLoads; ++k) {
            const int r = r0 + k;
            // part r's weight lives in lane r % 32 (e0 for r < 32, e1 above)
            const float e = __shfl_sync(0xffffffffu, r < 32 ? e0 : e1, r & 31);
            w[k] = r < p.parts ? e * inv : 0.0f;
            x[k] = make_uint2(0u, 0u);
            if (r < p.parts && w[k] != 0.0f)
                x[k] = reinterpret_cast<const uint2 *>(
                    p.parts_out + ((size_t)r * p.rows + row) * kHeadDim)[lane];
        }
#pragma unroll
        for (int k = 0; k < kRowLoads; ++k) {
            const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&x[k].x));
            const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&x[k].y));
            acc[0] += w[k] * a.x, acc[1] += w[k] * a.y;
            acc[2] += w[k] * b.x, acc[3] += w[k] * b.y;
        }
    }
    const __half2 lo = __floats2half2_rn(acc[0], acc[1]);
    const __half2 hi = __floats2half2_rn(acc[2], acc[3]);
    *dst = make_uint2(*reinterpret_cast<const uint32_t *>(&lo),
                      *reinterpret_cast<const uint32_t *>(&hi));
    if (lane == 0 && p.lse)
        p.lse[row] = m + logf(sum);
}

}  // namespace

cudaError_t launch_merge_states(const MergeParams &p, cudaStream_t stream)
{
    if (p.rows <= 0)
        return cudaSuccess;
    if (p.parts < 1 || p.parts > kParts)
        return cudaErrorInvalidValue;
    const long long blocks = (p.rows + 7) / 8;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    merge_states_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pkvq
