// Split-KV decode / draft-verify attention over the paged 8-bit cache.
//
// Source: "1Cat-LLM" README, "Layer 1" (paged KV is read through page ids
// with wide aligned loads, the page id reused for a whole page), "Layer 2"
// (GQA multi-head packing into wider tensor-core work, online softmax with
// FP32 state, Split-KV with an FP32 merge of the partial states) and
// "128-bit Loads" (fewer, wider, aligned cache loads).
//
// Work decomposition.  A CTA owns one (sequence, KV head, row group, split):
// the rows are the q_len x G query rows that share the KV head (GQA packing),
// the split is a contiguous range of cache blocks.  Every (KV head, row group)
// gets the same number C of CTA slots; slot c is mapped on the device, from
// the context lengths, to a sequence and a split of it, each sequence getting
// splits in proportion to its length (at least one), so that sequences of
// different lengths still give every CTA about the same work.  Each of its 4
// warps
// streams whole cache blocks (block_size x 128 codes of K and of V, one
// contiguous tile each) through a private ring of TMA stages: lane 0 issues a
// 2-D tensor copy per tile with 128-byte swizzle, so the fragment loads below
// are free of shared-memory bank conflicts.
//
// Tensor-core mapping (legacy mma.sync m16n8k16, fp16 x fp16 -> fp32).  The
// contraction puts KEYS on M and query ROWS on N: S^T = K Q^T and
// O^T += V^T P^T.  With G = 8 a decode step's rows fill one n8 tile exactly,
// so no tensor-core work is padded.  Codes are converted to fp16 in registers
// straight into A fragments (E4M3 and int8 values are exact in fp16); the head
// dimension is permuted consistently between Q and K so that every thread
// reads 32 contiguous code bytes per key.  P^T reaches the B-operand layout
// through movmatrix.trans, without shared memory.
//
// Scales.  FP8 (E4M3, E5M2): the per-head (or per-layer) K scale folds into
// the score multiplier and the V scale into the final normalisation.  INT8:
// the per-token K scale multiplies score columns in fp32; the per-token V
// scale multiplies the dequantised V in fp16 before the PV product (P itself
// stays unscaled, so small probabilities never meet small scales in fp16).
// FP16 caches hold the values themselves: a row of 128 values is 256 bytes,
// fetched as two 128-byte-wide boxes (d 0-63, d 64-127) and read straight
// into the MMA fragments.
//
// Visibility.  Key j is visible to a query row at position pos iff j <= pos,
// j < context length and, with a sliding window w, j > pos - w ("1Cat-LLM"
// README, "DFlash2 Long-Context Decay").  Positions are context - q_len + t,
// or given per query (a rank holding part of each sequence's keys).
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"
#include "split_map.cuh"

#include <math.h>

namespace pkvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr float kLn2 = 0.693147180559945309f;

template <int KVT, int BS>
struct DecodeCfg {
    static constexpr int kEB = kv_elem_bytes(KVT);
    // bytes of one (block, head) tile per warp stage; FP16 tiles are twice as
    // large, so they take fewer stages
    static constexpr int kTileBytes = BS * 128 * kEB;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kStages =
        kEB == 1 ? (BS == 16 ? 4 : (BS == 32 ? 3 : 2)) : (BS == 16 ? 3 : (BS == 32 ? 2 : 1));
    static constexpr int kUnroll = (BS == 16 && kEB == 1) ? 2 : 1;   // blocks per loop iteration
    static constexpr int kScaleHalves = 2 * BS;     // K then V scales of one block
    static constexpr int kMT = BS / 16;             // 16-key m-tiles per block
    static_assert(kStages >= kUnroll, "ring must hold one iteration");
};

template <int KVT, int BS>
constexpr size_t decode_smem_bytes()
{
    using C = DecodeCfg<KVT, BS>;
    return 1024 + (size_t)kWarps * C::kStages * C::kStageBytes +
           (size_t)kWarps * C::kStages * C::kScaleHalves * 2 + (size_t)kWarps * C::kStages * 8;
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p)
{
    return *reinterpret_cast<const uint4 *>(p);
}

template <int KVT>
__device__ __forceinline__ void cvt4(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    if constexpr (KVT == kKvFp8)
        e4m3x4_to_half2x2(x, lo, hi);
    else if constexpr (KVT == kKvE5m2)
        e5m2x4_to_half2x2(x, lo, hi);
    else
        s8x4_to_half2x2(x, lo, hi);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b)
{
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// S^T = K Q^T for one cache block (MT m-tiles of 16 keys), scaled to log2
// units.  Lane (g, t) reads 32 contiguous code bytes of keys g and g+8 of each
// m-tile; the swizzled 16-byte chunk c of row r sits at c ^ (r & 7).
template <int KVT, int NT, int MT>
__device__ __forceinline__ void qk_block(const uint8_t *kt, const uint16_t *st, int g, int t,
                                         const uint32_t (&qf)[NT][8][2], float kfac,
                                         float (&sc)[MT][NT][4])
{
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int r0 = mt * 16 + g;   // rows r0, r0 + 8 share (row & 7) == g
        const uint4 ka0 = lds128(kt + r0 * 128 + (((2 * t) ^ g) << 4));
        const uint4 ka1 = lds128(kt + r0 * 128 + (((2 * t + 1) ^ g) << 4));
        const uint4 kb0 = lds128(kt + (r0 + 8) * 128 + (((2 * t) ^ g) << 4));
        const uint4 kb1 = lds128(kt + (r0 + 8) * 128 + (((2 * t + 1) ^ g) << 4));
        const uint32_t wa[8] = {ka0.x, ka0.y, ka0.z, ka0.w, ka1.x, ka1.y, ka1.z, ka1.w};
        const uint32_t wb[8] = {kb0.x, kb0.y, kb0.z, kb0.w, kb1.x, kb1.y, kb1.z, kb1.w};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                sc[mt][nt][c] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a[4];
            cvt4<KVT>(wa[ks], a[0], a[2]);   // key g:   d = 32t+4ks+{0,1} | {2,3}
            cvt4<KVT>(wb[ks], a[1], a[3]);   // key g+8
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_f16_16816(sc[mt][nt], a, qf[nt][ks]);
        }
        float f0 = kfac, f1 = kfac;
        if constexpr (KVT == kKvInt8) {
            f0 *= __half2float(__ushort_as_half(st[r0]));
            f1 *= __half2float(__ushort_as_half(st[r0 + 8]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sc[mt][nt][0] *= f0, sc[mt][nt][1] *= f0;
            sc[mt][nt][2] *= f1, sc[mt][nt][3] *= f1;
        }
    }
}

// O^T += V^T P^T for one cache block.  Lane (g, t) reads the 16-byte chunk g
// (d = 16g .. 16g+15) of keys 2t, 2t+1, 2t+8, 2t+9 of each m-tile; one byte
// permute pairs two keys' codes for two d rows at once.
template <int KVT, int NT, int MT, int BS>
__device__ __forceinline__ void pv_block(const uint8_t *vt, const uint16_t *st, int g, int t,
                                         int key0, int ctx, const float (&pr)[MT][NT][4],
                                         float (&o)[NT][8][4])
{
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            pb[nt][0] = movmatrix_trans(pack_half2(pr[mt][nt][0], pr[mt][nt][1]));
            pb[nt][1] = movmatrix_trans(pack_half2(pr[mt][nt][2], pr[mt][nt][3]));
        }
        const int r0 = mt * 16 + 2 * t;   // key rows r0, r0+1, r0+8, r0+9
        uint4 v0 = lds128(vt + r0 * 128 + ((g ^ (r0 & 7)) << 4));
        uint4 v1 = lds128(vt + (r0 + 1) * 128 + ((g ^ ((r0 + 1) & 7)) << 4));
        uint4 v2 = lds128(vt + (r0 + 8) * 128 + ((g ^ ((r0 + 8) & 7)) << 4));
        uint4 v3 = lds128(vt + (r0 + 9) * 128 + ((g ^ ((r0 + 9) & 7)) << 4));
        uint32_t s01 = 0u, s23 = 0u;
        if constexpr (KVT == kKvInt8) {
            s01 = (uint32_t)st[BS + r0] | ((uint32_t)st[BS + r0 + 1] << 16);
            s23 = (uint32_t)st[BS + r0 + 8] | ((uint32_t)st[BS + r0 + 9] << 16);
        }
        if (key0 + BS > ctx) {
            // Slots past the context were never written: their codes (and
            // INT8 scales) may be NaN patterns, and 0 * NaN would poison O.
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            const int k0 = key0 + r0;
            if (k0 >= ctx) v0 = z, s01 &= 0xffff0000u;
            if (k0 + 1 >= ctx) v1 = z, s01 &= 0x0000ffffu;
            if (k0 + 8 >= ctx) v2 = z, s23 &= 0xffff0000u;
            if (k0 + 9 >= ctx) v3 = z, s23 &= 0x0000ffffu;
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t x0 = word_of(v0, w), x1 = word_of(v1, w);
            const uint32_t x2 = word_of(v2, w), x3 = word_of(v3, w);
#pragma unroll
            for (int hw = 0; hw < 2; ++hw) {   // d-tile dt = 2w + hw: bytes 4w+2hw, 4w+2hw+1
                const uint32_t sel = hw ? 0x7362u : 0x5140u;
                uint32_t a[4];
                cvt4<KVT>(__byte_perm(x0, x1, sel), a[0], a[1]);
                cvt4<KVT>(__byte_perm(x2, x3, sel), a[2], a[3]);
                if constexpr (KVT == kKvInt8) {
                    a[0] = hmul2_u32(a[0], s01);
                    a[1] = hmul2_u32(a[1], s01);
                    a[2] = hmul2_u32(a[2], s23);
                    a[3] = hmul2_u32(a[3], s23);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_f16_16816(o[nt][2 * w + hw], a, pb[nt]);
            }
        }
    }
}

// FP16 cache, S^T = K Q^T for one block.  A key row is two 128-byte halves
// (d 0-63 at the tile's start, d 64-127 at + BS * 128), each 128-byte
// swizzled.  Lane (g, t) reads d = 32t .. 32t+31 of keys g and g+8: chunks
// 4(t&1) .. 4(t&1)+3 of half t>>1; the A fragment of k-step ks is word
// 2(ks&1) (d 32t+4ks, +1) and word 2(ks&1)+1 (d +2, +3) of chunk ks>>1, the
// same d order as the 8-bit path, so Q's fragments serve both.
template <int NT, int MT, int BS>
__device__ __forceinline__ void qk_block_f16(const uint8_t *kt, int g, int t,
                                             const uint32_t (&qf)[NT][8][2], float kfac,
                                             float (&sc)[MT][NT][4])
{
    const uint8_t *half = kt + (t >> 1) * BS * 128;
    const int c0 = 4 * (t & 1);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int r0 = mt * 16 + g;   // rows r0, r0 + 8 share (row & 7) == g
        uint4 ka[4], kb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ka[i] = lds128(half + r0 * 128 + (((c0 + i) ^ g) << 4));
            kb[i] = lds128(half + (r0 + 8) * 128 + (((c0 + i) ^ g) << 4));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                sc[mt][nt][c] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint4 &wa = ka[ks >> 1], &wb = kb[ks >> 1];
            uint32_t a[4];
            a[0] = (ks & 1) ? wa.z : wa.x;
            a[2] = (ks & 1) ? wa.w : wa.y;
            a[1] = (ks & 1) ? wb.z : wb.x;
            a[3] = (ks & 1) ? wb.w : wb.y;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_f16_16816(sc[mt][nt], a, qf[nt][ks]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                sc[mt][nt][c] *= kfac;
    }
}

// FP16 cache, O^T += V^T P^T for one block.  Lane (g, t) reads d = 16g ..
// 16g+15 (chunks 2(g&3), 2(g&3)+1 of half g>>2) of keys 2t, 2t+1, 2t+8, 2t+9;
// word w of that range is d-tile w: row g <-> d = 16g+2w, row g+8 <-> +1, the
// same output order as the 8-bit path.
template <int NT, int MT, int BS>
__device__ __forceinline__ void pv_block_f16(const uint8_t *vt, int g, int t, int key0, int ctx,
                                             const float (&pr)[MT][NT][4],
                                             float (&o)[NT][8][4])
{
    const uint8_t *half = vt + (g >> 2) * BS * 128;
    const int c0 = 2 * (g & 3);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            pb[nt][0] = movmatrix_trans(pack_half2(pr[mt][nt][0], pr[mt][nt][1]));
            pb[nt][1] = movmatrix_trans(pack_half2(pr[mt][nt][2], pr[mt][nt][3]));
        }
        const int r0 = mt * 16 + 2 * t;   // key rows r0, r0+1, r0+8, r0+9
        const int rr[4] = {r0, r0 + 1, r0 + 8, r0 + 9};
        uint4 v[4][2];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                v[k][j] = lds128(half + rr[k] * 128 + (((c0 + j) ^ (rr[k] & 7)) << 4));
        if (key0 + BS > ctx) {
            // Slots past the context were never written: their values may be
            // NaN patterns, and 0 * NaN would poison O.
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (key0 + rr[k] >= ctx)
                    v[k][0] = v[k][1] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t x0 = word_of(v[0][w >> 2], w & 3), x1 = word_of(v[1][w >> 2], w & 3);
            const uint32_t x2 = word_of(v[2][w >> 2], w & 3), x3 = word_of(v[3][w >> 2], w & 3);
            uint32_t a[4];
            a[0] = __byte_perm(x0, x1, 0x5410);   // d = 16g+2w of keys r0, r0+1
            a[1] = __byte_perm(x0, x1, 0x7632);   // d + 1
            a[2] = __byte_perm(x2, x3, 0x5410);
            a[3] = __byte_perm(x2, x3, 0x7632);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_f16_16816(o[nt][w], a, pb[nt]);
        }
    }
}

// The step's new tokens (each sequence's last q_len positions) that fall in
// positions [lo_pos, hi_pos): their K and V rows of KV head h quantised and
// stored in the cache exactly as the KV write kernel does, 16 threads (a
// half-warp) per token and 8 tokens per pass.
template <int KVT, int BS>
__device__ __forceinline__ void append_tokens(const DecodeParams &p, int b, int h, int ctx,
                                              int lo_pos, int hi_pos, const int32_t *bt)
{
    const int grp = threadIdx.x >> 4, sub = threadIdx.x & 15;
    uint8_t *kc = const_cast<uint8_t *>(p.k_cache);
    uint8_t *vc = const_cast<uint8_t *>(p.v_cache);
    uint16_t *kst = const_cast<uint16_t *>(p.k_scale_tok);
    uint16_t *vst = const_cast<uint16_t *>(p.v_scale_tok);
    float ks = 0.0f, vs = 0.0f;
    if constexpr (kv_has_head_scale(KVT)) {
        ks = __ldg(p.k_scale + h * p.scale_stride);
        vs = __ldg(p.v_scale + h * p.scale_stride);
    }
    for (int t0 = 0; t0 < p.q_len; t0 += kThreads / 16) {   // the same passes on every thread
        const int t = t0 + grp;
        const int pos = ctx - p.q_len + t;
        bool mine = t < p.q_len && pos >= 0 && pos >= lo_pos && pos < hi_pos &&
                    pos / BS < p.max_blocks_per_seq;
        int phys = mine ? __ldg(bt + pos / BS) : 0;
#ifdef PKVQ_BOUNDS_CHECK
        if (mine && (phys < 0 || phys >= p.num_blocks)) {
            if (sub == 0)
                atomicOr(p.status, kStatusBadBlock);
            mine = false;
            phys = 0;
        }
#endif
        const size_t drow = ((size_t)phys * p.num_kv_heads + h) * BS + (mine ? pos % BS : 0);
        uint4 kx = make_uint4(0u, 0u, 0u, 0u), vx = kx;
        if (mine) {
            const size_t src =
                (((size_t)b * p.q_len + t) * p.num_kv_heads + h) * kHeadDim + sub * 8;
            kx = __ldg(reinterpret_cast<const uint4 *>(p.k_new + src));
            vx = __ldg(reinterpret_cast<const uint4 *>(p.v_new + src));
        }
        quant_store_piece<KVT>(kc, kst, ks, drow, sub, kx, mine);
        quant_store_piece<KVT>(vc, vst, vs, drow, sub, vx, mine);
    }
}

// Merge of the split partial states of one output row by one warp:
// M = max_i m_i, L = sum_i l_i 2^(m_i - M), O = sum_i O_i 2^(m_i - M) / L.
// The splits are taken kMergeChunk at a time: every lane issues the loads of
// a whole chunk (the (m, l) pairs, the same for all lanes, and its float4 of
// each O row) before using any, so a chunk costs one memory round trip; the
// chunks are combined online.  `preloaded`: the caller already loaded the
// first chunk for slots first .. (ml, v).
constexpr int kMergeChunk = 16;

struct MergeRow {
    size_t row0, stride;   // workspace row of the first slot, rows between slots
    float2 ml[kMergeChunk];
    float4 v[kMergeChunk];

    __device__ __forceinline__ void load(const DecodeParams &p, int first, int nsplit, int s0,
                                         int lane)
    {
#pragma unroll
        for (int k = 0; k < kMergeChunk; ++k) {
            ml[k] = make_float2(-INFINITY, 0.0f);
            v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s0 + k < nsplit && first + s0 + k < p.num_splits) {
                const size_t wrow = row0 + (size_t)(first + s0 + k) * stride;
                ml[k] = *reinterpret_cast<const float2 *>(p.ws_ml + wrow * 2);
                v[k] = reinterpret_cast<const float4 *>(p.ws_o + wrow * kHeadDim)[lane];
            }
        }
    }

    // Combines the nsplit partials (the first chunk already loaded) and
    // writes output row rr of sequence b, KV head h.
    __device__ __forceinline__ void finish(const DecodeParams &p, int first, int nsplit, int b,
                                           int h, int rr, int lane)
    {
        float M = -INFINITY, L = 0.0f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < nsplit; s0 += kMergeChunk) {
            if (s0 > 0)
                load(p, first, nsplit, s0, lane);
            float cm = M;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k)
                cm = fmaxf(cm, ml[k].x);
            const float mu = cm == -INFINITY ? 0.0f : cm;
            const float corr = fast_exp2(M - mu);
            L *= corr;
            O.x *= corr, O.y *= corr, O.z *= corr, O.w *= corr;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) {
                const float e = fast_exp2(ml[k].x - mu);
                L += ml[k].y * e;
                O.x += v[k].x * e, O.y += v[k].y * e, O.z += v[k].z * e, O.w += v[k].w * e;
            }
            M = cm;
        }
        const float vfac = p.v_scale ? __ldg(p.v_scale + h * p.scale_stride) : 1.0f;
        const float f = L > 0.0f ? vfac / L : 0.0f;
        const int tq = rr / p.group, gq = rr % p.group;
        const size_t orow = ((size_t)b * p.q_len + tq) * p.num_q_heads + h * p.group + gq;
        const __half2 lo = __floats2half2_rn(O.x * f, O.y * f);
        const __half2 hi = __floats2half2_rn(O.z * f, O.w * f);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t *>(&lo);
        pk.y = *reinterpret_cast<const uint32_t *>(&hi);
        reinterpret_cast<uint2 *>(p.out + orow * kHeadDim)[lane] = pk;
        if (lane == 0 && p.lse)
            p.lse[orow] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
};

constexpr int kMinBlocksPerWarp = 3;   // shortest split: 3 cache blocks per warp

template <int KVT, int NT, int BS>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const DecodeParams p)
{
    using C = DecodeCfg<KVT, BS>;
    constexpr int S = C::kStages;
    constexpr int U = C::kUnroll;
    constexpr int RC = 8 * NT;
    constexpr int MT = C::kMT;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tiles = smem;
    uint16_t *scales = reinterpret_cast<uint16_t *>(tiles + kWarps * S * C::kStageBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(scales + kWarps * S * C::kScaleHalves);

    const int slot = blockIdx.x;
    const int h = blockIdx.y % p.num_kv_heads;
    const int rg = blockIdx.y / p.num_kv_heads;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    // Prologue that reads no input: it may overlap the previous kernel in the
    // stream (this kernel is launched with programmatic dependent launch).
    uint64_t *my_bars = bars + warp * S;
    uint8_t *my_tiles = tiles + warp * S * C::kStageBytes;
    uint16_t *my_scales = scales + warp * S * C::kScaleHalves;
    if (lane == 0) {
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
#pragma unroll
        for (int s = 0; s < S; ++s)
            mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // Inputs may come from the previous kernel: wait for it to complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Let the merge kernel get scheduled early; it still waits for this grid
    // to finish before reading the workspace.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // (a CTA-wide decision: the kernel ends with CTA barriers)
    if (__syncthreads_or(device_wait_failed(p.status)))
        return;
    // The block ids of this warp's first 64 iterations and the query rows are
    // loaded for a guess of this slot's (sequence, split): the assignment all
    // sequences at max_context_len would give.  They are loaded while the
    // real assignment is computed from the context lengths, and reloaded
    // only when the guess was wrong (different lengths), so that with equal
    // lengths the first copies wait for one memory round trip, not two.
    int b = min(slot / p.uniform_splits, p.batch - 1);
    int blk_begin = (slot - b * p.uniform_splits) * p.uniform_bpc;
    const int h0 = h * p.group;
    int win0, win1;
    int win_base = 0;
    auto lblk = [&](int it) { return blk_begin + warp + kWarps * it; };
    auto load_window = [&]() {   // every index stays inside the table row
        const int32_t *bt = p.block_table + (size_t)b * p.max_blocks_per_seq;
        win0 = lblk(lane) < p.max_blocks_per_seq ? __ldg(bt + lblk(lane)) : 0;
        win1 = lblk(32 + lane) < p.max_blocks_per_seq ? __ldg(bt + lblk(32 + lane)) : 0;
    };
    // query fragments (B operand of S^T = K Q^T), loop invariant
    uint32_t qf[NT][8][2];
    auto load_q = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r = rg * RC + nt * 8 + g;
            uint32_t u[16];
            if (r < p.rows) {
                const int tq = r / p.group, gq = r % p.group;
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    p.q + (((size_t)b * p.q_len + tq) * p.num_q_heads + h0 + gq) * kHeadDim +
                    32 * t);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint4 w = __ldg(src + i);
                    u[4 * i] = w.x, u[4 * i + 1] = w.y, u[4 * i + 2] = w.z, u[4 * i + 3] = w.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    u[i] = 0u;
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[nt][ks][0] = u[2 * ks];       // d = 32t + 4ks + {0,1}
                qf[nt][ks][1] = u[2 * ks + 1];   // d = 32t + 4ks + {2,3}
            }
        }
    };
    load_window();
    load_q();
    const SplitInfo si = find_split<BS>(p, slot, -1);
    if (si.b < 0)
        return;   // a slot past the last split: no work
    const int real_begin = si.blk0 + si.split * si.bpc;
    if (si.b != b || real_begin != blk_begin) {
        const bool new_seq = si.b != b;
        b = si.b;
        blk_begin = real_begin;
        load_window();
        if (new_seq)
            load_q();
    }
    const int ctx = si.ctx;
    const int nblk_seq = (ctx + BS - 1) / BS;
    const int nblk = max(0, min(nblk_seq, blk_begin + si.bpc) - blk_begin);
    const int n_it = warp < nblk ? (nblk - warp + kWarps - 1) / kWarps : 0;
    const int32_t *bt = p.block_table + (size_t)b * p.max_blocks_per_seq;
    // Appending call: the step's new tokens in this CTA's blocks are
    // quantised and stored first (no other CTA of this KV head reads those
    // slots), then made visible to the tensor copies below.
    if (p.k_new) {
        append_tokens<KVT, BS>(p, b, h, ctx, blk_begin * BS, (blk_begin + nblk) * BS, bt);
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncthreads();
    }
    // each thread's two rows per n8 tile: last visible key (pos) and first
    // (lo); padding rows see the whole split
    int pos[NT][2], lo[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int rr = rg * RC + nt * 8 + 2 * t + i;
            pos[nt][i] = rr < p.rows ? min(ctx - 1, query_position(p, b, ctx, rr / p.group))
                                     : ctx - 1;
            lo[nt][i] = p.window > 0 && rr < p.rows ? pos[nt][i] - p.window + 1 : 0;
        }
    // a block needs masking when it reaches past the lowest position or
    // starts below the highest window start of the CTA's rows
    int min_pos = ctx - 1, max_lo = 0;
    for (int tq = 0; tq < p.q_len; ++tq) {
        const int ps = min(ctx - 1, query_position(p, b, ctx, tq));
        min_pos = min(min_pos, ps);
        if (p.window > 0)
            max_lo = max(max_lo, ps - p.window + 1);
    }

    float kfac = p.scale_log2;
    if constexpr (kv_has_head_scale(KVT))
        kfac *= __ldg(p.k_scale + h * p.scale_stride);

    float o[NT][8][4];
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int dt = 0; dt < 8; ++dt)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                o[nt][dt][c] = 0.0f;
#pragma unroll
        for (int i = 0; i < 2; ++i)
            m[nt][i] = -INFINITY, l[nt][i] = 0.0f;
    }

    // ---- block ids: a sliding window of 64 iterations held in two registers ----

    constexpr uint32_t kTx = C::kStageBytes + (KVT == kKvInt8 ? C::kScaleHalves * 2 : 0);
    auto issue = [&](int j) {   // warp-uniform call
        const int a = __shfl_sync(0xffffffffu, win0, j & 31);
        const int c = __shfl_sync(0xffffffffu, win1, j & 31);
        int phys = (j - win_base) < 32 ? a : c;
        if (lane == 0) {
#ifdef PKVQ_BOUNDS_CHECK
            if (phys < 0 || phys >= p.num_blocks) {
                atomicOr(p.status, kStatusBadBlock);
                phys = 0;
            }
#endif
            const int stage = j % S;
            uint64_t *bar = &my_bars[stage];
            mbar_arrive_expect_tx(bar, kTx);
            const int y = (phys * p.num_kv_heads + h) * BS;
            uint8_t *dst = my_tiles + stage * C::kStageBytes;
            tma_tile_2d_g2s(dst, &kmap, 0, y, bar);
            tma_tile_2d_g2s(dst + C::kTileBytes, &vmap, 0, y, bar);
            if constexpr (KVT == kKvFp16) {   // second 128-byte half of each row
                tma_tile_2d_g2s(dst + BS * 128, &kmap, 128, y, bar);
                tma_tile_2d_g2s(dst + C::kTileBytes + BS * 128, &vmap, 128, y, bar);
            }
            if constexpr (KVT == kKvInt8) {
                uint16_t *sd = my_scales + stage * C::kScaleHalves;
                tma_bulk_g2s(sd, p.k_scale_tok + (size_t)y, BS * 2, bar);
                tma_bulk_g2s(sd + BS, p.v_scale_tok + (size_t)y, BS * 2, bar);
            }
        }
    };

    int issued = 0;
    for (; issued < S && issued < n_it; ++issued)
        issue(issued);

    int it = 0;
    bool ok = true;
    for (; it < n_it; it += U) {
        // ---- wait for this iteration's U blocks ----
        bool have[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            have[u] = it + u < n_it;
            if (have[u] && !mbar_wait(&my_bars[(it + u) % S], ((it + u) / S) & 1, p.status))
                ok = false;
        }
        if (!ok)
            break;

        // ---- S^T = K Q^T, masked ----
        float sc[U][MT][NT][4];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int stage = (it + u) % S;
            const uint8_t *kt = my_tiles + stage * C::kStageBytes;
            const uint16_t *st = my_scales + stage * C::kScaleHalves;
            if (have[u]) {
                if constexpr (KVT == kKvFp16)
                    qk_block_f16<NT, MT, BS>(kt, g, t, qf, kfac, sc[u]);
                else
                    qk_block<KVT, NT, MT>(kt, st, g, t, qf, kfac, sc[u]);
                const int key0 = lblk(it + u) * BS;
                // a key may lie past a row's position or below its window
                if (key0 + BS - 1 > min_pos || key0 < max_lo) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int key = key0 + mt * 16 + g + (c >> 1) * 8;
                                if (key > pos[nt][c & 1] || key < lo[nt][c & 1])
                                    sc[u][mt][nt][c] = -INFINITY;
                            }
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            sc[u][mt][nt][c] = -INFINITY;
            }
        }

        // ---- online softmax (base 2) over the U blocks ----
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float mx = -INFINITY;
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        mx = fmaxf(mx, fmaxf(sc[u][mt][nt][i], sc[u][mt][nt][2 + i]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m[nt][i], mx);
                const float m_use = m_new == -INFINITY ? 0.0f : m_new;
                const float corr = fast_exp2(m[nt][i] - m_use);
                m[nt][i] = m_new;
                if (__any_sync(0xffffffffu, corr != 1.0f)) {
                    l[nt][i] *= corr;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        o[nt][dt][i] *= corr;
                        o[nt][dt][2 + i] *= corr;
                    }
                }
                float ls = 0.0f;
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const float p0 = fast_exp2(sc[u][mt][nt][i] - m_use);
                        const float p1 = fast_exp2(sc[u][mt][nt][2 + i] - m_use);
                        sc[u][mt][nt][i] = p0;
                        sc[u][mt][nt][2 + i] = p1;
                        ls += p0 + p1;
                    }
                l[nt][i] += ls;
            }
        }

        // ---- O^T += V^T P^T ----
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!have[u])
                continue;
            const int stage = (it + u) % S;
            const uint8_t *vt = my_tiles + stage * C::kStageBytes + C::kTileBytes;
            const uint16_t *st = my_scales + stage * C::kScaleHalves;
            if constexpr (KVT == kKvFp16)
                pv_block_f16<NT, MT, BS>(vt, g, t, lblk(it + u) * BS, ctx, sc[u], o);
            else
                pv_block<KVT, NT, MT, BS>(vt, st, g, t, lblk(it + u) * BS, ctx, sc[u], o);
        }

        __syncwarp();
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (issued < n_it) {
                issue(issued);
                ++issued;
            }
        if (it + U >= win_base + 32) {
            win_base += 32;
            win0 = win1;
            win1 = lblk(win_base + 32 + lane) < p.max_blocks_per_seq
                       ? __ldg(bt + lblk(win_base + 32 + lane)) : 0;
        }
    }
    if (!ok) {
        // A wait gave up: let the copies still in flight land (bounded) before
        // this CTA's shared memory is reused or released.
        for (int j = it; j < issued; ++j)
            mbar_wait(&my_bars[j % S], (j / S) & 1, nullptr);
    }

    // row sums: reduce the per-thread partial sums over the 8 key lanes
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float s = l[nt][i];
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            s += __shfl_xor_sync(0xffffffffu, s, 8);
            s += __shfl_xor_sync(0xffffffffu, s, 16);
            l[nt][i] = s;
        }

    // ---- merge the 4 warps' states through shared memory (tiles are idle now) ----
    __syncthreads();
    float *so = reinterpret_cast<float *>(smem);      // [W][RC][128]
    float *sm = so + kWarps * RC * kHeadDim;          // [W][RC]
    float *sl = sm + kWarps * RC;                     // [W][RC]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = nt * 8 + 2 * t + i;
            float *dst = so + (warp * RC + r) * kHeadDim + 16 * g;
#pragma unroll
            for (int dt = 0; dt < 8; ++dt) {
                dst[2 * dt] = o[nt][dt][i];
                dst[2 * dt + 1] = o[nt][dt][2 + i];
            }
            if (g == 0) {
                sm[warp * RC + r] = m[nt][i];
                sl[warp * RC + r] = l[nt][i];
            }
        }
    __syncthreads();

    const int d = threadIdx.x;   // 128 threads <-> 128 dims
    float vfac = 1.0f;
    if constexpr (kv_has_head_scale(KVT))
        vfac = __ldg(p.v_scale + h * p.scale_stride);
    // Rows are independent: the loop is unrolled so that their shared-memory
    // reads and global stores overlap.
#pragma unroll 4
    for (int r = 0; r < RC; ++r) {
        const int rr = rg * RC + r;
        if (rr >= p.rows)
            continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            M = fmaxf(M, sm[w * RC + r]);
        const float Mu = M == -INFINITY ? 0.0f : M;
        float L = 0.0f, O = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float e = fast_exp2(sm[w * RC + r] - Mu);
            L += sl[w * RC + r] * e;
            O += so[(w * RC + r) * kHeadDim + d] * e;
        }
        if (si.nsplit == 1) {
            const int tq = rr / p.group, gq = rr % p.group;
            const size_t orow = ((size_t)b * p.q_len + tq) * p.num_q_heads + h0 + gq;
            p.out[orow * kHeadDim + d] = __float2half_rn(L > 0.0f ? O / L * vfac : 0.0f);
            if (d == 0 && p.lse)
                p.lse[orow] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
        } else {
            const size_t wrow = ((size_t)blockIdx.y * p.num_splits + slot) * RC + r;
            p.ws_o[wrow * kHeadDim + d] = O;
            if (d == 0)
                *reinterpret_cast<float2 *>(p.ws_ml + wrow * 2) = make_float2(M, L);
        }
    }
}

// Merge of the split partial states by a separate kernel, one warp per
// output row; programmatic dependent launch lets it start while the split
// kernel's last CTAs finish.  (A variant in which the last CTA of each
// sequence merged its splits itself, found through arrival counters, took
// the same time on the batch-8 x 32K workload and needed a zeroed
// workspace.)
template <int BS>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 4 + warp;
    const long long total = (long long)p.batch * p.num_kv_heads * p.rows;
    if (gw >= total)
        return;
    const int rr = (int)(gw % p.rows);
    const int h = (int)((gw / p.rows) % p.num_kv_heads);
    const int b = (int)(gw / ((long long)p.rows * p.num_kv_heads));
    // slots first .. first + nsplit - 1 of unit (row group, KV head) y
    const int y = (rr / p.rows_per_cta) * p.num_kv_heads + h;
    MergeRow mr;
    mr.row0 = (size_t)y * p.num_splits * p.rows_per_cta + rr % p.rows_per_cta;
    mr.stride = p.rows_per_cta;
    // The slots of sequence b come from the context lengths, inputs the split
    // kernel does not write: they are found while the split kernel's last
    // CTAs still run, and only the partials wait for its completion.
    const SplitInfo si = find_split<BS>(p, -1, b);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (si.nsplit <= 1)
        return;   // a single split wrote the final row itself
    mr.load(p, si.first, si.nsplit, 0, lane);
    mr.finish(p, si.first, si.nsplit, b, h, rr, lane);
}

template <int KVT, int NT, int BS>
cudaError_t launch_split(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                         cudaStream_t stream)
{
    constexpr size_t smem = decode_smem_bytes<KVT, BS>();
    auto kern = decode_split_kernel<KVT, NT, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.num_splits, p.num_kv_heads * p.row_groups, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, kmap, vmap, p);
}

template <int KVT, int NT>
cudaError_t launch_bs(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                      cudaStream_t stream)
{
    switch (p.block_size) {
    case 16: return launch_split<KVT, NT, 16>(p, kmap, vmap, stream);
    case 32: return launch_split<KVT, NT, 32>(p, kmap, vmap, stream);
    case 64: return launch_split<KVT, NT, 64>(p, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <int KVT, int NT, int BS>
int occupancy_of()
{
    auto kern = decode_split_kernel<KVT, NT, BS>;
    constexpr size_t smem = decode_smem_bytes<KVT, BS>();
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess)
        return 0;
    return n;
}

template <int KVT, int NT>
int occupancy_bs(int block_size)
{
    switch (block_size) {
    case 16: return occupancy_of<KVT, NT, 16>();
    case 32: return occupancy_of<KVT, NT, 32>();
    case 64: return occupancy_of<KVT, NT, 64>();
    default: return 0;
    }
}

// Resident split CTAs per SM for one kernel instance (registers and shared
// memory decide it), cached per device; 2 where it cannot be queried.
template <int KVT>
int occupancy_nt(int nt, int block_size)
{
    return nt == 1 ? occupancy_bs<KVT, 1>(block_size) : occupancy_bs<KVT, 2>(block_size);
}

int split_occupancy(int kv_dtype, int nt, int block_size)
{
    constexpr int kMaxDev = 64;
    static int cache[kMaxDev][4][2][3] = {};
    int dev = 0;
    const int bi = block_size == 16 ? 0 : (block_size == 32 ? 1 : 2);
    if (kv_dtype < 0 || kv_dtype > 3 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
        dev >= kMaxDev)
        return 2;
    int &c = cache[dev][kv_dtype][nt - 1][bi];
    if (!c) {
        int n = 0;
        switch (kv_dtype) {
        case kKvFp8: n = occupancy_nt<kKvFp8>(nt, block_size); break;
        case kKvInt8: n = occupancy_nt<kKvInt8>(nt, block_size); break;
        case kKvE5m2: n = occupancy_nt<kKvE5m2>(nt, block_size); break;
        default: n = occupancy_nt<kKvFp16>(nt, block_size); break;
        }
        c = n > 0 ? n : 2;
    }
    return c;
}

}  // namespace

bool decode_plan(int kv_dtype, int batch, int q_len, int num_q_heads, int num_kv_heads,
                 int block_size, int max_context_len, DecodePlan *plan)
{
    if (batch <= 0 || q_len <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads)
        return false;
    const int group = num_q_heads / num_kv_heads;
    const int rows = q_len * group;
    // More than 16 rows per KV head (up to 128): the tensor-core kernel, one
    // CTA for all rows, so every code is fetched and converted once; the
    // mma.sync kernel would split the rows into groups that each convert it.
    plan->tc = rows > 16 && rows <= 128;
    plan->nt = plan->tc ? 0 : (rows <= 8 ? 1 : 2);
    plan->rows_per_cta = plan->tc ? rows : 8 * plan->nt;
    plan->row_groups = (rows + plan->rows_per_cta - 1) / plan->rows_per_cta;
    const int max_blocks = (max_context_len + block_size - 1) / block_size;
    const int units = num_kv_heads * plan->row_groups;   // grid y: (row group, KV head)
    // splits: tensor-core kernel in whole 64-key tiles, at least 256 keys;
    // mma.sync kernel at least kMinBlocksPerWarp blocks per warp
    const int min_blocks = plan->tc ? 256 / block_size : kWarps * kMinBlocksPerWarp;
    plan->split_min_blocks = min_blocks;
    plan->split_gran = plan->tc ? 64 / block_size : 1;
    // C CTA slots per unit, at most `ctas_per_sm` CTAs on every SM (3, or
    // what fits), all resident in one wave, each slot given about the same
    // number of blocks on the device.  Rounding the count up instead would
    // put one more CTA on some SMs, and those SMs' CTAs would all finish last
    // (a memory-bound CTA gets a share of its SM's bandwidth); more resident
    // CTAs keep more copies in flight.  At least one slot per sequence, and
    // no more slots than splits of kMinBlocksPerWarp blocks per warp.
    // PKVQ_DECODE_CTAS_PER_SM (1..16) replaces the target as given, even
    // beyond what fits in one wave.
    // (the tensor-core kernel takes most of an SM's shared memory: one CTA)
    int ctas_per_sm = plan->tc ? 1 : min(3, split_occupancy(kv_dtype, plan->nt, block_size));
    if (const char *env = getenv("PKVQ_DECODE_CTAS_PER_SM")) {
        const int v = atoi(env);
        if (v >= 1 && v <= 16)
            ctas_per_sm = v;
    }
    const long long target = (long long)ctas_per_sm * device_sm_count();
    long long C = max((long long)batch, target / units);
    const long long useful = (long long)batch * max(1, max_blocks / min_blocks);
    C = min(C, max((long long)batch, useful));
    if (C > (1LL << 30))
        return false;
    plan->num_splits = (int)C;
    // the split every slot gets when all sequences hold max_context_len tokens
    plan->uniform_bpc = split_blocks((long long)batch * max_blocks, (int)C, batch, max_blocks,
                                     plan->split_min_blocks, plan->split_gran);
    plan->uniform_splits = max(1, (max_blocks + plan->uniform_bpc - 1) / plan->uniform_bpc);
    const size_t partials = C > batch ? (size_t)units * C * plan->rows_per_cta *
                                            (kHeadDim + 2) * sizeof(float)
                                      : 0;
    plan->workspace_bytes = partials;
    return true;
}

cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, int kv_dtype,
                          const CUtensorMap &kmap, const CUtensorMap &vmap, cudaStream_t stream)
{
    cudaError_t e;
    const bool one = plan.nt == 1;
    if (plan.tc)
        e = launch_decode_tc(p, kv_dtype, kmap, vmap, stream);
    else if (kv_dtype == kKvFp8)
        e = one ? launch_bs<kKvFp8, 1>(p, kmap, vmap, stream)
                : launch_bs<kKvFp8, 2>(p, kmap, vmap, stream);
    else if (kv_dtype == kKvInt8)
        e = one ? launch_bs<kKvInt8, 1>(p, kmap, vmap, stream)
                : launch_bs<kKvInt8, 2>(p, kmap, vmap, stream);
    else if (kv_dtype == kKvE5m2)
        e = one ? launch_bs<kKvE5m2, 1>(p, kmap, vmap, stream)
                : launch_bs<kKvE5m2, 2>(p, kmap, vmap, stream);
    else
        e = one ? launch_bs<kKvFp16, 1>(p, kmap, vmap, stream)
                : launch_bs<kKvFp16, 2>(p, kmap, vmap, stream);
    if (e != cudaSuccess || p.num_splits <= p.batch)
        return e;   // one slot per sequence: every CTA wrote final rows
    const long long rows_total = (long long)p.batch * p.num_kv_heads * p.rows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows_total + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (p.block_size) {
    case 16: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<16>, p);
    case 32: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<32>, p);
    case 64: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<64>, p);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
