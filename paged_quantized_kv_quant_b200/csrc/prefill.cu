// Causal (chunked) prefill over the paged 8-bit cache: warp-level tensor-core
// version (mma.sync m16n8k16).
//
// Source: "1Cat-LLM" README, "Layer 2" (causal online softmax with FP32
// accumulation, GQA multi-head packing, prefix / causal-tail separation, wide
// QK/PV tiles) and "Layer 1" (pages read once, wide); "ReVolta" PyPI page
// (chunked prefill with an 8,192-token budget).
//
// A CTA owns 128 query rows = (128 / G) query tokens x the G query heads of
// one KV head, so every dequantised key/value tile is shared by all G heads.
// Key tiles of 64 keys arrive as 2-D TMA copies (one per cache block, 128-byte
// swizzle) into a 2-stage ring; all 256 threads convert a tile once into fp16
// K/V tiles in shared memory (XOR-swizzled for conflict-free ldmatrix), then
// each warp runs S = Q K^T, the online softmax and O += P V on its 16 rows.
// Tiles wholly below every row's causal limit skip the mask (the fully
// visible prefix); only tiles that cross the diagonal are masked.
#include "common.cuh"
#include "internal.h"

#include <math.h>

namespace pkvq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kKT = 64;           // keys per tile
constexpr float kLn2 = 0.693147180559945309f;

struct PrefillSmem {
    static constexpr int kCodeTile = kKT * 128;               // bytes of K (or V) codes
    static constexpr int kCodeStage = 2 * kCodeTile;          // K + V
    static constexpr int kHalfTile = kKT * 128 * 2;           // fp16 K (or V) tile
    static constexpr int kOffCodes = 0;                       // 2 stages
    static constexpr int kOffKh = 2 * kCodeStage;             // 32 KB
    static constexpr int kOffVh = kOffKh + kHalfTile;
    static constexpr int kOffScales = kOffVh + kHalfTile;     // 2 stages x (K, V) x 64 halves
    static constexpr int kOffBars = kOffScales + 2 * 2 * kKT * 2;
    static constexpr int kBytes = kOffBars + 2 * 8;
};

__device__ __forceinline__ uint32_t cvt_pair(int kvt, uint32_t pair)
{
    return kvt == kKvFp8 ? e4m3x2_to_half2(pair) : s8x2_to_half2(pair);
}

template <int KVT, int BS>
__global__ void __launch_bounds__(kThreads)
prefill_mma_kernel(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const PrefillParams p)
{
    using L = PrefillSmem;
    constexpr int kBlocksPerTile = kKT / BS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *codes = smem + L::kOffCodes;
    uint8_t *kh = smem + L::kOffKh;
    uint8_t *vh = smem + L::kOffVh;
    uint16_t *scl = reinterpret_cast<uint16_t *>(smem + L::kOffScales);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBars);

    const int tile = p.q_tiles - 1 - blockIdx.x;   // longest causal work first
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int q_start = p.cu_seqlens_q[b];
    const int q_len = p.cu_seqlens_q[b + 1] - q_start;
    const int q0 = tile * p.tokens_per_tile;
    if (q0 >= q_len || device_wait_failed(p.status))
        return;
    const int ctx = p.context_lens[b];
    const int G = p.group;
    const int tq_end = min(q_len, q0 + p.tokens_per_tile);
    const int pos_lo = ctx - q_len + q0;             // position of the tile's first token
    const int pos_hi = ctx - q_len + tq_end - 1;     // ... and of its last
    const int nkeys = max(0, min(ctx, pos_hi + 1));
    const int ntiles = (nkeys + kKT - 1) / kKT;
    const int nblk_seq = (ctx + BS - 1) / BS;
    const int32_t *bt = p.block_table + (size_t)b * p.max_blocks_per_seq;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;

    if (tid == 0) {
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int kt) {   // called by thread 0 only
        const int stage = kt & 1;
        const int blk0 = kt * kBlocksPerTile;
        const int nb = min(kBlocksPerTile, nblk_seq - blk0);
        uint32_t tx = (uint32_t)nb * BS * 128 * 2;
        if constexpr (KVT == kKvInt8)
            tx += (uint32_t)nb * BS * 2 * 2;
        mbar_arrive_expect_tx(&bars[stage], tx);
        for (int i = 0; i < nb; ++i) {
            int phys = __ldg(bt + blk0 + i);
#ifdef PKVQ_BOUNDS_CHECK
            if (phys < 0 || phys >= p.num_blocks) {
                atomicOr(p.status, kStatusBadBlock);
                phys = 0;
            }
#endif
            const int y = (phys * p.num_kv_heads + h) * BS;
            uint8_t *dk = codes + stage * L::kCodeStage + i * BS * 128;
            tma_tile_2d_g2s(dk, &kmap, 0, y, &bars[stage]);
            tma_tile_2d_g2s(dk + L::kCodeTile, &vmap, 0, y, &bars[stage]);
            if constexpr (KVT == kKvInt8) {
                uint16_t *sd = scl + stage * 2 * kKT + i * BS;
                tma_bulk_g2s(sd, p.k_scale_tok + (size_t)y, BS * 2, &bars[stage]);
                tma_bulk_g2s(sd + kKT, p.v_scale_tok + (size_t)y, BS * 2, &bars[stage]);
            }
        }
    };
    if (tid == 0) {
        if (ntiles > 0)
            issue(0);
        if (ntiles > 1)
            issue(1);
    }

    // ---- Q fragments for this warp's 16 rows (A operand, row-major) ----
    const int ra = warp * 16 + g, rb = ra + 8;     // CTA rows held by this thread
    const int tqa = q0 + ra / G, tqb = q0 + rb / G;
    const bool va = ra < p.tokens_per_tile * G && tqa < q_len;
    const bool vb = rb < p.tokens_per_tile * G && tqb < q_len;
    const int posa = ctx - q_len + tqa, posb = ctx - q_len + tqb;
    const __half *qa = p.q + ((size_t)(q_start + tqa) * p.num_q_heads + h * G + ra % G) * kHeadDim;
    const __half *qb = p.q + ((size_t)(q_start + tqb) * p.num_q_heads + h * G + rb % G) * kHeadDim;
    uint32_t qf[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const int d0 = ks * 16 + 2 * t;
        qf[ks][0] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + d0)) : 0u;
        qf[ks][1] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + d0)) : 0u;
        qf[ks][2] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + d0 + 8)) : 0u;
        qf[ks][3] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + d0 + 8)) : 0u;
    }

    float kfac = p.scale_log2;
    if constexpr (KVT == kKvFp8)
        kfac *= __ldg(p.k_scale + h);

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
        o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};

    bool ok = true;
    for (int kt = 0; kt < ntiles; ++kt) {
        const int stage = kt & 1;
        ok = mbar_wait(&bars[stage], (kt >> 1) & 1, p.status);
        if (__syncthreads_or(!ok)) {
            // let copies still in flight land (bounded) before leaving
            if (tid == 0)
                for (int j = kt; j < min(ntiles, kt + 2); ++j)
                    mbar_wait(&bars[j & 1], (j >> 1) & 1, nullptr);
            __syncthreads();
            return;
        }
        const int key0 = kt * kKT;
        // ---- convert codes -> fp16 tiles (each thread: 4 K and 4 V chunks of 8) ----
        {
            const uint8_t *ck = codes + stage * L::kCodeStage;
            const uint16_t *sk = scl + stage * 2 * kKT;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int idx = tid + j * kThreads;      // 0 .. 2047
                const int isv = idx >> 10;               // 0: K, 1: V
                const int r = (idx >> 4) & 63;           // key row in tile
                const int c = idx & 15;                  // 16-byte fp16 chunk (8 dims)
                const int cc = c >> 1;                   // 16-byte code chunk
                const uint8_t *src = ck + isv * L::kCodeTile + r * 128 + ((cc ^ (r & 7)) << 4) + (c & 1) * 8;
                uint2 w = *reinterpret_cast<const uint2 *>(src);
                uint4 hv;
                hv.x = cvt_pair(KVT, w.x & 0xffffu);
                hv.y = cvt_pair(KVT, w.x >> 16);
                hv.z = cvt_pair(KVT, w.y & 0xffffu);
                hv.w = cvt_pair(KVT, w.y >> 16);
                const bool live = key0 + r < ctx;
                if (KVT == kKvInt8 && isv) {
                    const uint16_t s = sk[kKT + r];
                    const uint32_t s2 = (uint32_t)s | ((uint32_t)s << 16);
                    __half2 s2h = *reinterpret_cast<const __half2 *>(&s2);
                    uint32_t *hp = reinterpret_cast<uint32_t *>(&hv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&hp[e]), s2h);
                        hp[e] = *reinterpret_cast<uint32_t *>(&x);
                    }
                }
                if (!live)
                    hv = make_uint4(0u, 0u, 0u, 0u);   // unwritten slots may hold NaN codes
                uint8_t *dst = (isv ? vh : kh) + r * 256 + ((c ^ (r & 7)) << 4);
                *reinterpret_cast<uint4 *>(dst) = hv;
            }
        }
        float ksc[8][2];   // INT8: per-key K scales of this thread's score columns
        if constexpr (KVT == kKvInt8) {
            const uint16_t *sk = scl + stage * 2 * kKT;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                ksc[n][0] = __half2float(__ushort_as_half(sk[n * 8 + 2 * t]));
                ksc[n][1] = __half2float(__ushort_as_half(sk[n * 8 + 2 * t + 1]));
            }
        }
        __syncthreads();
        if (tid == 0 && kt + 2 < ntiles)
            issue(kt + 2);   // the code stage is free once converted

        // ---- S = Q K^T (16 rows x 64 keys per warp) ----
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
            s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            // rows n*8 .. n*8+7 of the K tile; lanes 0-7 / 8-15 / 16-23 / 24-31
            // address the d-chunks 2k, 2k+1, 2k+2, 2k+3 for the k-step pair k.
            const int kr = n * 8 + (lane & 7);
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                const int c = kp * 4 + (lane >> 3);
                uint32_t r4[4];
                ldmatrix_x4(r4, smem_u32(kh + kr * 256 + ((c ^ (kr & 7)) << 4)));
                const uint32_t b0[2] = {r4[0], r4[1]};
                const uint32_t b1[2] = {r4[2], r4[3]};
                mma_f16_16816(s[n], qf[2 * kp], b0);
                mma_f16_16816(s[n], qf[2 * kp + 1], b1);
            }
        }
        // scale, mask the diagonal tiles, online softmax
        const bool need_mask = key0 + kKT - 1 > pos_lo;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f = kfac;
                if constexpr (KVT == kKvInt8)
                    f *= ksc[n][c & 1];
                float v = s[n][c] * f;
                if (need_mask) {
                    const int key = key0 + n * 8 + 2 * t + (c & 1);
                    if (key > ((c >> 1) ? posb : posa))
                        v = -INFINITY;
                }
                s[n][c] = v;
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int n = 0; n < 8; ++n)
                mx = fmaxf(mx, fmaxf(s[n][2 * i], s[n][2 * i + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m[i], mx);
            const float m_use = m_new == -INFINITY ? 0.0f : m_new;
            const float corr = fast_exp2(m[i] - m_use);
            m[i] = m_new;
            float ls = l[i] * corr;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                o[n][2 * i] *= corr;
                o[n][2 * i + 1] *= corr;
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const float p0 = fast_exp2(s[n][2 * i] - m_use);
                const float p1 = fast_exp2(s[n][2 * i + 1] - m_use);
                s[n][2 * i] = p0;
                s[n][2 * i + 1] = p1;
                ls += p0 + p1;
            }
            l[i] = ls;
        }
        // ---- O += P V ----
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t a[4] = {pack_half2(s[2 * kk][0], s[2 * kk][1]),
                                   pack_half2(s[2 * kk][2], s[2 * kk][3]),
                                   pack_half2(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                                   pack_half2(s[2 * kk + 1][2], s[2 * kk + 1][3])};
            // lanes 0-7: keys 16kk+0..7, lanes 8-15: keys 16kk+8..15 (d-tile n),
            // lanes 16-23 / 24-31: same keys, d-tile n+1
            const int vr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int n = 0; n < 16; n += 2) {
                const int c = n + (lane >> 4);
                uint32_t r4[4];
                ldmatrix_x4_trans(r4, smem_u32(vh + vr * 256 + ((c ^ (vr & 7)) << 4)));
                const uint32_t b0[2] = {r4[0], r4[1]};
                const uint32_t b1[2] = {r4[2], r4[3]};
                mma_f16_16816(o[n], a, b0);
                mma_f16_16816(o[n + 1], a, b1);
            }
        }
        __syncthreads();   // K/V fp16 tiles are rewritten by the next conversion
    }

    // ---- epilogue ----
    float vfac = 1.0f;
    if constexpr (KVT == kKvFp8)
        vfac = __ldg(p.v_scale + h);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool v = i ? vb : va;
        if (!v)
            continue;
        const int tq = i ? tqb : tqa;
        const int r = i ? rb : ra;
        const size_t orow = (size_t)(q_start + tq) * p.num_q_heads + h * G + r % G;
        const float f = l[i] > 0.0f ? vfac / l[i] : 0.0f;
        __half *dst = p.out + orow * kHeadDim;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            const float x0 = l[i] > 0.0f ? o[n][2 * i] / l[i] * vfac : 0.0f;
            const float x1 = l[i] > 0.0f ? o[n][2 * i + 1] / l[i] * vfac : 0.0f;
            *reinterpret_cast<__half2 *>(dst + n * 8 + 2 * t) = __floats2half2_rn(x0, x1);
        }
        (void)f;
        if (t == 0 && p.lse)
            p.lse[orow] = l[i] > 0.0f ? (m[i] + log2f(l[i])) * kLn2 : -INFINITY;
    }
}

template <int KVT, int BS>
cudaError_t launch_one(const PrefillParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                       cudaStream_t stream)
{
    constexpr size_t smem = PrefillSmem::kBytes + 1024;
    auto kern = prefill_mma_kernel<KVT, BS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.q_tiles, p.num_kv_heads, p.batch);
    kern<<<grid, kThreads, smem, stream>>>(kmap, vmap, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams &p, int kv_dtype, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, cudaStream_t stream)
{
    if (p.q_tiles == 0 || p.batch == 0)
        return cudaSuccess;
    const bool fp8 = kv_dtype == kKvFp8;
    switch (p.block_size) {
    case 16: return fp8 ? launch_one<kKvFp8, 16>(p, kmap, vmap, stream)
                        : launch_one<kKvInt8, 16>(p, kmap, vmap, stream);
    case 32: return fp8 ? launch_one<kKvFp8, 32>(p, kmap, vmap, stream)
                        : launch_one<kKvInt8, 32>(p, kmap, vmap, stream);
    case 64: return fp8 ? launch_one<kKvFp8, 64>(p, kmap, vmap, stream)
                        : launch_one<kKvInt8, 64>(p, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
