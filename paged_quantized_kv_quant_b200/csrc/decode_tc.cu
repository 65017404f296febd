// Decode / draft-verify attention with many query rows per KV head on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory),
// split-KV.
//
// Source: "1Cat-LLM" README, "Layer 2" (GQA multi-head packing into wider
// tensor-core work, online softmax with FP32 state, Split-KV with an FP32
// merge, MTP verify of several query tokens) and "Layer 1" (paged KV read
// once and wide); "ReVolta" PyPI page ("Weight and KV formats": 8-bit KV
// converted to FP16 for compute).
//
// pkvq_paged_attn_decode takes this kernel when a KV head has more than 16
// query rows (q_len x G, e.g. 5 verify tokens x 8 heads = 40).  The mma.sync
// kernel would split them into row groups, each fetching and converting every
// code again; here one CTA owns all rows of a (sequence, KV head) -- up to 128,
// one tensor-memory lane each -- and one split of its cached tokens, given by
// the same length-proportional slot map (split sizes a multiple of the 64-key
// tile), so each code is fetched and dequantised once.  With a single query
// tile, tensor memory holds two S buffers: S(j+2) = Q K(j+2)^T is issued as
// soon as P(j) V has been, and the softmax finds its next S ready.
//
// Warp roles (12 warps; the softmax warps form one aligned group of four, as
// each warp reaches only the tensor-memory lanes 32 * (warp % 4) + 0..31):
//   warps 0-3, 6-7  dequant: code tiles -> fp16 K/V tiles in the
//              128-byte-swizzled layout [d half][key][64 d] (the K-major B
//              operand of Q K^T and the MN-major B operand of P V), one key
//              row per thread: warps 0-1 convert d 0-63 of K, warps 6-7 d
//              64-127 of K, warps 2-3 all of V.  With one query tile nothing
//              else shares the conversion of a tile, so it takes six warps to
//              keep pace with the softmax; K is split further because Q K^T
//              of a tile waits for it.
//   warp 4     TMA producer: one 2-D box per cache block into a 5-stage ring.
//   warp 5     TMEM allocation; the whole warp runs the issue loop, one
//              elected lane issues each tcgen05 instruction.
//   warps 8-11 softmax, thread i owns row i: Q row into tensor memory, S row
//              read with tcgen05.ld, causal mask where a tile can cross a
//              row's position, FP32 running max/sum, fp16 P row written over
//              its S columns, lazy O rescale.
// Epilogue: the final fp16 row when one split covers the sequence, otherwise
// an FP32 partial (unnormalised O, max in log2 units, sum) in the decode
// workspace, which the decode merge kernel combines.
//
// FP16 caches need no conversion: the TMA warp copies each block's two
// 128-byte row halves straight into a K/V buffer (the same swizzled layout),
// and the dequant warps only clear the rows past the context or the split
// before releasing the buffer to the MMA warp (never-written slots may hold
// NaN patterns, and 0 * NaN in P V would poison O).
#include "common.cuh"
#include "internal.h"
#include "kv_stage.cuh"
#include "split_map.cuh"
#include "tc.cuh"

#include <climits>
#include <math.h>

namespace pkvq {
namespace {

constexpr int kThreads = 384;
constexpr int kKT = 64;              // keys per tile
// 5 code stages (80 KB per SM in flight) and 4 K/V buffers: issuing Q K^T
// two tiles ahead holds tiles j, j+1 and j+2, and the fourth lets the
// dequantisation of j+3 start before P(j) V has completed.
constexpr int kCodeStages = 5;
constexpr int kKVBufs = 4;
// L2 prefetch distance in tiles: with 16-token blocks the farthest prefetched
// block stays within 60 entries of the block-table window's base
constexpr int kPrefetchTiles = 6;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kDequantWarps = 6;   // warps 0-3 and 6-7

__device__ __forceinline__ bool is_dequant_warp(int w) { return w < 4 || w == 6 || w == 7; }
constexpr int kSoftmaxWarp0 = 8;

// tensor memory: S/P buffers 0 and 1 (P in the first 32 columns of its
// buffer), O, Q (two fp16 per column)
constexpr uint32_t kTmS = 0, kTmO = 128, kTmQ = 256;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr int kOffKV = 0;                                 // bufs x (K 8K+8K, V 8K+8K)
constexpr int kKVBuf = 32768;
constexpr int kOffCodes = kOffKV + kKVBufs * kKVBuf;      // stages x (K 8K, V 8K)
constexpr int kCodeStage = 16384;
constexpr int kOffScl = kOffCodes + kCodeStages * kCodeStage;   // stages x (K 64, V 64) halves
constexpr int kOffKsf = kOffScl + kCodeStages * 256;            // bufs x 64 fp32 K factors
constexpr int kOffBars = kOffKsf + kKVBufs * 64 * 4;
constexpr int kNumBars = 1 + 2 * kCodeStages + 3 * kKVBufs + 3 * 2 + 1;
constexpr int kOffTaddr = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = kOffTaddr + 16;
constexpr size_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

constexpr uint32_t kIdescQK = idesc_f16_f32(128, kKT, false);
constexpr uint32_t kIdescPV = idesc_f16_f32(128, 128, true);

struct Bars {
    uint64_t *q_full;
    uint64_t *code_full, *code_empty;   // [kCodeStages]
    uint64_t *kv_full, *kv_empty;       // [kKVBufs]
    uint64_t *s_full, *p_full, *pv_done;   // [S/P buffer]
    uint64_t *mma_done;
    uint64_t *kv_tma;                   // [kKVBufs] FP16: the buffer's copies landed
};

__device__ __forceinline__ Bars carve_bars(uint8_t *smem)
{
    uint64_t *b = reinterpret_cast<uint64_t *>(smem + kOffBars);
    Bars r;
    r.q_full = b;
    r.code_full = b + 1;
    r.code_empty = r.code_full + kCodeStages;
    r.kv_full = r.code_empty + kCodeStages;
    r.kv_empty = r.kv_full + kKVBufs;
    r.s_full = r.kv_empty + kKVBufs;
    r.p_full = r.s_full + 2;
    r.pv_done = r.p_full + 2;
    r.mma_done = r.pv_done + 2;
    r.kv_tma = r.mma_done + 1;
    return r;
}

// byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint32_t *status)
{
    const bool ok = mbar_wait(bar, parity, status);
    return __all_sync(0xffffffffu, ok);
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

template <int KVT, int BS>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const DecodeParams p)
{
    constexpr int kBPT = kKT / BS;   // cache blocks per key tile
    static_assert((kPrefetchTiles + 1) * kBPT <= 32, "prefetches stay in the table window");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Bars bars = carve_bars(smem);
    uint32_t *taddr_smem = reinterpret_cast<uint32_t *>(smem + kOffTaddr);

    const int slot = blockIdx.x;
    const int h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(bars.q_full, 4);
        for (int s = 0; s < kCodeStages; ++s) {
            mbar_init(&bars.code_full[s], 32);   // one cp.async arrival per producer lane
            mbar_init(&bars.code_empty[s], kDequantWarps);
        }
        for (int i = 0; i < kKVBufs; ++i) {
            mbar_init(&bars.kv_full[i], kDequantWarps);
            mbar_init(&bars.kv_empty[i], 1);
            mbar_init(&bars.kv_tma[i], 32);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.p_full[i], 4);
            mbar_init(&bars.pv_done[i], 1);
        }
        mbar_init(bars.mma_done, 1);
        fence_mbar_init();
    }
    // Inputs may come from the previous kernel: wait for it to complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // every warp computes the (sequence, split) of this slot (warp-uniform)
    const SplitInfo si = find_split<BS>(p, slot, -1);
    // a CTA-wide vote, so that the whole CTA leaves together
    if (__syncthreads_or(si.b < 0 || device_wait_failed(p.status)))
        return;
    const int b = si.b;
    const int ctx = si.ctx;
    const int nblk_seq = (ctx + BS - 1) / BS;
    const int blk_begin = si.blk0 + si.split * si.bpc;   // bpc is a multiple of kBPT
    const int blk_end = min(nblk_seq, blk_begin + si.bpc);
    const int nblk = max(0, blk_end - blk_begin);
    const int ntiles = (nblk + kBPT - 1) / kBPT;
    const int key_begin = blk_begin * BS;
    const int G = p.group;

    if (warp == kWarpMma) {
        tmem_alloc(taddr_smem, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_smem;

    if (warp == kWarpTma) {
        // ---------------------------------------------- copy producer --
        // 16-byte cp.async copies by all 32 lanes; each lane arrives on the
        // tile's barrier once its own copies have landed.  The tiles up to
        // kPrefetchTiles past the one being loaded are first fetched into L2.
        const CacheView cv{p.k_cache, p.v_cache, p.k_scale_tok, p.v_scale_tok, p.num_kv_heads,
                           p.num_blocks, p.status};
        BlockWindow w;
        // every index stays inside the table row, even for a context longer
        // than the row can address (a caller error: those keys read block 0)
        w.init(p.block_table + (size_t)b * p.max_blocks_per_seq + blk_begin,
               min(nblk, p.max_blocks_per_seq - blk_begin), lane);
        // FP16: each tile goes straight into K/V buffer j % kKVBufs
        constexpr int kRing = KVT == kKvFp16 ? kKVBufs : kCodeStages;
        int pf_next = kRing;
        for (int j = 0; j < ntiles; ++j) {
            for (; pf_next < ntiles && pf_next <= j + kPrefetchTiles; ++pf_next)
                prefetch_blocks<BS, KVT>(cv, h, w, pf_next * kBPT,
                                         min(kBPT, nblk - pf_next * kBPT), lane);
            const int s = j % kRing;
            uint64_t *empty = KVT == kKvFp16 ? bars.kv_empty : bars.code_empty;
            if (j >= kRing && !warp_wait(&empty[s], ((j - kRing) / kRing) & 1, p.status))
                break;
            const int blk0 = j * kBPT;   // within this split
            const int nb = min(kBPT, nblk - blk0);
            if constexpr (KVT == kKvFp16) {
                const uint32_t kv = sbase + kOffKV + s * kKVBuf;
                copy_fp16_rows<BS>(kv, kv + 16384, 8192, cv, h, w, blk0, nb, kKT, lane);
                cp_async_mbar_arrive(&bars.kv_tma[s]);
            } else {
                const uint32_t dst = sbase + kOffCodes + s * kCodeStage;
                copy_code_rows<BS>(dst, dst + 8192, cv, h, w, blk0, nb, kKT, lane);
                if constexpr (KVT == kKvInt8) {
                    const uint32_t sd = sbase + kOffScl + s * 256;
                    copy_int8_scales<BS>(sd, sd + 128, cv, h, w, blk0, nb, lane);
                }
                cp_async_mbar_arrive(&bars.code_full[s]);
            }
            if (j + 1 < ntiles)
                w.slide(blk0 + kBPT, lane);
        }
        // copies this warp issued land before it exits
        cp_async_wait_all();
    } else if (warp == kWarpMma) {
        // --------------------------------------------------- MMA issuer --
        // S(k) overwrites P(k-2) in the same buffer, so Q K(k)^T is issued
        // once K(k) is dequantised and P(k-2) V has been issued (the tensor
        // core executes one thread's MMAs in issue order).  Nothing blocks on
        // one event while another could proceed; when a round issued
        // nothing, the warp sleeps (bounded) on the P that is due.
        if (ntiles > 0) {
            bool ok = warp_wait(bars.q_full, 0, p.status);
            tc_fence_after();
            const uint64_t kd0 = desc_sw128(sbase + kOffKV, 16, 1024);
            const uint64_t vd0 = desc_sw128(sbase + kOffKV + 16384, 8192, 1024);
            constexpr uint32_t kPollSleepNs = 200;
            int nqk = 0, nxt = 0;
            uint64_t t_last = 0;
            uint32_t idle = 0;
            while (ok && nxt < ntiles) {
                bool progressed = false;
                if (nqk < ntiles && nqk <= nxt + 1 &&
                    __any_sync(0xffffffffu, mbar_test_wait(&bars.kv_full[nqk % kKVBufs],
                                                           (nqk / kKVBufs) & 1))) {
                    tc_fence_after();
                    const uint32_t sd = tmem + kTmS + (nqk & 1) * kKT;
                    const uint64_t kd = kd0 + (uint64_t)(((nqk % kKVBufs) * kKVBuf) >> 4);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_f16_ts_elect(sd, tmem + kTmQ + ks * 8,
                                         kd + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4),
                                         kIdescQK, ks > 0 ? 1u : 0u);
                    mma_commit_elect(&bars.s_full[nqk & 1]);
                    ++nqk;
                    progressed = true;
                }
                if (nxt < nqk) {
                    uint64_t *bar = &bars.p_full[nxt & 1];
                    const uint32_t par = (nxt >> 1) & 1;
                    const bool rdy = progressed ? mbar_test_wait(bar, par)
                                                : mbar_try_wait_for(bar, par, kPollSleepNs);
                    if (__any_sync(0xffffffffu, rdy)) {
                        tc_fence_after();
                        const uint32_t pa = tmem + kTmS + (nxt & 1) * kKT;
                        const uint64_t vd = vd0 + (uint64_t)(((nxt % kKVBufs) * kKVBuf) >> 4);
#pragma unroll
                        for (int ks = 0; ks < kKT / 16; ++ks)
                            mma_f16_ts_elect(tmem + kTmO, pa + ks * 8,
                                             vd + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                                             (nxt > 0 || ks > 0) ? 1u : 0u);
                        mma_commit_elect(&bars.pv_done[nxt & 1]);
                        mma_commit_elect(&bars.kv_empty[nxt % kKVBufs]);
                        ++nxt;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else if ((++idle & 15u) == 0) {
                    // lane 0's clock decides, so that the warp stays converged
                    const uint64_t now = __shfl_sync(0xffffffffu, global_timer_ns(), 0);
                    if (idle == 16u) {
                        t_last = now;
                    } else if (now - t_last > kWaitLimitNs) {
                        if (lane == 0)
                            atomicOr(p.status, kStatusWaitTimeout);
                        ok = false;
                    }
                }
            }
            mma_commit_elect(bars.mma_done);
            warp_wait(bars.mma_done, 0, p.status);
        }
    } else if (is_dequant_warp(warp)) {
        // ------------------------------------------------------ dequant --
        const int row = (warp & 1) * 32 + lane;   // key row of this thread
        const int isv = (warp == 2 || warp == 3) ? 1 : 0;   // 0: K (warps 0, 1, 6, 7), 1: V
        const int c0 = warp >= 6 ? 4 : 0;         // first 16-byte chunk of the row
        const int nch = isv ? 8 : 4;              // chunks this warp converts
        const float kfac = p.scale_log2;
        if constexpr (KVT == kKvFp16) {
            // clear the rows no key of this split may read, then release
            for (int j = 0; j < ntiles; ++j) {
                const int bj = j % kKVBufs;
                if (!warp_wait(&bars.kv_tma[bj], (j / kKVBufs) & 1, p.status))
                    break;
                const int key = key_begin + j * kKT + row;
                if (key >= ctx || j * kKT + row >= nblk * BS) {
                    // the whole 128-byte row of each d half this warp owns
                    // (K: half c0 / 4; V: both)
                    uint8_t *kv = smem + kOffKV + bj * kKVBuf + isv * 16384;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!isv && hh != (c0 >> 2))
                            continue;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(kv + hh * 8192 + row * 128 + c * 16) = z;
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars.kv_full[bj]);
            }
        }
        for (int j = 0; KVT != kKvFp16 && j < ntiles; ++j) {
            const int s = j % kCodeStages, bj = j % kKVBufs;
            if (!warp_wait(&bars.code_full[s], (j / kCodeStages) & 1, p.status))
                break;
            if (j >= kKVBufs &&
                !warp_wait(&bars.kv_empty[bj], ((j - kKVBufs) / kKVBufs) & 1, p.status))
                break;
            const uint8_t *codes = smem + kOffCodes + s * kCodeStage + isv * 8192;
            const uint16_t *scl = reinterpret_cast<const uint16_t *>(smem + kOffScl + s * 256);
            uint8_t *kv = smem + kOffKV + bj * kKVBuf + isv * 16384;
            const int key = key_begin + j * kKT + row;
            const bool live = key < ctx && j * kKT + row < nblk * BS;
            uint32_t s2 = 0u;
            if constexpr (KVT == kKvInt8) {
                const uint32_t sc = scl[64 + row];   // V scale of this key
                s2 = sc | (sc << 16);
            }
            // all eight 16-byte code chunks of the row are loaded before any is
            // converted: one shared-memory round trip per tile, not eight
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < nch)
                    wv[i] = *reinterpret_cast<const uint4 *>(codes + swz(row, c0 + i));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i >= nch)
                    break;
                const int cc = c0 + i;   // 16-byte code chunk
                const uint4 w = wv[i];
                uint32_t hv[8];
                cvt4<KVT>(w.x, hv[0], hv[1]);
                cvt4<KVT>(w.y, hv[2], hv[3]);
                cvt4<KVT>(w.z, hv[4], hv[5]);
                cvt4<KVT>(w.w, hv[6], hv[7]);
                if constexpr (KVT == kKvInt8) {
                    if (isv) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&hv[e]),
                                                *reinterpret_cast<const __half2 *>(&s2));
                            hv[e] = *reinterpret_cast<uint32_t *>(&x);
                        }
                    }
                }
                if (!live) {   // past the context or the split: codes may be anything
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        hv[e] = 0u;
                }
                uint8_t *dst = kv + (cc >> 2) * 8192;
                *reinterpret_cast<uint4 *>(dst + swz(row, (2 * cc) & 7)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<uint4 *>(dst + swz(row, (2 * cc + 1) & 7)) =
                    make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
            if constexpr (KVT == kKvInt8) {
                if (!isv && c0 == 0) {   // per-key score factor: softmax scale * log2(e) * K scale
                    float *ksf = reinterpret_cast<float *>(smem + kOffKsf) + bj * 64;
                    ksf[row] = live ? kfac * __half2float(__ushort_as_half(scl[row])) : 0.0f;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.code_empty[s]);
                mbar_arrive(&bars.kv_full[bj]);
            }
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------ softmax --
        const int r = tid - 32 * kSoftmaxWarp0;   // row == TMEM lane
        const int sw = warp & 3;           // lane quadrant of this warp
        const uint32_t tl = tmem + ((uint32_t)(32 * sw) << 16);
        const int tq = r / G, gq = r % G;
        const bool valid = r < p.rows;
        // keys lo..pos are visible to this row (padding rows: the whole split)
        const int pos = valid ? min(ctx - 1, query_position(p, b, ctx, tq)) : ctx - 1;
        const int lo = p.window > 0 && valid ? pos - p.window + 1 : INT_MIN;
        // a tile needs masking when it reaches past the lowest position or
        // starts below the highest window start of the rows
        int pos_lo = ctx - 1, lo_hi = INT_MIN;
        for (int t = 0; t < p.q_len; ++t) {
            const int ps = min(ctx - 1, query_position(p, b, ctx, t));
            pos_lo = min(pos_lo, ps);
            if (p.window > 0)
                lo_hi = max(lo_hi, ps - p.window + 1);
        }
        const size_t qrow = ((size_t)b * p.q_len + tq) * p.num_q_heads + (size_t)h * G + gq;

        // Q row -> tensor memory (two fp16 per column), zeros for padding rows
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.q + qrow * kHeadDim);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = valid ? __ldg(src + half * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * c] = v.x, w[4 * c + 1] = v.y, w[4 * c + 2] = v.z, w[4 * c + 3] = v.w;
                }
                tmem_st32(tl + kTmQ + 32 * half, w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.q_full);
        }

        float kfac = p.scale_log2;
        if constexpr (kv_has_head_scale(KVT))
            kfac *= __ldg(p.k_scale + h * p.scale_stride);
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!warp_wait(&bars.s_full[j & 1], (j >> 1) & 1, p.status)) {
                ok = false;
                break;
            }
            if constexpr (KVT == kKvInt8) {
                // the per-key factors below were written by the dequant warps
                if (!warp_wait(&bars.kv_full[j % kKVBufs], (j / kKVBufs) & 1, p.status)) {
                    ok = false;
                    break;
                }
            }
            tc_fence_after();
            float v[kKT];
            {
                uint32_t ua[32], ub[32];
                tmem_ld64(tl + kTmS + (j & 1) * kKT, ua, ub);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    v[c] = __uint_as_float(ua[c]);
                    v[32 + c] = __uint_as_float(ub[c]);
                }
            }
            const int key0 = key_begin + j * kKT;
            if constexpr (KVT != kKvInt8) {
                const float2 f2 = make_float2(kfac, kfac);
#pragma unroll
                for (int c = 0; c < kKT; c += 2) {
                    const float2 r2 = __fmul2_rn(make_float2(v[c], v[c + 1]), f2);
                    v[c] = r2.x, v[c + 1] = r2.y;
                }
            } else {
                const float *ksf =
                    reinterpret_cast<const float *>(smem + kOffKsf) + (j % kKVBufs) * 64;
#pragma unroll
                for (int c = 0; c < kKT; c += 2) {
                    const float2 r2 = __fmul2_rn(make_float2(v[c], v[c + 1]),
                                                 make_float2(ksf[c], ksf[c + 1]));
                    v[c] = r2.x, v[c + 1] = r2.y;
                }
            }
            // keys past a row's position, past the context or past this
            // split are masked; only tiles that reach past the first row's
            // position or the split's end need it
            const int key_lim = key_begin + nblk * BS;   // first key past the split
            if (key0 + kKT - 1 > pos_lo || key0 + kKT > key_lim || key0 < lo_hi) {
#pragma unroll
                for (int c = 0; c < kKT; ++c)
                    if (key0 + c > pos || key0 + c >= key_lim || key0 + c < lo)
                        v[c] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                m8[i] = v[i];
#pragma unroll
                for (int c = i + 8; c < kKT; c += 8)
                    m8[i] = fmaxf(m8[i], v[c]);
            }
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            // lazy rescale: only when the max grew by more than 2^8
            const bool need = m_used != -INFINITY && mx > m_used + kRescaleLog2;
            if (__any_sync(0xffffffffu, need)) {
                // O must hold P V of tile j-1 before it is rescaled
                if (!warp_wait(&bars.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float corr = need ? fast_exp2(m_used - mx) : 1.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    tmem_ld32(tl + kTmO + 32 * q, o);
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
                    tmem_st32(tl + kTmO + 32 * q, o);
                }
                if (need) {
                    l *= corr;
                    m_used = mx;
                }
            }
            if (m_used == -INFINITY)
                m_used = mx;   // first finite max (O is still empty)
            const float mu = m_used == -INFINITY ? 0.0f : m_used;
            const float2 nmu = make_float2(-mu, -mu);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            uint32_t pk[kKT / 2];
#pragma unroll
            for (int c = 0; c < kKT; c += 2) {
                const float2 d = __fadd2_rn(make_float2(v[c], v[c + 1]), nmu);
                const float2 e = make_float2(fast_exp2(d.x), fast_exp2(d.y));
                acc[(c >> 1) & 3] = __fadd2_rn(acc[(c >> 1) & 3], e);
                pk[c / 2] = pack_half2(e.x, e.y);
            }
            const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
            const float2 a = __fadd2_rn(a01, a23);
            l += a.x + a.y;
            // P row over the first 32 columns of its S buffer (A operand of P V)
            tmem_st32(tl + kTmS + (j & 1) * kKT, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.p_full[j & 1]);
        }

        // ---- epilogue ----
        const int jl = ntiles - 1;   // P V of the last tile retires after all others
        const bool have_o =
            ok && ntiles > 0 && warp_wait(&bars.pv_done[jl & 1], (jl >> 1) & 1, p.status);
        if (have_o)
            tc_fence_after();
        if (si.nsplit == 1) {
            float vfac = 1.0f;
            if constexpr (kv_has_head_scale(KVT))
                vfac = __ldg(p.v_scale + h * p.scale_stride);
            const float f = (have_o && l > 0.0f) ? vfac / l : 0.0f;
            __half *dst = p.out + qrow * kHeadDim;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                if (have_o)   // warp-uniform
                    tmem_ld32(tl + kTmO + 32 * q, o);
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            y[e] = have_o ? __uint_as_float(o[c + e]) * f : 0.0f;
                        uint4 w;
                        w.x = pack_half2(y[0], y[1]);
                        w.y = pack_half2(y[2], y[3]);
                        w.z = pack_half2(y[4], y[5]);
                        w.w = pack_half2(y[6], y[7]);
                        *reinterpret_cast<uint4 *>(dst + 32 * q + c) = w;
                    }
                }
            }
            if (valid && p.lse)
                p.lse[qrow] = (have_o && l > 0.0f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
        } else {
            // FP32 partial: unnormalised O, max (log2 units) and sum of row r
            const size_t wrow = ((size_t)h * p.num_splits + slot) * p.rows_per_cta + r;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                if (have_o)
                    tmem_ld32(tl + kTmO + 32 * q, o);
                if (valid) {
                    float4 *dst = reinterpret_cast<float4 *>(p.ws_o + wrow * kHeadDim + 32 * q);
#pragma unroll
                    for (int c = 0; c < 32; c += 4)
                        dst[c / 4] = have_o ? make_float4(__uint_as_float(o[c]),
                                                          __uint_as_float(o[c + 1]),
                                                          __uint_as_float(o[c + 2]),
                                                          __uint_as_float(o[c + 3]))
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (valid)
                *reinterpret_cast<float2 *>(p.ws_ml + wrow * 2) =
                    have_o ? make_float2(m_used, l) : make_float2(-INFINITY, 0.0f);
        }
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int KVT, int BS>
cudaError_t launch_tc(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                      cudaStream_t stream)
{
    auto kern = decode_tc_kernel<KVT, BS>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.num_splits, p.num_kv_heads, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, kmap, vmap, p);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeParams &p, int kv_dtype, const CUtensorMap &kmap,
                             const CUtensorMap &vmap, cudaStream_t stream)
{
    switch (kv_dtype * 100 + p.block_size) {
#define PKVQ_TC_CASE(T, B) \
    case T * 100 + B: return launch_tc<T, B>(p, kmap, vmap, stream);
        PKVQ_TC_CASE(kKvFp8, 16) PKVQ_TC_CASE(kKvFp8, 32) PKVQ_TC_CASE(kKvFp8, 64)
        PKVQ_TC_CASE(kKvInt8, 16) PKVQ_TC_CASE(kKvInt8, 32) PKVQ_TC_CASE(kKvInt8, 64)
        PKVQ_TC_CASE(kKvE5m2, 16) PKVQ_TC_CASE(kKvE5m2, 32) PKVQ_TC_CASE(kKvE5m2, 64)
        PKVQ_TC_CASE(kKvFp16, 16) PKVQ_TC_CASE(kKvFp16, 32) PKVQ_TC_CASE(kKvFp16, 64)
#undef PKVQ_TC_CASE
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
