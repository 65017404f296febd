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
// Warp roles (15 warps; the softmax warps form one aligned group of four, as
// each warp reaches only the tensor-memory lanes 32 * (warp % 4) + 0..31):
//   warps 0-7  dequant: code tiles -> fp16 K/V tiles in the 128-byte-
//              swizzled layout [d half][key][64 d] (the K-major B operand of
//              Q K^T and the MN-major B operand of P V).  Warps 0-3 convert
//              K, warps 4-7 V, each 16 key rows of a tile (64 codes per thread
//              and tile), so every SM sub-partition runs one K and one V warp.
//              Each warp copies its own rows into a 4-stage ring with
//              coalesced 16-byte cp.async three tiles ahead and reads back
//              only those: no producer warp issues a tile's copies alone, and
//              no barrier hands the codes over.
//   warp 8     TMEM allocation and the Q K^T products, warp 14 the P V
//              products: a thread's tcgen05.mma returns only once the tensor
//              core has taken it, so one issuer queueing Q K(j+2)^T would
//              delay P(j+1) V.  One elected lane of the (converged) warp
//              issues each tcgen05 instruction.
//   warp 9     L2 prefetch of the tiles up to kPrefetchTiles ahead of the
//              conversion (FP16 caches: also the copies, see below).
//   warps 10-13 softmax: Q rows into tensor memory, S read with tcgen05.ld,
//              causal mask where a tile can cross a row's position, FP32
//              running max/sum, fp16 P written over its S columns, lazy O
//              rescale.  Up to 64 rows, row 4 i + q sits in lane i of quadrant
//              q and each such lane's scores are split over two threads
//              (16x32bx2 tensor-memory loads): exponentials of padding lanes
//              are never computed.  Beyond 64 rows each thread owns one row.
// Epilogue: the final fp16 row when one split covers the sequence, otherwise
// an FP32 partial (unnormalised O, max in log2 units, sum) in the decode
// workspace, which the decode merge kernel combines.
//
// FP16 caches need no conversion: warp 9 copies each key's two 128-byte row
// halves straight into a K/V buffer (the same swizzled layout) with cp.async,
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

constexpr int kThreads = 480;
constexpr int kKT = 64;              // keys per tile
// 4 K/V buffers: issuing Q K^T two tiles ahead holds tiles j, j+1 and j+2,
// and the fourth lets the dequantisation of j+3 start before P(j) V has
// completed.
constexpr int kKVBufs = 4;
// L2 prefetch distance in tiles (~100 KB per SM in flight for 8-bit K/V):
// with 16-token blocks the farthest prefetched block stays within 60 entries
// of the block-table window's base
constexpr int kPrefetchTiles = 6;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr int kDequantWarps = 8;   // warps 0-7
constexpr int kWarpMma = 8;
constexpr int kWarpPf = 9;         // L2 prefetch (FP16: the copies)
constexpr int kSoftmaxWarp0 = 10;  // warps 10-13: lane quadrants 2, 3, 0, 1
constexpr int kWarpPv = 14;        // issues P V (warp 8 issues Q K^T)

// tensor memory: S/P buffers 0 and 1 (P in the first 32 columns of its
// buffer), O, Q (two fp16 per column)
constexpr int kSBufs = 2;
constexpr uint32_t kTmS = 0, kTmO = kSBufs * 64, kTmQ = kTmO + 128;
static_assert(kTmQ + 64 <= 512, "tensor memory columns");
__device__ __forceinline__ int sbuf(int j) { return j % kSBufs; }
__device__ __forceinline__ uint32_t sphase(int j) { return (uint32_t)(j / kSBufs) & 1u; }

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr int kOffKV = 0;                                 // bufs x (K 8K+8K, V 8K+8K)
constexpr int kKVBuf = 32768;
// 8-bit codes: a ring of kCodeStages stages (K 8K, V 8K; rows 128-byte
// swizzled), each dequant warp copying and reading back only its own 16 rows;
// copies run kCodeStages - 1 tiles ahead of the conversion
constexpr int kCodeStages = 4;
constexpr int kOffCodes = kOffKV + kKVBufs * kKVBuf;
constexpr int kCodeStage = 16384;
constexpr int kOffScl = kOffCodes + kCodeStages * kCodeStage;   // stages x 8 warps x 32 halves (16 used)
constexpr int kOffKsf = kOffScl + kCodeStages * kDequantWarps * 64;   // bufs x 64 fp32 K factors
constexpr int kOffBars = kOffKsf + kKVBufs * 64 * 4;
constexpr int kNumBars = 1 + 3 * kKVBufs + 3 * kSBufs + 2;
constexpr int kOffTaddr = kOffBars + kNumBars * 8;
constexpr int kOffProgress = kOffTaddr + 8;   // tiles dequantised so far (prefetch pacing)
constexpr int kSmemBytes = kOffProgress + 8;
constexpr size_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

constexpr uint32_t kIdescQK = idesc_f16_f32(128, kKT, false);
constexpr uint32_t kIdescPV = idesc_f16_f32(128, 128, true);

struct Bars {
    uint64_t *q_full;
    uint64_t *kv_full, *kv_empty;       // [kKVBufs]
    uint64_t *s_full, *p_full, *pv_done;   // [S/P buffer]
    uint64_t *mma_done, *qk_done;      // each issuer's products retired (before TMEM is freed)
    uint64_t *kv_tma;                   // [kKVBufs] FP16: the buffer's copies landed
};

__device__ __forceinline__ Bars carve_bars(uint8_t *smem)
{
    uint64_t *b = reinterpret_cast<uint64_t *>(smem + kOffBars);
    Bars r;
    r.q_full = b;
    r.kv_full = b + 1;
    r.kv_empty = r.kv_full + kKVBufs;
    r.s_full = r.kv_empty + kKVBufs;
    r.p_full = r.s_full + kSBufs;
    r.pv_done = r.p_full + kSBufs;
    r.mma_done = r.pv_done + kSBufs;
    r.qk_done = r.mma_done + 1;
    r.kv_tma = r.qk_done + 1;
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

template <int KVT, int BS, bool kHalf>
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
        *reinterpret_cast<volatile int *>(smem + kOffProgress) = 0;
        for (int i = 0; i < kKVBufs; ++i) {
            mbar_init(&bars.kv_full[i], kDequantWarps);
            mbar_init(&bars.kv_empty[i], 1);
            mbar_init(&bars.kv_tma[i], 32);
        }
        for (int i = 0; i < kSBufs; ++i) {
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.p_full[i], 4);
            mbar_init(&bars.pv_done[i], 1);
        }
        mbar_init(bars.mma_done, 1);
        mbar_init(bars.qk_done, 1);
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

    if (warp == kWarpPf) {
        // -------------------------------------------- L2 prefetch / copies --
        const CacheView cv{p.k_cache, p.v_cache, p.k_scale_tok, p.v_scale_tok, p.num_kv_heads,
                           p.num_blocks, p.status};
        BlockWindow w;
        // every index stays inside the table row, even for a context longer
        // than the row can address (a caller error: those keys read block 0)
        w.init(p.block_table + (size_t)b * p.max_blocks_per_seq + blk_begin,
               min(nblk, p.max_blocks_per_seq - blk_begin), lane);
        if constexpr (KVT == kKvFp16) {
            // FP16 needs no conversion: 16-byte cp.async copies by all 32
            // lanes go straight into K/V buffer j % kKVBufs, and each lane
            // arrives on the buffer's barrier once its own copies have landed.
            // The tiles up to kPrefetchTiles past the one being copied are
            // first fetched into L2.
            int pf_next = kKVBufs;
            for (int j = 0; j < ntiles; ++j) {
                for (; pf_next < ntiles && pf_next <= j + kPrefetchTiles; ++pf_next)
                    prefetch_blocks<BS, KVT>(cv, h, w, pf_next * kBPT,
                                             min(kBPT, nblk - pf_next * kBPT), lane);
                const int s = j % kKVBufs;
                if (j >= kKVBufs &&
                    !warp_wait(&bars.kv_empty[s], ((j - kKVBufs) / kKVBufs) & 1, p.status))
                    break;
                const int blk0 = j * kBPT;   // within this split
                const uint32_t kv = sbase + kOffKV + s * kKVBuf;
                copy_fp16_rows<BS>(kv, kv + 16384, 8192, cv, h, w, blk0,
                                   min(kBPT, nblk - blk0), kKT, lane);
                cp_async_mbar_arrive(&bars.kv_tma[s]);
                if (j + 1 < ntiles)
                    w.slide(blk0 + kBPT, lane);
            }
            // copies this warp issued land before it exits
            cp_async_wait_all();
        } else {
            // 8-bit codes: each dequant warp loads its own rows one tile
            // ahead; this warp keeps the lines of up to kPrefetchTiles tiles
            // past the one being converted on their way into L2, paced by the
            // count of converted tiles.
            const volatile int *progress =
                reinterpret_cast<const volatile int *>(smem + kOffProgress);
            for (int j = 1; j < ntiles; ++j) {
                if (j > kPrefetchTiles &&
                    __shfl_sync(0xffffffffu, *progress, 0) < j - kPrefetchTiles) {
                    const uint64_t t0 = global_timer_ns();
                    bool ok = true;
                    while (__shfl_sync(0xffffffffu, *progress, 0) < j - kPrefetchTiles) {
                        __nanosleep(128);
                        // lane 0's clock and status decide, so the warp stays converged
                        const bool late = __shfl_sync(0xffffffffu,
                                                      global_timer_ns() - t0 > kWaitLimitNs ||
                                                          device_wait_failed(p.status),
                                                      0);
                        if (late) {
                            ok = false;
                            break;
                        }
                    }
                    if (!ok)
                        break;   // the dequant warps stopped: nothing left to prefetch for
                }
                w.slide(j * kBPT, lane);
                prefetch_blocks<BS, KVT>(cv, h, w, j * kBPT, min(kBPT, nblk - j * kBPT), lane);
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------ Q K^T issuer --
        // Two issuing warps, one per product: a thread's tcgen05.mma returns
        // only once the tensor core has accepted it, so a single issuer that
        // is queueing Q K(j+2)^T cannot issue P(j+1) V the moment P(j+1) is
        // ready.  S(k) overwrites P(k - kSBufs) in the same columns: Q K(k)^T
        // waits for that P V to complete (another thread issued it).
        if (ntiles > 0) {
            bool ok = warp_wait(bars.q_full, 0, p.status);
            tc_fence_after();
            const uint64_t kd0 = desc_sw128(sbase + kOffKV, 16, 1024);
            for (int k = 0; ok && k < ntiles; ++k) {
                if (!warp_wait(&bars.kv_full[k % kKVBufs], (k / kKVBufs) & 1, p.status))
                    break;
                if (k >= kSBufs &&
                    !warp_wait(&bars.pv_done[sbuf(k - kSBufs)], sphase(k - kSBufs), p.status))
                    break;
                tc_fence_after();
                const uint32_t sd = tmem + kTmS + sbuf(k) * kKT;
                const uint64_t kd = kd0 + (uint64_t)(((k % kKVBufs) * kKVBuf) >> 4);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts_elect(sd, tmem + kTmQ + ks * 8,
                                     kd + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4),
                                     kIdescQK, ks > 0 ? 1u : 0u);
                mma_commit_elect(&bars.s_full[sbuf(k)]);
            }
            // all of this thread's products retired before tensor memory is
            // freed (on an early exit some may still be running)
            mma_commit_elect(bars.qk_done);
            warp_wait(bars.qk_done, 0, p.status);
        }
    } else if (warp == kWarpPv) {
        // --------------------------------------------------- P V issuer --
        // P(j) follows S(j), which followed K(j) and V(j) (one barrier for
        // both halves of the buffer).  Its last commit covers every product:
        // each Q K^T completed before the P V of the same tile was issued.
        if (ntiles > 0) {
            const uint64_t vd0 = desc_sw128(sbase + kOffKV + 16384, 8192, 1024);
            for (int j = 0; j < ntiles; ++j) {
                if (!warp_wait(&bars.p_full[sbuf(j)], sphase(j), p.status))
                    break;
                tc_fence_after();
                const uint32_t pa = tmem + kTmS + sbuf(j) * kKT;
                const uint64_t vd = vd0 + (uint64_t)(((j % kKVBufs) * kKVBuf) >> 4);
#pragma unroll
                for (int ks = 0; ks < kKT / 16; ++ks)
                    mma_f16_ts_elect(tmem + kTmO, pa + ks * 8, vd + (uint64_t)((ks * 2048) >> 4),
                                     kIdescPV, (j > 0 || ks > 0) ? 1u : 0u);
                mma_commit_elect(&bars.pv_done[sbuf(j)]);
                mma_commit_elect(&bars.kv_empty[j % kKVBufs]);
            }
            mma_commit_elect(bars.mma_done);
            warp_wait(bars.mma_done, 0, p.status);
        }
    } else if (warp < kDequantWarps) {
        // ------------------------------------------------------ dequant --
        // warps 0-3 convert K, warps 4-7 V; warp w takes key rows
        // 16 (w & 3) .. +15 of every tile, thread l row 16 (w & 3) + l % 16 and
        // d half l / 16 (so 8 consecutive lanes touch 8 consecutive rows of one
        // half: no bank conflicts).  Each SM sub-partition (warp % 4) runs one
        // K and one V warp.
        const int isv = warp >> 2;
        const int row0 = 16 * (warp & 3);         // first key row of this warp in a tile
        const int row = row0 + (lane & 15);       // key row of this thread
        const int dh = lane >> 4;                 // d half: 16-byte code chunks 4 dh .. 4 dh + 3
        if constexpr (KVT == kKvFp16) {
            // the copies landed: clear the rows no key of this split may read
            // (never-written slots may hold NaN patterns, and 0 * NaN in P V
            // would poison O), then release the buffer to the MMA warp
            for (int j = 0; j < ntiles; ++j) {
                const int bj = j % kKVBufs;
                if (!warp_wait(&bars.kv_tma[bj], (j / kKVBufs) & 1, p.status))
                    break;
                const int key = key_begin + j * kKT + row;
                if (key >= ctx || j * kKT + row >= nblk * BS) {
                    uint8_t *kv = smem + kOffKV + bj * kKVBuf + isv * 16384 + dh * 8192;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(kv + row * 128 + c * 16) = z;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars.kv_full[bj]);
            }
        } else {
            // Each warp copies its own 16 rows of every tile (2 KB: 4 rows x
            // 128 bytes per instruction, 8 lanes per row, so each instruction
            // touches 4 cache lines; and the INT8 scales of those rows, 32
            // bytes) into the code ring kCodeStages - 1 tiles ahead with
            // 16-byte cp.async, and reads back only what it copied: per-thread
            // copy groups and a warp barrier, no cross-warp handshake.
            const uint8_t *cache = isv ? p.v_cache : p.k_cache;
            const uint16_t *scl = isv ? p.v_scale_tok : p.k_scale_tok;
            const int32_t *bt_row = p.block_table + (size_t)b * p.max_blocks_per_seq + blk_begin;
            // table entries read stay below this count (past it: block 0)
            const int nread = min(nblk, p.max_blocks_per_seq - blk_begin);
            const float kfac = p.scale_log2;
            // physical block of this warp's 16 rows of tile t (one block: BS >= 16)
            auto block_of = [&](int t) {
                const int e = (t * kKT + row0) / BS;
                int phys = (t < ntiles && e < nread) ? __ldg(bt_row + e) : 0;
#ifdef PKVQ_BOUNDS_CHECK
                if (phys < 0 || phys >= p.num_blocks) {
                    atomicOr(p.status, kStatusBadBlock);
                    phys = 0;
                }
#endif
                return phys;
            };
            // copies of tile t into stage t % kCodeStages (an empty group past the end)
            auto issue = [&](int t, int phys) {
                if (t < ntiles) {
                    const int st = t % kCodeStages;
                    const size_t y0 =
                        ((size_t)phys * p.num_kv_heads + h) * BS + (t * kKT + row0) % BS;
                    const uint32_t dst = sbase + kOffCodes + st * kCodeStage + isv * 8192;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 4 * i + (lane >> 3), c = lane & 7;   // row within the warp's 16
                        cp_async_16(dst + swz(row0 + r, c), cache + (y0 + r) * 128 + 16 * c);
                    }
                    if (KVT == kKvInt8 && lane < 2)   // 8 rows' scales per lane
                        cp_async_16(sbase + kOffScl + (st * kDequantWarps + warp) * 64 + 16 * lane,
                                    scl + y0 + 8 * lane);
                }
                cp_async_commit();
            };
            for (int t = 0; t < kCodeStages - 1; ++t)
                issue(t, block_of(t));
            int phys_next = block_of(kCodeStages - 1);
            for (int j = 0; j < ntiles; ++j) {
                // the stage of tile j - 1 takes tile j + kCodeStages - 1
                issue(j + kCodeStages - 1, phys_next);
                phys_next = block_of(j + kCodeStages);   // used by the next round
                cp_async_wait_group<kCodeStages - 1>();   // this thread's copies of tile j
                __syncwarp();                             // and the other lanes' copies
                const int st = j % kCodeStages, bj = j % kKVBufs;
                if (j >= kKVBufs &&
                    !warp_wait(&bars.kv_empty[bj], ((j - kKVBufs) / kKVBufs) & 1, p.status))
                    break;
                const uint8_t *codes = smem + kOffCodes + st * kCodeStage + isv * 8192;
                uint4 cur[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    cur[i] = *reinterpret_cast<const uint4 *>(codes + swz(row, 4 * dh + i));
                uint32_t sc = 0;
                if constexpr (KVT == kKvInt8)
                    sc = reinterpret_cast<const uint16_t *>(
                        smem + kOffScl + (st * kDequantWarps + warp) * 64)[lane & 15];
                uint8_t *kv = smem + kOffKV + bj * kKVBuf + isv * 16384 + dh * 8192;
                const int key = key_begin + j * kKT + row;
                const bool live = key < ctx && j * kKT + row < nblk * BS;
                const uint32_t s2 = sc | (sc << 16);   // INT8 V: the key's scale twice
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t hv[8];
                    cvt4<KVT>(cur[i].x, hv[0], hv[1]);
                    cvt4<KVT>(cur[i].y, hv[2], hv[3]);
                    cvt4<KVT>(cur[i].z, hv[4], hv[5]);
                    cvt4<KVT>(cur[i].w, hv[6], hv[7]);
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
                    // 16 codes -> 32 bytes: chunks 2 i and 2 i + 1 of the row's 128-byte half
                    *reinterpret_cast<uint4 *>(kv + swz(row, 2 * i)) =
                        make_uint4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<uint4 *>(kv + swz(row, 2 * i + 1)) =
                        make_uint4(hv[4], hv[5], hv[6], hv[7]);
                }
                if constexpr (KVT == kKvInt8) {
                    if (!isv && dh == 0) {   // per-key score factor: softmax scale * log2(e) * K scale
                        float *ksf = reinterpret_cast<float *>(smem + kOffKsf) + bj * 64;
                        ksf[row] =
                            live ? kfac * __half2float(__ushort_as_half((uint16_t)sc)) : 0.0f;
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars.kv_full[bj]);
                    if (warp == 0)   // prefetch pacing
                        *reinterpret_cast<volatile int *>(smem + kOffProgress) = j + 1;
                }
            }
            // copies this thread issued land before it exits
            cp_async_wait_all();
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ------------------------------------------------------ softmax --
        const int sw = warp & 3;           // lane quadrant of this warp
        const uint32_t tl = tmem + ((uint32_t)(32 * sw) << 16);
        // erow: the row in this thread's TMEM lane (Q in, O out); srow: the
        // row whose scores this thread processes.  Up to 64 rows, row 4 i + q
        // sits in lane i (< 16) of quadrant q and each lane's two threads
        // (t, t + 16) take half of its 64 keys each: the exponentials of
        // padding lanes are not computed.  Otherwise row == lane, one thread
        // per row.
        const int erow = kHalf ? (lane < 16 ? 4 * lane + sw : INT_MAX) : 32 * sw + lane;
        const int srow = kHalf ? 4 * (lane & 15) + sw : erow;
        const int kh = kHalf ? lane >> 4 : 0;   // key half of this thread
        constexpr int kCols = kHalf ? kKT / 2 : kKT;   // scores per thread and tile
        const bool valid = erow < p.rows;
        const bool svalid = srow < p.rows;
        const int tq = valid ? erow / G : 0, gq = valid ? erow % G : 0;
        // keys lo..pos are visible to this row (padding rows: the whole split)
        const int pos = svalid ? min(ctx - 1, query_position(p, b, ctx, srow / G)) : ctx - 1;
        const int lo = p.window > 0 && svalid ? pos - p.window + 1 : INT_MIN;
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
            if (!warp_wait(&bars.s_full[sbuf(j)], sphase(j), p.status)) {
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
            float v[kCols];
            if constexpr (kHalf) {
                uint32_t ua[32];
                tmem_ld16x2_32(tl + kTmS + sbuf(j) * kKT, ua);
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    v[c] = __uint_as_float(ua[c]);
            } else {
                uint32_t ua[32], ub[32];
                tmem_ld64(tl + kTmS + sbuf(j) * kKT, ua, ub);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    v[c] = __uint_as_float(ua[c]);
                    v[32 + c] = __uint_as_float(ub[c]);
                }
            }
            const int tile0 = key_begin + j * kKT;   // first key of the tile
            const int key0 = tile0 + kh * kCols;     // first key of this thread's scores
            if constexpr (KVT != kKvInt8) {
                const float2 f2 = make_float2(kfac, kfac);
#pragma unroll
                for (int c = 0; c < kCols; c += 2) {
                    const float2 r2 = __fmul2_rn(make_float2(v[c], v[c + 1]), f2);
                    v[c] = r2.x, v[c + 1] = r2.y;
                }
            } else {
                const float *ksf =
                    reinterpret_cast<const float *>(smem + kOffKsf) + (j % kKVBufs) * 64 + kh * kCols;
#pragma unroll
                for (int c = 0; c < kCols; c += 2) {
                    const float2 r2 = __fmul2_rn(make_float2(v[c], v[c + 1]),
                                                 make_float2(ksf[c], ksf[c + 1]));
                    v[c] = r2.x, v[c + 1] = r2.y;
                }
            }
            // keys past a row's position, past the context or past this
            // split are masked; only tiles that reach past the first row's
            // position or the split's end need it
            const int key_lim = key_begin + nblk * BS;   // first key past the split
            if (tile0 + kKT - 1 > pos_lo || tile0 + kKT > key_lim || tile0 < lo_hi) {
#pragma unroll
                for (int c = 0; c < kCols; ++c)
                    if (key0 + c > pos || key0 + c >= key_lim || key0 + c < lo)
                        v[c] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                m8[i] = v[i];
#pragma unroll
                for (int c = i + 8; c < kCols; c += 8)
                    m8[i] = fmaxf(m8[i], v[c]);
            }
            float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            if constexpr (kHalf)   // the row's other key half
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            // lazy rescale: only when the max grew by more than 2^8
            const bool need = m_used != -INFINITY && mx > m_used + kRescaleLog2;
            if (__any_sync(0xffffffffu, need)) {
                // O must hold P V of tile j-1 before it is rescaled
                if (!warp_wait(&bars.pv_done[sbuf(j - 1)], sphase(j - 1), p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float corr = need ? fast_exp2(m_used - mx) : 1.0f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {   // 16 columns at a time: the scores stay live
                    uint32_t o[16];
                    tmem_ld16(tl + kTmO + 16 * q, o);
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
                    tmem_st16(tl + kTmO + 16 * q, o);
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
            // P row over the first 32 columns of its S buffer (A operand of
            // P V), 32 keys (16 columns) at a time
#pragma unroll
            for (int g = 0; g < kCols / 32; ++g) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const int cc = 32 * g + c;
                    const float2 d = __fadd2_rn(make_float2(v[cc], v[cc + 1]), nmu);
                    const float2 e = make_float2(fast_exp2(d.x), fast_exp2(d.y));
                    acc[(c >> 1) & 3] = __fadd2_rn(acc[(c >> 1) & 3], e);
                    pk[c / 2] = pack_half2(e.x, e.y);
                }
                if constexpr (kHalf)
                    tmem_st16x2_16(tl + kTmS + sbuf(j) * kKT, pk);
                else
                    tmem_st16(tl + kTmS + sbuf(j) * kKT + 16 * g, pk);
            }
            const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
            const float2 a = __fadd2_rn(a01, a23);
            l += a.x + a.y;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.p_full[sbuf(j)]);
        }

        // ---- epilogue ----
        if constexpr (kHalf)   // each thread summed its own key half
            l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int jl = ntiles - 1;   // P V of the last tile retires after all others
        const bool have_o =
            ok && ntiles > 0 && warp_wait(&bars.pv_done[sbuf(jl)], sphase(jl), p.status);
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
            const size_t wrow = ((size_t)h * p.num_splits + slot) * p.rows_per_cta + erow;
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
    auto kern = p.rows <= 64 ? decode_tc_kernel<KVT, BS, true> : decode_tc_kernel<KVT, BS, false>;
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
