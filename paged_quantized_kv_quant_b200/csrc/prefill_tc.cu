// Causal (chunked) prefill over the paged 8-bit cache on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Source: "1Cat-LLM" README, "Layer 2" (causal online softmax with FP32
// accumulation, GQA multi-head packing, Wide QK/PV tiles, prefix / causal-tail
// separation) and "Layer 1" (pages read once and wide); "ReVolta" PyPI page
// ("Weight and KV formats": 8-bit KV converted to FP16 for compute; chunked
// prefill with an 8,192-token budget).
//
// A CTA owns two adjacent query tiles A and B of 128 rows each (a tile is
// 128/G query tokens x the G query heads of one KV head).  Both tiles read the
// same keys, so every 64-key tile is fetched and dequantised once for 256
// query rows.  Q and P are kept in tensor memory, so the MMAs read only the
// fp16 K/V tiles from shared memory (operand bandwidth, not arithmetic, is
// what bounds a 128 x 64 product).  Warp roles (12 warps):
//   warps 0-1   dequant: E4M3/int8 code tiles -> fp16 K and V tiles in the
//               128-byte-swizzled canonical layout [d half][key][64 d].  The
//               same bytes are the K-major B operand of S = Q K^T and the
//               MN-major B operand of O = P V, so V is never transposed.
//   warp 2      TMA producer: one 2-D tensor copy per cache block and head
//               into a 3-stage code ring; block ids come from a register window.
//   warp 3      allocates all 512 TMEM columns (per tile: S/P 64, O 128, Q 64)
//               and issues every MMA: the whole warp runs the loop on
//               warp-uniform values and an elected lane issues each tcgen05
//               instruction.  It serves whichever tile has its P ready
//               (O += P V, then S = Q K_next in the same columns), sleeping
//               with a bounded mbarrier wait on the tile that is due.
//               Completion is signalled with tcgen05.commit on mbarriers.
//   warps 4-7   softmax for tile A, warps 8-11 softmax for tile B: thread i of
//               a group owns row i (TMEM lane i): it stores its Q row in TMEM,
//               reads its S row, masks only on tiles that cross the diagonal,
//               keeps the FP32 running max/sum in registers, writes its fp16 P
//               row over the S columns it came from, and rescales its O row in
//               TMEM only when the row maximum grew by more than 2^8.  The
//               tensor core runs one group's products while the other group's
//               softmax runs.
//
// FP16 caches need no conversion: the TMA warp copies each block's two
// 128-byte row halves straight into a K/V buffer, and the dequant warps only
// clear rows past the context.  With a sliding window w ("1Cat-LLM" README,
// "DFlash2 Long-Context Decay") the key loop starts at the tile holding the
// window start of the CTA's first row, and rows mask keys below their own
// window start.
#include "common.cuh"
#include "internal.h"
#include "kv_stage.cuh"
#include "tc.cuh"

#include <climits>
#include <math.h>

namespace pkvq {
namespace {

constexpr int kThreads = 384;
constexpr int kKT = 64;              // keys per tile
constexpr int kCodeStages = 3;
constexpr int kKVBufs = 4;           // dequantised K/V tiles in flight
// L2 prefetch distance in tiles: with 16-token blocks the farthest prefetched
// block stays within 60 entries of the block-table window's base
constexpr int kPrefetchTiles = 6;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

constexpr int kWarpTma = 2;
constexpr int kWarpMma = 3;
constexpr int kDequantWarps = 2;

// tensor memory, per query tile x at x * 256: S/P (P in the first 32), O, Q
constexpr uint32_t kTmS = 0, kTmO = 64, kTmQ = 192;

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
    uint64_t *s_full, *p_full, *pv_done;   // [tile]
    uint64_t *mma_done;                 // all MMAs retired (before TMEM is freed)
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

// Every lane waits; the result is made warp-uniform so that a (pathological)
// timeout makes the whole warp leave its loop together.
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

// Per-tile geometry of one of the CTA's two query tiles.
struct QTile {
    int q0;        // first query token (within the sequence)
    int pos_lo;    // position of its first token
    int pos_hi;    // position of its last token
    int ntiles;    // key tiles it needs from the CTA's first tile jbase on
                   // (0: tile absent or sees no key)
};

__device__ __forceinline__ QTile make_qtile(int tile, int tokens_per_tile, int q_len, int ctx,
                                            int jbase)
{
    QTile t;
    t.q0 = tile * tokens_per_tile;
    t.pos_lo = ctx - q_len + t.q0;
    t.pos_hi = t.pos_lo;
    t.ntiles = 0;
    if (t.q0 < q_len) {
        const int tq_end = min(q_len, t.q0 + tokens_per_tile);
        t.pos_hi = ctx - q_len + tq_end - 1;
        const int nkeys = max(0, min(ctx, ctx - q_len + tq_end));
        t.ntiles = max(0, (nkeys + kKT - 1) / kKT - jbase);
    }
    return t;
}

template <int KVT, int BS>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const PrefillParams p)
{
    constexpr int kBPT = kKT / BS;   // cache blocks per key tile
    static_assert((kPrefetchTiles + 1) * kBPT <= 32, "prefetches stay in the table window");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Bars bars = carve_bars(smem);
    uint32_t *taddr_smem = reinterpret_cast<uint32_t *>(smem + kOffTaddr);

    const int npairs = (p.q_tiles + 1) / 2;
    const int pair = npairs - 1 - blockIdx.x;   // longest causal work first
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int q_start = p.cu_seqlens_q[b];
    const int q_len = p.cu_seqlens_q[b + 1] - q_start;
    if (2 * pair * p.tokens_per_tile >= q_len || device_wait_failed(p.status))
        return;
    const int ctx = p.context_lens[b];
    const int G = p.group;
    // first key tile any row of the CTA sees (tile A holds the lower positions)
    const int jbase =
        p.window > 0 ? max(0, ctx - q_len + 2 * pair * p.tokens_per_tile - p.window + 1) / kKT : 0;
    const QTile qt[2] = {make_qtile(2 * pair, p.tokens_per_tile, q_len, ctx, jbase),
                         make_qtile(2 * pair + 1, p.tokens_per_tile, q_len, ctx, jbase)};
    const int ntiles = max(qt[0].ntiles, qt[1].ntiles);   // counted from jbase
    const int nblk_seq = (ctx + BS - 1) / BS;
    const int blk_base = jbase * kBPT;                    // first block read

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(bars.q_full, 8);
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
        w.init(p.block_table + (size_t)b * p.max_blocks_per_seq + blk_base,
               min(min(nblk_seq - blk_base, ntiles * kBPT), p.max_blocks_per_seq - blk_base),
               lane);
        // FP16: each tile goes straight into K/V buffer j % kKVBufs
        constexpr int kRing = KVT == kKvFp16 ? kKVBufs : kCodeStages;
        int pf_next = kRing;
        for (int j = 0; j < ntiles; ++j) {
            for (; pf_next < ntiles && pf_next <= j + kPrefetchTiles; ++pf_next)
                prefetch_blocks<BS, KVT>(cv, h, w, pf_next * kBPT,
                                         min(kBPT, nblk_seq - blk_base - pf_next * kBPT), lane);
            const int s = j % kRing;
            uint64_t *empty = KVT == kKvFp16 ? bars.kv_empty : bars.code_empty;
            if (j >= kRing && !warp_wait(&empty[s], ((j - kRing) / kRing) & 1, p.status))
                break;
            const int blk0 = j * kBPT;   // from blk_base
            const int nb = min(kBPT, nblk_seq - blk_base - blk0);
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
        // Serves whichever query tile has its P ready (no head-of-line
        // blocking between the two softmax groups); a K/V buffer is released
        // once every tile that uses it has issued its P V product.  The whole
        // warp runs this loop on warp-uniform values (every wait and probe is
        // made uniform by a vote) and one elected lane issues each tcgen05
        // instruction.
        if (ntiles > 0) {
            bool ok = warp_wait(bars.q_full, 0, p.status);
            tc_fence_after();
            // descriptors of K/V buffer 0; buffer b adds b * kKVBuf bytes
            const uint64_t kd0 = desc_sw128(sbase + kOffKV, 16, 1024);
            const uint64_t vd0 = desc_sw128(sbase + kOffKV + 16384, 8192, 1024);
            auto qk = [&](int x, int j) -> bool {   // S_x = Q_x K(j)^T
                const int kvb = j % kKVBufs;
                if (!warp_wait(&bars.kv_full[kvb], (j / kKVBufs) & 1, p.status))
                    return false;
                tc_fence_after();
                const uint32_t tx = tmem + x * 256;
                const uint64_t kd = kd0 + (uint64_t)((kvb * kKVBuf) >> 4);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts_elect(tx + kTmS, tx + kTmQ + ks * 8,
                                     kd + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4),
                                     kIdescQK, ks > 0 ? 1u : 0u);
                mma_commit_elect(&bars.s_full[x]);
                return true;
            };
            auto pv = [&](int x, int j) {   // O_x += P_x(j) V(j); P_x(j) is ready
                tc_fence_after();
                const uint32_t tx = tmem + x * 256;
                const uint64_t vd = vd0 + (uint64_t)(((j % kKVBufs) * kKVBuf) >> 4);
#pragma unroll
                for (int ks = 0; ks < kKT / 16; ++ks)
                    mma_f16_ts_elect(tx + kTmO, tx + kTmS + ks * 8,
                                     vd + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                                     (j > 0 || ks > 0) ? 1u : 0u);
                mma_commit_elect(&bars.pv_done[x]);
            };
            for (int x = 0; ok && x < 2; ++x)
                if (qt[x].ntiles > 0 && !qk(x, 0))
                    ok = false;
            int nxt[2] = {0, 0};   // next P V tile of each query tile
            int released = 0;      // K/V tiles released so far
            // The warp sleeps (bounded, kPollSleepNs) on the barrier of the tile
            // whose P is due first, so it neither spins on issue slots the
            // softmax warps of its scheduler need nor reacts late to that
            // tile; the other tile is then probed without blocking.  The clock
            // is read every 16 idle rounds.
            constexpr uint32_t kPollSleepNs = 200;
            uint64_t t_last = 0;
            uint32_t idle = 0;
            while (ok && (nxt[0] < qt[0].ntiles || nxt[1] < qt[1].ntiles)) {
                bool progressed = false;
                // the tile due first: fewer P V products issued (A on ties)
                const int xd = (nxt[0] < qt[0].ntiles &&
                                (nxt[0] <= nxt[1] || nxt[1] >= qt[1].ntiles)) ? 0 : 1;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int x = xd ^ k;
                    const int j = nxt[x];
                    if (j >= qt[x].ntiles)
                        continue;
                    const bool rdy = k == 0
                                         ? mbar_try_wait_for(&bars.p_full[x], j & 1, kPollSleepNs)
                                         : mbar_test_wait(&bars.p_full[x], j & 1);
                    if (!__any_sync(0xffffffffu, rdy))
                        continue;
                    pv(x, j);
                    nxt[x] = j + 1;
                    progressed = true;
                    // The next S overwrites this tile's P in the same columns;
                    // the tensor core executes a thread's MMAs in issue order.
                    if (j + 1 < qt[x].ntiles && !qk(x, j + 1)) {
                        ok = false;
                        break;
                    }
                }
                while (released < ntiles && (released >= qt[0].ntiles || nxt[0] > released) &&
                       (released >= qt[1].ntiles || nxt[1] > released)) {
                    mma_commit_elect(&bars.kv_empty[released % kKVBufs]);
                    ++released;
                }
                if (progressed) {
                    idle = 0;
                } else if ((++idle & 15u) == 0) {
                    // lane 0's clock decides, so that the warp stays converged
                    const uint64_t now = __shfl_sync(0xffffffffu, global_timer_ns(), 0);
                    if (idle == 16u) {
                        t_last = now;   // first check of this idle stretch
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
    } else if (warp < kDequantWarps) {
        // ------------------------------------------------------ dequant --
        const int row = tid;   // 0..63: this thread converts key row `row` of K and V
        const float kfac = p.scale_log2;
        if constexpr (KVT == kKvFp16) {
            // clear the rows past the context, then release the buffer
            for (int j = 0; j < ntiles; ++j) {
                const int bj = j % kKVBufs;
                if (!warp_wait(&bars.kv_tma[bj], (j / kKVBufs) & 1, p.status))
                    break;
                if ((jbase + j) * kKT + row >= ctx) {
                    uint8_t *kv = smem + kOffKV + bj * kKVBuf;
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int hh = 0; hh < 4; ++hh)   // K d halves 0, 1, V d halves 0, 1
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(kv + hh * 8192 + row * 128 + c * 16) = z;
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
            const uint8_t *codes = smem + kOffCodes + s * kCodeStage;
            const uint16_t *scl = reinterpret_cast<const uint16_t *>(smem + kOffScl + s * 256);
            uint8_t *kv = smem + kOffKV + bj * kKVBuf;
            const int key0 = (jbase + j) * kKT;
#pragma unroll 4
            for (int k = 0; k < 16; ++k) {
                const int isv = k >> 3;
                const int cc = k & 7;   // 16-byte code chunk
                const uint4 w = *reinterpret_cast<const uint4 *>(codes + isv * 8192 + swz(row, cc));
                uint32_t hv[8];
                cvt4<KVT>(w.x, hv[0], hv[1]);
                cvt4<KVT>(w.y, hv[2], hv[3]);
                cvt4<KVT>(w.z, hv[4], hv[5]);
                cvt4<KVT>(w.w, hv[6], hv[7]);
                if constexpr (KVT == kKvInt8) {
                    if (isv) {
                        const uint32_t sc = scl[64 + row];
                        const uint32_t s2 = sc | (sc << 16);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&hv[e]),
                                                *reinterpret_cast<const __half2 *>(&s2));
                            hv[e] = *reinterpret_cast<uint32_t *>(&x);
                        }
                    }
                }
                if (key0 + row >= ctx) {   // never-written slot: may hold NaN codes
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        hv[e] = 0u;
                }
                uint8_t *dst = kv + isv * 16384 + (cc >> 2) * 8192;
                *reinterpret_cast<uint4 *>(dst + swz(row, (2 * cc) & 7)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<uint4 *>(dst + swz(row, (2 * cc + 1) & 7)) =
                    make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
            if constexpr (KVT == kKvInt8) {
                // per-key score factor: softmax scale * log2(e) * K scale
                float *ksf = reinterpret_cast<float *>(smem + kOffKsf) + bj * 64;
                ksf[row] =
                    key0 + row < ctx ? kfac * __half2float(__ushort_as_half(scl[row])) : 0.0f;
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.code_empty[s]);
                mbar_arrive(&bars.kv_full[bj]);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ softmax --
        const int x = (warp - 4) >> 2;       // query tile of this group
        const int r = tid - 128 - 128 * x;   // row == TMEM lane
        const int sw = warp & 3;             // lane quadrant of this warp
        const uint32_t tl = tmem + ((uint32_t)(32 * sw) << 16) + x * 256;
        const QTile T = qt[x];
        const int tq = T.q0 + r / G, gq = r % G;
        const bool valid = r < p.tokens_per_tile * G && tq < q_len;   // rows that exist
        const int pos = ctx - q_len + tq;
        const size_t qrow = (size_t)(q_start + tq) * p.num_q_heads + (size_t)h * G + gq;

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
        // keys lo..pos are visible to this row
        const int lo = p.window > 0 ? pos - p.window + 1 : INT_MIN;
        const int lo_hi = p.window > 0 ? T.pos_hi - p.window + 1 : INT_MIN;
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < T.ntiles; ++j) {
            // S(j) complete also means P V of tile j-1 has completed (in-order MMAs)
            if (!warp_wait(&bars.s_full[x], j & 1, p.status)) {
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
                tmem_ld64(tl + kTmS, ua, ub);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    v[c] = __uint_as_float(ua[c]);
                    v[32 + c] = __uint_as_float(ub[c]);
                }
            }

            const int key0 = (jbase + j) * kKT;
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
            // a key may lie past a row's position or below its window
            if (key0 + kKT - 1 > T.pos_lo || key0 < lo_hi) {
#pragma unroll
                for (int c = 0; c < kKT; ++c)
                    if (key0 + c > pos || key0 + c < lo)
                        v[c] = -INFINITY;
            }
            // row max: eight independent chains, then a tree
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
            // P row over the first 32 S columns (the A operand of P V)
            tmem_st32(tl + kTmS, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars.p_full[x]);
        }

        // ---- epilogue: O / l -> fp16 ----
        float vfac = 1.0f;
        if constexpr (kv_has_head_scale(KVT))
            vfac = __ldg(p.v_scale + h * p.scale_stride);
        const bool have_o = ok && T.ntiles > 0 &&
                            warp_wait(&bars.pv_done[x], (T.ntiles - 1) & 1, p.status);
        if (have_o)
            tc_fence_after();
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
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int KVT, int BS>
cudaError_t launch_tc(const PrefillParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                      cudaStream_t stream)
{
    auto kern = prefill_tc_kernel<KVT, BS>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess)
        return e;
    dim3 grid((p.q_tiles + 1) / 2, p.num_kv_heads, p.batch);
    kern<<<grid, kThreads, kSmemAlloc, stream>>>(kmap, vmap, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillParams &p, int kv_dtype, const CUtensorMap &kmap,
                              const CUtensorMap &vmap, cudaStream_t stream)
{
    if (p.q_tiles == 0 || p.batch == 0)
        return cudaSuccess;
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
