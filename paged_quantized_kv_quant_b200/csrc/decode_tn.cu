// Decode / draft-verify attention for 17..64 query rows per KV head on the
// 5th-generation tensor cores, with the KEYS on the MMA's M dimension
// (tcgen05, accumulators in tensor memory), split-KV.
//
// Source: "1Cat-LLM" README, "Layer 2" (GQA multi-head packing into wider
// tensor-core work, online softmax with FP32 state, Split-KV with an FP32
// merge, MTP verify of several query tokens) and "Layer 1" (paged KV read
// once and wide); "ReVolta" PyPI page ("Weight and KV formats": 8-bit KV
// converted to FP16 for compute; MTP4: 1 + 4 verify positions).
//
// A verify step has q_len x G rows per KV head (5 x 8 = 40): too few for a
// 128-row query tile, where 88 of 128 lanes would run the softmax for
// nothing.  This kernel transposes both products so that the 128-wide M
// dimension holds keys and the query rows are the (padded) N = 64:
//   S^T[key][row]  = K^[key][:] . Q[row][:]        M 128 keys, N 64, K 128 d
//   O^T[d][row]   += V^[:][d]^T P^T[key][row]       M 128 d,    N 64, K 128 keys
// K^ is the K-major A operand and V^ (the same [d half][key][64 d] tiles) the
// MN-major A operand; Q and P^T are B operands in shared memory.  Thread j of
// the softmax owns key j of the tile (TMEM lane j) and every row: its scores
// arrive in one tcgen05.ld, and its per-key INT8 K scale is one scalar.
//
// Softmax.  Rows keep a reference maximum m (log2 units, FP32) shared by all
// keys; P = 2^(s - m) in fp16 and per-thread partial sums l in FP32.  m only
// changes when some score of some row exceeds it by more than 2^8: the four
// softmax warps take a CTA-wide vote each tile (bar.red.or), and only then
// reduce the tile's row maxima across keys, rescale l and O^T (in tensor
// memory) and move m.  The first tile always does so.  P stays <= 2^8, and
// the final O / l uses the same m for both.  The scores are read from tensor
// memory twice per tile (for the vote, then for P), which costs less than
// keeping them in registers.
//
// Warp roles (16 warps):
//   warps 0-3    softmax: warp w reads TMEM lanes 32 w .. 32 w + 31 (its
//                keys) and every row, in two chunks of columns (fewer
//                registers live).  They also stage Q, run the epilogue
//                (thread = output element d of O^T) and write the final rows
//                or the split's FP32 partial.
//   warps 4-9    dequant: code tiles (64 keys) -> fp16 K^/V^ in the
//                128-byte-swizzled layout, one key row per thread: warps 4-5
//                K d 0-63, 8-9 K d 64-127, 6-7 all of V; rows past the
//                context or the split are written as zeros.  (Twelve warps
//                keep three per scheduler, so every thread has 168
//                registers.)
//   warp 10      TMA producer: one 2-D box per cache block into a 3-stage
//                ring of 64-key code stages (FP16 caches: straight into the
//                K^/V^ buffer).
//   warp 11      TMEM allocation and the MMA issue loop (one elected lane
//                issues each tcgen05 instruction).
//
// INT8 V scales.  Each per-token V scale s (fp16) is split as s = f * 2^e
// with f in [1, 2): the dequant warps produce V^ = code * 2^e, which is exact
// in fp16 and costs one fused multiply-add per two codes in the magic-number
// conversion ((1152 + code) * 2^e - 1152 * 2^e, every term exact), and the
// softmax thread that owns the key multiplies its P row by f (P f <= 2^9, and
// no smaller than P, so no new underflow).  Scales with e > 8 (|x| above
// 2^15) keep V^ = fp16(code * s) and f = 1, so V^ cannot overflow; subnormal
// scales use e = -14 and f < 1.
// Epilogue: the final fp16 rows when one split covers the sequence,
// otherwise an FP32 partial (unnormalised O, max in log2 units, sum) in the
// decode workspace, combined by the decode merge kernel.
#include "common.cuh"
#include "internal.h"
#include "split_map.cuh"
#include "tc.cuh"

#include <climits>
#include <math.h>

namespace pkvq {
namespace {

constexpr int kThreads = 384;
constexpr int kKT = 128;             // keys per tile (the M of both products)
constexpr int kHT = 64;              // keys per code stage (half a tile)
constexpr int kN = 64;               // query rows, padded (the N of both products)
constexpr int kCodeStages = 3;
constexpr int kKVBufs = 2;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleLog2 = 8.0f;   // move m only when a score exceeds it by > 2^8
constexpr int kSoftmaxWarps = 4;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kDequantWarp0 = 4;
constexpr int kDequantWarps = 6;
constexpr int kWarpTma = 10;
constexpr int kWarpMma = 11;
constexpr int kBarSoftmax = 1;         // named barrier of the softmax warps

// tensor memory: S^T buffers 0 and 1, O^T, and the softmax threads' per-row
// partial sums (one TMEM lane per key)
constexpr uint32_t kTmS = 0, kTmO = 2 * kN, kTmL = 3 * kN;
constexpr uint32_t kTmCols = 256;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr int kKVBuf = 65536;                                   // K^ 32K then V^ 32K
constexpr int kKVHalf = 16384;                                  // one d half of K^ or V^
constexpr int kOffKV = 0;
constexpr int kOffCodes = kOffKV + kKVBufs * kKVBuf;            // stages x (K 8K, V 8K)
constexpr int kCodeStage = 16384;
constexpr int kOffScl = kOffCodes + kCodeStages * kCodeStage;   // stages x (K 64, V 64) halves
constexpr int kOffKsf = kOffScl + kCodeStages * 256;            // bufs x 128 fp32 K factors
constexpr int kOffVsf = kOffKsf + kKVBufs * kKT * 4;            // bufs x 128 fp32 V mantissas
constexpr int kOffP = (kOffVsf + kKVBufs * kKT * 4 + 1023) / 1024 * 1024;   // P^T [128][64]
constexpr int kOffQ = kOffP + kKT * 128;                        // Q [d half][64 rows][64 d]
constexpr int kOffRed = kOffQ + 2 * kN * 128;                   // [4][64] fp32 exchange
constexpr int kOffPos = kOffRed + 4 * kN * 4;                   // pos[64], lo[64], corr[64]
constexpr int kOffM = kOffPos + 3 * kN * 4;                     // row references [2][64]
constexpr int kOffBars = kOffM + 2 * kN * 4;
constexpr int kNumBars = 1 + 2 * kCodeStages + 3 * kKVBufs + 2 + 1 + 1 + 1;
constexpr int kOffTaddr = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = kOffTaddr + 16;
constexpr size_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

constexpr uint32_t kIdescS = idesc_f16_f32(kKT, kN, false, false);
constexpr uint32_t kIdescO = idesc_f16_f32(128, kN, true, true);

struct Bars {
    uint64_t *q_full;
    uint64_t *code_full, *code_empty;   // [kCodeStages]
    uint64_t *kv_full, *kv_empty;       // [kKVBufs]
    uint64_t *kv_tma;                   // [kKVBufs] FP16: the buffer's copies landed
    uint64_t *s_full;                   // [2]
    uint64_t *p_full, *pv_done, *mma_done;
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
    r.kv_tma = r.kv_empty + kKVBufs;
    r.s_full = r.kv_tma + kKVBufs;
    r.p_full = r.s_full + 2;
    r.pv_done = r.p_full + 1;
    r.mma_done = r.pv_done + 1;
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

// True on every softmax thread if `pred` holds on any of them.
__device__ __forceinline__ bool softmax_any(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(kBarSoftmax), "n"(kSoftmaxThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void softmax_sync()
{
    asm volatile("bar.sync %0, %1;" ::"n"(kBarSoftmax), "n"(kSoftmaxThreads) : "memory");
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

// N columns (rows of the query) of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void ld_rows(uint32_t taddr, uint32_t (&r)[N])
{
    if constexpr (N == 16)
        tmem_ld16(taddr, r);
    else if constexpr (N == 24)
        tmem_ld24(taddr, r);
    else
        tmem_ld32(taddr, r);
}

template <int KVT, int BS, int NR>
__global__ void __launch_bounds__(kThreads, 1)
decode_tn_kernel(const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const DecodeParams p)
{
    constexpr int kBPH = kHT / BS;     // cache blocks per code stage
    constexpr int kBPT = kKT / BS;     // cache blocks per tile
    static_assert(NR % 16 == 0 && NR <= kN, "row split");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Bars bars = carve_bars(smem);
    uint32_t *taddr_smem = reinterpret_cast<uint32_t *>(smem + kOffTaddr);
    float *red = reinterpret_cast<float *>(smem + kOffRed);     // [4][kN]
    int *pos_row = reinterpret_cast<int *>(smem + kOffPos);     // [kN]
    int *lo_row = pos_row + kN;                                 // [kN]
    float *corr_row = reinterpret_cast<float *>(lo_row + kN);   // [kN]

    const int slot = blockIdx.x;
    const int h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
        mbar_init(bars.q_full, kSoftmaxWarps);
        for (int s = 0; s < kCodeStages; ++s) {
            mbar_init(&bars.code_full[s], 1);
            mbar_init(&bars.code_empty[s], kDequantWarps);
        }
        for (int i = 0; i < kKVBufs; ++i) {
            mbar_init(&bars.kv_full[i], 2 * kDequantWarps);   // two code stages per tile
            mbar_init(&bars.kv_empty[i], 1);
            mbar_init(&bars.kv_tma[i], 1);
        }
        for (int i = 0; i < 2; ++i)
            mbar_init(&bars.s_full[i], 1);
        mbar_init(bars.p_full, kSoftmaxWarps);
        mbar_init(bars.pv_done, 1);
        mbar_init(bars.mma_done, 1);
        fence_mbar_init();
    }
    // Inputs may come from the previous kernel: wait for it to complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

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
    const int nhalf = (nblk + kBPH - 1) / kBPH;          // 64-key code stages
    const int ntiles = (nhalf + 1) / 2;                  // 128-key tiles
    const int key_begin = blk_begin * BS;
    const int key_lim = key_begin + nblk * BS;           // first key past the split
    const int G = p.group;

    if (warp == kWarpMma) {
        tmem_alloc(taddr_smem, kTmCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_smem;

    if (warp == kWarpTma) {
        // ------------------------------------------------ TMA producer --
        const int32_t *bt = p.block_table + (size_t)b * p.max_blocks_per_seq + blk_begin;
        // every index stays inside the table row, even for a context longer
        // than the row can address (a caller error: those keys read block 0)
        const int nwin = min(nblk, p.max_blocks_per_seq - blk_begin);
        int win0 = lane < nwin ? __ldg(bt + lane) : 0;
        int win1 = 32 + lane < nwin ? __ldg(bt + 32 + lane) : 0;
        int wbase = 0;
        auto block_id = [&](int bi) {   // warp-uniform call; bi within [wbase, wbase + 64)
            const int a = __shfl_sync(0xffffffffu, win0, bi & 31);
            const int c = __shfl_sync(0xffffffffu, win1, bi & 31);
            int phys = (bi - wbase) < 32 ? a : c;
#ifdef PKVQ_BOUNDS_CHECK
            if (phys < 0 || phys >= p.num_blocks) {
                if (lane == 0)
                    atomicOr(p.status, kStatusBadBlock);
                phys = 0;
            }
#endif
            return phys;
        };
        auto slide = [&](int next_blk) {   // keep the window ahead of next_blk
            while (next_blk >= wbase + 32) {
                wbase += 32;
                win0 = win1;
                win1 = wbase + 32 + lane < nwin ? __ldg(bt + wbase + 32 + lane) : 0;
            }
        };
        if constexpr (KVT == kKvFp16) {
            // a whole tile straight into K/V buffer t % 2
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int bj = t % kKVBufs;
                if (t >= kKVBufs &&
                    !warp_wait(&bars.kv_empty[bj], ((t - kKVBufs) / kKVBufs) & 1, p.status))
                    break;
                issued = t + 1;
                const int blk0 = t * kBPT;
                const int nb = min(kBPT, nblk - blk0);
                if (lane == 0)
                    mbar_arrive_expect_tx(&bars.kv_tma[bj], (uint32_t)nb * BS * 256 * 2);
                uint8_t *kv = smem + kOffKV + bj * kKVBuf;
                for (int i = 0; i < nb; ++i) {
                    const int phys = block_id(blk0 + i);
                    if (lane == 0) {
                        const int y = (phys * p.num_kv_heads + h) * BS;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            tma_tile_2d_g2s(kv + half * kKVHalf + i * BS * 128, &kmap, 128 * half,
                                            y, &bars.kv_tma[bj]);
                            tma_tile_2d_g2s(kv + 32768 + half * kKVHalf + i * BS * 128, &vmap,
                                            128 * half, y, &bars.kv_tma[bj]);
                        }
                    }
                    if (i + 1 < nb || t + 1 < ntiles)
                        slide(blk0 + i + 1);
                }
            }
            if (lane == 0)
                for (int t = max(0, issued - kKVBufs); t < issued; ++t)
                    mbar_wait(&bars.kv_tma[t % kKVBufs], (t / kKVBufs) & 1, nullptr);
        } else {
            // 64-key code stages; an odd last tile gets an empty stage
            int issued = 0;
            for (int u = 0; u < 2 * ntiles; ++u) {
                const int s = u % kCodeStages;
                if (u >= kCodeStages &&
                    !warp_wait(&bars.code_empty[s], ((u - kCodeStages) / kCodeStages) & 1,
                               p.status))
                    break;
                issued = u + 1;
                const int blk0 = u * kBPH;
                const int nb = max(0, min(kBPH, nblk - blk0));
                if (lane == 0) {
                    uint32_t tx = (uint32_t)nb * BS * 128 * 2;
                    if constexpr (KVT == kKvInt8)
                        tx += (uint32_t)nb * BS * 2 * 2;
                    mbar_arrive_expect_tx(&bars.code_full[s], tx);
                }
                uint8_t *dst = smem + kOffCodes + s * kCodeStage;
                uint16_t *sd = reinterpret_cast<uint16_t *>(smem + kOffScl + s * 256);
                for (int i = 0; i < nb; ++i) {
                    const int phys = block_id(blk0 + i);
                    if (lane == 0) {
                        const int y = (phys * p.num_kv_heads + h) * BS;
                        tma_tile_2d_g2s(dst + i * BS * 128, &kmap, 0, y, &bars.code_full[s]);
                        tma_tile_2d_g2s(dst + 8192 + i * BS * 128, &vmap, 0, y,
                                        &bars.code_full[s]);
                        if constexpr (KVT == kKvInt8) {
                            tma_bulk_g2s(sd + i * BS, p.k_scale_tok + (size_t)y, BS * 2,
                                         &bars.code_full[s]);
                            tma_bulk_g2s(sd + 64 + i * BS, p.v_scale_tok + (size_t)y, BS * 2,
                                         &bars.code_full[s]);
                        }
                    }
                    slide(blk0 + i + 1);
                }
            }
            // copies this CTA issued must land before it exits (bounded wait)
            if (lane == 0)
                for (int u = max(0, issued - kCodeStages); u < issued; ++u)
                    mbar_wait(&bars.code_full[u % kCodeStages], (u / kCodeStages) & 1, nullptr);
        }
    } else if (warp == kWarpMma) {
        // --------------------------------------------------- MMA issuer --
        // S(t) reuses the TMEM columns of S(t-2): it is issued once the
        // softmax has read S(t-2) (its P is complete) and K^(t) is ready.
        // O^T += V^(t)^T P(t)^T is issued once P(t) is in shared memory.
        if (ntiles > 0) {
            bool ok = warp_wait(bars.q_full, 0, p.status);
            tc_fence_after();
            const uint64_t qd0 = desc_sw128(sbase + kOffQ, 16, 1024);
            const uint64_t pd0 = desc_sw128(sbase + kOffP, 8192, 1024);
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
                    const uint32_t kb = sbase + kOffKV + (nqk % kKVBufs) * kKVBuf;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (ks >> 2) * kKVHalf + (ks & 3) * 32;
                        const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                        mma_f16_ss_elect(tmem + kTmS + (nqk & 1) * kN,
                                         desc_sw128(kb + off, 16, 1024),
                                         qd0 + (uint64_t)(qoff >> 4), kIdescS, ks > 0 ? 1u : 0u);
                    }
                    mma_commit_elect(&bars.s_full[nqk & 1]);
                    ++nqk;
                    progressed = true;
                }
                if (nxt < nqk) {
                    const bool rdy = progressed
                                         ? mbar_test_wait(bars.p_full, nxt & 1)
                                         : mbar_try_wait_for(bars.p_full, nxt & 1, kPollSleepNs);
                    if (__any_sync(0xffffffffu, rdy)) {
                        tc_fence_after();
                        const uint32_t vb = sbase + kOffKV + (nxt % kKVBufs) * kKVBuf + 32768;
                        const uint64_t vd0 = desc_sw128(vb, kKVHalf, 1024);
#pragma unroll
                        for (int ks = 0; ks < kKT / 16; ++ks)
                            mma_f16_ss_elect(tmem + kTmO, vd0 + (uint64_t)((ks * 2048) >> 4),
                                             pd0 + (uint64_t)((ks * 2048) >> 4), kIdescO,
                                             (nxt > 0 || ks > 0) ? 1u : 0u);
                        mma_commit_elect(bars.pv_done);
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
    } else if (warp >= kDequantWarp0 && warp < kDequantWarp0 + kDequantWarps) {
        // ------------------------------------------------------ dequant --
        const int dw = warp - kDequantWarp0;
        const int row = (dw & 1) * 32 + lane;     // key row of this thread in a code stage
        const int isv = (dw == 2 || dw == 3) ? 1 : 0;   // K: dw 0, 1, 4, 5; V: dw 2, 3
        const int c0 = dw >= 4 ? 4 : 0;           // first 16-byte code chunk of the row
        const int nch = isv ? 8 : 4;              // chunks this thread converts
        const float kfac = p.scale_log2;
        for (int u = 0; u < 2 * ntiles; ++u) {
            const int t = u >> 1, hk = u & 1, bj = t % kKVBufs;
            const int krow = hk * kHT + row;      // key row within the tile
            const int key = key_begin + t * kKT + krow;
            const bool live = key < ctx && key < key_lim;
            uint8_t *kv = smem + kOffKV + bj * kKVBuf + isv * 32768;
            if constexpr (KVT == kKvFp16) {
                if (hk == 0 && !warp_wait(&bars.kv_tma[bj], (t / kKVBufs) & 1, p.status))
                    break;
                if (!live) {   // the row's d halves this warp owns (K: one, V: both)
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!isv && hh != (c0 >> 2))
                            continue;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4 *>(kv + hh * kKVHalf + krow * 128 + c * 16) = z;
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars.kv_full[bj]);
                continue;
            }
            const int s = u % kCodeStages;
            if (!warp_wait(&bars.code_full[s], (u / kCodeStages) & 1, p.status))
                break;
            if (hk == 0 && t >= kKVBufs &&
                !warp_wait(&bars.kv_empty[bj], ((t - kKVBufs) / kKVBufs) & 1, p.status))
                break;
            const uint8_t *codes = smem + kOffCodes + s * kCodeStage + isv * 8192;
            const uint16_t *scl = reinterpret_cast<const uint16_t *>(smem + kOffScl + s * 256);
            // INT8 V: V^ = code * 2^e by one fma of the magic-number form,
            // unless the scale is too large (then code * s in fp16)
            __half2 p2 = __half2half2(__ushort_as_half(0x3C00)), nb2 = p2;
            bool big = false;
            uint32_t s2 = 0u;
            if constexpr (KVT == kKvInt8) {
                if (isv) {
                    const uint32_t sb = scl[64 + row];   // V scale of this key
                    const uint32_t ef = (sb >> 10) & 31u;
                    big = ef > 15u + 8u;
                    const uint16_t pw = ef == 0 ? 0x0400 : (uint16_t)(sb & 0x7C00u);
                    p2 = __half2half2(__ushort_as_half(pw));
                    nb2 = __hmul2(p2, __half2half2(__ushort_as_half(0xE480)));   // -1152 * 2^e
                    s2 = sb | (sb << 16);
                }
            }
            // all code chunks of the row are loaded before any is converted
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < nch)
                    wv[i] = *reinterpret_cast<const uint4 *>(codes + swz(row, c0 + i));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i >= nch)
                    break;
                const int cc = c0 + i;   // 16-byte code chunk: d 16cc .. 16cc+15
                const uint4 w = wv[i];
                uint32_t hv[8];
                if constexpr (KVT == kKvInt8) {
                    if (isv && !big) {
                        s8x4_to_half2x2_scaled(w.x, p2, nb2, hv[0], hv[1]);
                        s8x4_to_half2x2_scaled(w.y, p2, nb2, hv[2], hv[3]);
                        s8x4_to_half2x2_scaled(w.z, p2, nb2, hv[4], hv[5]);
                        s8x4_to_half2x2_scaled(w.w, p2, nb2, hv[6], hv[7]);
                    } else {
                        cvt4<KVT>(w.x, hv[0], hv[1]);
                        cvt4<KVT>(w.y, hv[2], hv[3]);
                        cvt4<KVT>(w.z, hv[4], hv[5]);
                        cvt4<KVT>(w.w, hv[6], hv[7]);
                        if (isv) {   // scales of 2^8 and above: code * s in fp16
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                __half2 x = __hmul2(*reinterpret_cast<__half2 *>(&hv[e]),
                                                    *reinterpret_cast<const __half2 *>(&s2));
                                hv[e] = *reinterpret_cast<uint32_t *>(&x);
                            }
                        }
                    }
                } else {
                    cvt4<KVT>(w.x, hv[0], hv[1]);
                    cvt4<KVT>(w.y, hv[2], hv[3]);
                    cvt4<KVT>(w.z, hv[4], hv[5]);
                    cvt4<KVT>(w.w, hv[6], hv[7]);
                }
                if (!live) {   // past the context or the split: codes may be anything
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        hv[e] = 0u;
                }
                uint8_t *dst = kv + (cc >> 2) * kKVHalf;
                *reinterpret_cast<uint4 *>(dst + swz(krow, (2 * cc) & 7)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<uint4 *>(dst + swz(krow, (2 * cc + 1) & 7)) =
                    make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
            if constexpr (KVT == kKvInt8) {
                if (!isv && c0 == 0) {   // per-key score factor: softmax scale * log2(e) * K scale
                    float *ksf = reinterpret_cast<float *>(smem + kOffKsf) + bj * kKT;
                    ksf[krow] = live ? kfac * __half2float(__ushort_as_half(scl[row])) : 0.0f;
                }
                if (isv) {   // the mantissa of the V scale, applied to P
                    const uint32_t sb = scl[64 + row];
                    const uint32_t ef = (sb >> 10) & 31u;
                    float f = 1.0f;
                    if (ef == 0)
                        f = __half2float(__ushort_as_half((uint16_t)sb)) * 16384.0f;
                    else if (ef <= 15u + 8u)
                        f = __half2float(__ushort_as_half((uint16_t)(0x3C00u | (sb & 0x3FFu))));
                    float *vsf = reinterpret_cast<float *>(smem + kOffVsf) + bj * kKT;
                    vsf[krow] = live ? f : 0.0f;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.code_empty[s]);
                mbar_arrive(&bars.kv_full[bj]);
            }
        }
    } else if (warp < kSoftmaxWarps) {
        // ------------------------------------------------------ softmax --
        constexpr int NRC = NR == 48 ? 24 : 16;    // rows per column chunk
        const int quad = warp;                     // TMEM lane quadrant
        const int key_in_tile = 32 * quad + lane;  // TMEM lane of this thread
        const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);
        // row references (log2 units) in shared memory, double-buffered: all
        // threads read the same values (broadcast)
        float *m_arr = reinterpret_cast<float *>(smem + kOffM);   // [2][kN]
        int sel = 0;

        // Q rows -> shared memory (K-major B operand), zeros for padding rows;
        // each row's visible key range; P^T columns no thread writes stay 0
        for (int c = tid; c < kN * 16; c += kSoftmaxThreads) {
            const int r = c >> 4, dc = c & 15;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < p.rows) {
                const int tq = r / G, gq = r % G;
                const size_t qrow =
                    ((size_t)b * p.q_len + tq) * p.num_q_heads + (size_t)h * G + gq;
                v = __ldg(reinterpret_cast<const uint4 *>(p.q + qrow * kHeadDim) + dc);
            }
            *reinterpret_cast<uint4 *>(smem + kOffQ + (dc >> 3) * 8192 + swz(r, dc & 7)) = v;
        }
        for (int c = tid; c < kKT * 8; c += kSoftmaxThreads)
            *reinterpret_cast<uint4 *>(smem + kOffP + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        if (tid < kN) {
            const int r = tid;
            const bool valid = r < p.rows;
            const int ps = valid ? min(ctx - 1, query_position(p, b, ctx, r / G)) : ctx - 1;
            pos_row[r] = ps;
            lo_row[r] = p.window > 0 && valid ? ps - p.window + 1 : INT_MIN;
            m_arr[r] = -INFINITY;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars.q_full);
        softmax_sync();
        // a tile needs masking when it reaches past the lowest position, past
        // the split, or starts below the highest window start
        int pos_lo = ctx - 1, lo_hi = INT_MIN;
        for (int r = 0; r < p.rows && r < kN; ++r) {
            pos_lo = min(pos_lo, pos_row[r]);
            lo_hi = max(lo_hi, lo_row[r]);
        }

        float kfac_head = p.scale_log2;
        if constexpr (kv_has_head_scale(KVT))
            kfac_head *= __ldg(p.k_scale + h * p.scale_stride);
        // per-row partial sums of this key's lane live in tensor memory
        {
            uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
            for (int c = 0; c < NR; c += 8)
                tmem_st8(tl + kTmL + c, z);
            tmem_st_wait();
        }
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            if (!warp_wait(&bars.s_full[t & 1], (t >> 1) & 1, p.status))
                ok = false;
            if constexpr (KVT == kKvInt8) {
                // the per-key factors were written by the dequant warps
                if (ok && !warp_wait(&bars.kv_full[t % kKVBufs], (t / kKVBufs) & 1, p.status))
                    ok = false;
            }
            // every softmax thread takes the same barrier steps, even after a
            // failed wait (the votes below would otherwise never complete)
            tc_fence_after();
            float kfac = kfac_head, vf = 1.0f;
            if constexpr (KVT == kKvInt8) {
                kfac = reinterpret_cast<const float *>(smem + kOffKsf)[(t % kKVBufs) * kKT +
                                                                      key_in_tile];
                vf = reinterpret_cast<const float *>(smem + kOffVsf)[(t % kKVBufs) * kKT +
                                                                    key_in_tile];
            }
            const int key0 = key_begin + t * kKT;
            const int key = key0 + key_in_tile;
            const bool masked = key0 + kKT - 1 > pos_lo || key0 + kKT > key_lim || key0 < lo_hi;
            const uint32_t scol = tl + kTmS + (t & 1) * kN;
            // this thread's scores of rows c0 .. c0 + NRC - 1, scaled and masked
            auto scores = [&](int c0, float (&sv)[NRC]) {
                uint32_t u[NRC];
                if (ok)
                    ld_rows<NRC>(scol + c0, u);
#pragma unroll
                for (int i = 0; i < NRC; ++i)
                    sv[i] = ok ? __uint_as_float(u[i]) * kfac : -INFINITY;
                if (masked) {
#pragma unroll
                    for (int i = 0; i < NRC; ++i)
                        if (key > pos_row[c0 + i] || key >= key_lim || key < lo_row[c0 + i])
                            sv[i] = -INFINITY;
                }
            };
            bool exceeds = false;
#pragma unroll
            for (int c0 = 0; c0 < NR; c0 += NRC) {
                float sv[NRC];
                scores(c0, sv);
                const float *mc = m_arr + sel * kN + c0;
#pragma unroll
                for (int i = 0; i < NRC; i += 4) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(mc + i);
                    exceeds |= sv[i] > m4.x + kRescaleLog2;
                    exceeds |= sv[i + 1] > m4.y + kRescaleLog2;
                    exceeds |= sv[i + 2] > m4.z + kRescaleLog2;
                    exceeds |= sv[i + 3] > m4.w + kRescaleLog2;
                }
            }
            if (softmax_any(exceeds || !ok)) {
                if (softmax_any(!ok)) {
                    ok = false;
                } else {
                    // move every row's reference to the running maximum:
                    // tile maxima across keys (lanes, then quadrants)
#pragma unroll
                    for (int c0 = 0; c0 < NR; c0 += NRC) {
                        float sv[NRC];
                        scores(c0, sv);
#pragma unroll
                        for (int i = 0; i < NRC; ++i) {
                            float mx = sv[i];
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1)
                                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                            if (lane == 0)
                                red[quad * kN + c0 + i] = mx;
                        }
                    }
                    softmax_sync();
                    // every thread computes the same new references; one
                    // writes them and the rows' factors
                    const float *mc = m_arr + sel * kN;
                    float *mn_arr = m_arr + (sel ^ 1) * kN;
                    bool moved = false;
#pragma unroll 1
                    for (int i = 0; i < NR; ++i) {
                        const float mt = fmaxf(fmaxf(red[i], red[kN + i]),
                                               fmaxf(red[2 * kN + i], red[3 * kN + i]));
                        const float mo = mc[i];
                        const float mn = fmaxf(mo, mt);
                        const float corr = mn == -INFINITY ? 1.0f : fast_exp2(mo - mn);
                        moved |= corr != 1.0f;
                        if (tid == 0) {
                            mn_arr[i] = mn;
                            corr_row[i] = corr;
                        }
                    }
                    softmax_sync();   // red read by all; new references written
                    sel ^= 1;
                    // partial sums shrink with their references
                    if (ok && moved) {
#pragma unroll
                        for (int c = 0; c < NR; c += 8) {
                            uint32_t lv[8];
                            tmem_ld8(tl + kTmL + c, lv);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                lv[i] = __float_as_uint(__uint_as_float(lv[i]) * corr_row[c + i]);
                            tmem_st8(tl + kTmL + c, lv);
                        }
                        tmem_st_wait();
                    }
                    // O^T columns (lane = d), 8 at a time, once every P V
                    // issued so far has completed
                    if (t > 0 && moved) {
                        if (!warp_wait(bars.pv_done, (t - 1) & 1, p.status))
                            ok = false;
                        tc_fence_after();
                        if (ok) {
#pragma unroll
                            for (int c = 0; c < NR; c += 8) {
                                uint32_t o[8];
                                tmem_ld8(tl + kTmO + c, o);
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    o[i] = __float_as_uint(__uint_as_float(o[i]) *
                                                           corr_row[c + i]);
                                tmem_st8(tl + kTmO + c, o);
                            }
                            tmem_st_wait();
                        }
                    }
                }
            }
            // P^T row of this key, fp16 2^(s - m) (times the INT8 V scale's
            // mantissa); P^T is single-buffered, so P V of the previous tile
            // must be done before the first store
            uint8_t *prow = smem + kOffP + key_in_tile * 128;
#pragma unroll
            for (int c0 = 0; c0 < NR; c0 += NRC) {
                float sv[NRC];
                scores(c0, sv);
                const float *mu = m_arr + sel * kN + c0;
                uint32_t lv[NRC];
                if (ok)
                    ld_rows<NRC>(tl + kTmL + c0, lv);
                uint32_t pk[NRC / 2];
#pragma unroll
                for (int i = 0; i < NRC; i += 4) {
                    float4 m4 = *reinterpret_cast<const float4 *>(mu + i);
                    m4.x = m4.x == -INFINITY ? 0.0f : m4.x;
                    m4.y = m4.y == -INFINITY ? 0.0f : m4.y;
                    m4.z = m4.z == -INFINITY ? 0.0f : m4.z;
                    m4.w = m4.w == -INFINITY ? 0.0f : m4.w;
                    const float e0 = fast_exp2(sv[i] - m4.x), e1 = fast_exp2(sv[i + 1] - m4.y);
                    const float e2 = fast_exp2(sv[i + 2] - m4.z), e3 = fast_exp2(sv[i + 3] - m4.w);
                    lv[i] = __float_as_uint(__uint_as_float(lv[i]) + e0);
                    lv[i + 1] = __float_as_uint(__uint_as_float(lv[i + 1]) + e1);
                    lv[i + 2] = __float_as_uint(__uint_as_float(lv[i + 2]) + e2);
                    lv[i + 3] = __float_as_uint(__uint_as_float(lv[i + 3]) + e3);
                    pk[i / 2] = pack_half2(e0 * vf, e1 * vf);
                    pk[i / 2 + 1] = pack_half2(e2 * vf, e3 * vf);
                }
                if (ok) {
#pragma unroll
                    for (int c = 0; c < NRC; c += 8)
                        tmem_st8(tl + kTmL + c0 + c, lv + c);
                }
                if (c0 == 0 && t > 0 && !warp_wait(bars.pv_done, (t - 1) & 1, p.status))
                    ok = false;
#pragma unroll
                for (int c = 0; c < NRC / 8; ++c) {
                    const int chunk = c0 / 8 + c;   // 8 rows of this key
                    *reinterpret_cast<uint4 *>(prow + ((chunk ^ (key_in_tile & 7)) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.p_full);
        }

        // ---- epilogue: row sums across keys, then O^T / l ----
#pragma unroll
        for (int c = 0; c < NR; c += 8) {
            uint32_t lv[8];
            tmem_ld8(tl + kTmL + c, lv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float s = __uint_as_float(lv[i]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0)
                    red[quad * kN + c + i] = s;
            }
        }
        softmax_sync();
        const float *mfin = m_arr + sel * kN;
        const int jl = ntiles - 1;
        const bool have_o = ok && ntiles > 0 && warp_wait(bars.pv_done, jl & 1, p.status);
        if (have_o)
            tc_fence_after();
        const int d = key_in_tile;   // TMEM lane of O^T = output element d
        float vfac = 1.0f;
        if constexpr (kv_has_head_scale(KVT))
            vfac = __ldg(p.v_scale + h * p.scale_stride);
#pragma unroll 1
        for (int c = 0; c < NR; c += 8) {
            uint32_t o[8];
            if (have_o)   // warp-uniform
                tmem_ld8(tl + kTmO + c, o);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = c + i;
                if (r >= p.rows)
                    break;
                const float lsum =
                    red[r] + red[kN + r] + red[2 * kN + r] + red[3 * kN + r];
                const float mrow = mfin[r];
                if (si.nsplit == 1) {
                    const int tq = r / G, gq = r % G;
                    const size_t qrow =
                        ((size_t)b * p.q_len + tq) * p.num_q_heads + (size_t)h * G + gq;
                    const bool has = have_o && lsum > 0.0f;
                    const float y = has ? __uint_as_float(o[i]) * (vfac / lsum) : 0.0f;
                    p.out[qrow * kHeadDim + d] = __float2half_rn(y);
                    if (d == 0 && p.lse)
                        p.lse[qrow] = has ? (mrow + log2f(lsum)) * kLn2 : -INFINITY;
                } else {
                    // FP32 partial: unnormalised O, max (log2 units) and sum
                    const size_t wrow = ((size_t)h * p.num_splits + slot) * p.rows_per_cta + r;
                    p.ws_o[wrow * kHeadDim + d] = have_o ? __uint_as_float(o[i]) : 0.0f;
                    if (d == 0)
                        *reinterpret_cast<float2 *>(p.ws_ml + wrow * 2) =
                            have_o ? make_float2(mrow, lsum) : make_float2(-INFINITY, 0.0f);
                }
            }
        }
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmCols);
    }
}

template <int KVT, int BS, int NR>
cudaError_t launch_tn(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                      cudaStream_t stream)
{
    auto kern = decode_tn_kernel<KVT, BS, NR>;
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

template <int KVT, int BS>
cudaError_t launch_tn_rows(const DecodeParams &p, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, cudaStream_t stream)
{
    if (p.rows <= 32)
        return launch_tn<KVT, BS, 32>(p, kmap, vmap, stream);
    if (p.rows <= 48)
        return launch_tn<KVT, BS, 48>(p, kmap, vmap, stream);
    return launch_tn<KVT, BS, 64>(p, kmap, vmap, stream);
}

}  // namespace

cudaError_t launch_decode_tn(const DecodeParams &p, int kv_dtype, const CUtensorMap &kmap,
                             const CUtensorMap &vmap, cudaStream_t stream)
{
    switch (kv_dtype * 100 + p.block_size) {
#define PKVQ_TN_CASE(T, B) \
    case T * 100 + B: return launch_tn_rows<T, B>(p, kmap, vmap, stream);
        PKVQ_TN_CASE(kKvFp8, 16) PKVQ_TN_CASE(kKvFp8, 32) PKVQ_TN_CASE(kKvFp8, 64)
        PKVQ_TN_CASE(kKvInt8, 16) PKVQ_TN_CASE(kKvInt8, 32) PKVQ_TN_CASE(kKvInt8, 64)
        PKVQ_TN_CASE(kKvE5m2, 16) PKVQ_TN_CASE(kKvE5m2, 32) PKVQ_TN_CASE(kKvE5m2, 64)
        PKVQ_TN_CASE(kKvFp16, 16) PKVQ_TN_CASE(kKvFp16, 32) PKVQ_TN_CASE(kKvFp16, 64)
#undef PKVQ_TN_CASE
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
