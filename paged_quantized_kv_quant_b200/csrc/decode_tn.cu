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
// dimension holds keys and the query rows are the (padded) N:
//   S^T[key][row]  = K^[key][:] . Q[row][:]        M 128 keys, N NP, K 128 d
//   O^T[d][row]   += V^[:][d]^T P^T[key][row]       M 128 d,    N NP, K 128 keys
// K^ is the K-major A operand and V^ (the same [d half][key][64 d] tiles) the
// MN-major A operand; Q and P^T are B operands in shared memory.
//
// Pipeline.  What bounds a tile is the chain dequantise -> S -> softmax ->
// P V, so nothing in it waits for more than it needs:
//   * K^ and V^ have separate double buffers.  K^(t+2) is written once the
//     softmax has read S(t) (S(t) complete, its per-key factors consumed);
//     V^(t+2) once P(t) V has completed.
//   * The softmax warps issue P V themselves, right after the last P^T
//     store; the MMA warp only issues Q K^T, so each waits on one barrier.
//   * The copy warp keeps six 64-key stages in flight to L2 ahead of the
//     three-stage shared-memory ring.
//
// Softmax (one pass per tile in the common case).  Thread j of a softmax
// warp owns key j of its quadrant (TMEM lane) and a range of rows; the two
// warps of a quadrant split the rows.  Rows keep a reference maximum m (log2
// units, FP32, finite: -1e30 before any key) shared by all keys; P =
// 2^(s - m) and per-thread partial sums l in FP32 (tensor memory).  m moves only
// when a score exceeds it by more than 2^8: one CTA-wide vote per tile
// (bar.red), and only then the tile's row maxima across keys, a rescale of l
// and O^T (tensor memory) and a recomputation of P.  The first tile always
// does so.  P stays <= 2^8, and O / l uses the same m for both.
//
// Warp roles (16 warps, four per scheduler):
//   warps 0-7    softmax: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its
//                keys) and rows [0, R0) (w < 4) or [R0, NR) (w >= 4).  They
//                also stage Q, run the epilogue (thread = output element d of
//                O^T) and write the final rows or the split's FP32 partial;
//                warp 0 issues P V.
//   warps 8-13   dequant, the same share of code per scheduler: warp 10 K
//                rows 0-31 and warp 11 V rows 0-31 of a 64-key stage (all of
//                d), warps 8 / 12 K rows 32-63 (d 0-63 / 64-127), warps 9 / 13
//                V rows 32-63 (same halves); rows past the context or the
//                split are written as zeros.
//   warp 14      copy producer (cp.async, 32 lanes; see kv_stage.cuh).
//   warp 15      TMEM allocation and the Q K^T issue loop.
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
#include "kv_stage.cuh"
#include "split_map.cuh"
#include "tc.cuh"

#include <climits>
#include <math.h>

namespace pkvq {
namespace {

constexpr int kThreads = 512;
constexpr int kKT = 128;             // keys per tile (the M of both products)
constexpr int kHT = 64;              // keys per code stage (half a tile)
constexpr int kN = 64;               // query rows at most
constexpr int kCodeStages = 3;
// L2 prefetch distance in code stages: with 16-token blocks the farthest
// prefetched block stays within 60 entries of the block-table window's base
constexpr int kPrefetchStages = 6;
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kRescaleLog2 = 8.0f;   // move m only when a score exceeds it by > 2^8
constexpr float kMInit = -1e30f;       // row reference before any visible key
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kDequantWarp0 = 8;
constexpr int kDequantWarps = 6;
constexpr int kWarpCopy = 14;
constexpr int kWarpMma = 15;
constexpr int kBarSoftmax = 1;         // named barrier of the softmax warps

// tensor memory: S^T buffers 0 and 1, O^T, and the softmax threads' per-row
// partial sums (one TMEM lane per key)
constexpr uint32_t kTmS = 0, kTmO = 2 * kN, kTmL = 3 * kN;
constexpr uint32_t kTmCols = 256;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr int kHatBuf = 32768;                                  // [d half][128 keys][64 d]
constexpr int kKVHalf = 16384;
constexpr int kOffK = 0;                                        // K^ buffers 0, 1
constexpr int kOffV = 2 * kHatBuf;                              // V^ buffers 0, 1
constexpr int kOffCodes = 4 * kHatBuf;                          // stages x (K 8K, V 8K)
constexpr int kCodeStage = 16384;
constexpr int kOffScl = kOffCodes + kCodeStages * kCodeStage;   // stages x (K 64, V 64) halves
constexpr int kOffKsf = kOffScl + kCodeStages * 256;            // [2][128] fp32 K factors
constexpr int kOffVsf = kOffKsf + 2 * kKT * 4;                  // [2][128] fp32 V mantissas
constexpr int kOffP = (kOffVsf + 2 * kKT * 4 + 1023) / 1024 * 1024;   // P^T [128][64]
constexpr int kOffQ = kOffP + kKT * 128;                        // Q [d half][64 rows][64 d]
constexpr int kOffRed = kOffQ + 2 * kN * 128;                   // [4][64] fp32 exchange
constexpr int kOffPos = kOffRed + 4 * kN * 4;                   // pos[64], lo[64]
constexpr int kOffM = kOffPos + 2 * kN * 4;                     // row references [2][64]
constexpr int kOffCorr = kOffM + 2 * kN * 4;                   // row rescale factors [64]
constexpr int kOffBars = kOffCorr + kN * 4;
constexpr int kNumBars = 1 + 2 * kCodeStages + 2 * 6 + 3;
constexpr int kOffTaddr = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = kOffTaddr + 16;
constexpr size_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");

struct Bars {
    uint64_t *q_full;
    uint64_t *code_full, *code_empty;   // [kCodeStages]
    uint64_t *kfull, *vfull;            // [2] K^ / V^ buffer written
    uint64_t *vempty;                   // [2] P V of the buffer's tile completed
    uint64_t *kv_tma;                   // [2] FP16: the tile's copies landed
    uint64_t *s_full;                   // [2] S^T buffer computed
    uint64_t *s_free;                   // [2] softmax done with S^T and the K factors
    uint64_t *pv_done, *mma_done, *pv_drain;
};

__device__ __forceinline__ Bars carve_bars(uint8_t *smem)
{
    uint64_t *b = reinterpret_cast<uint64_t *>(smem + kOffBars);
    Bars r;
    r.q_full = b;
    r.code_full = b + 1;
    r.code_empty = r.code_full + kCodeStages;
    r.kfull = r.code_empty + kCodeStages;
    r.vfull = r.kfull + 2;
    r.vempty = r.vfull + 2;
    r.kv_tma = r.vempty + 2;
    r.s_full = r.kv_tma + 2;
    r.s_free = r.s_full + 2;
    r.pv_done = r.s_free + 2;
    r.mma_done = r.pv_done + 1;
    r.pv_drain = r.mma_done + 1;
    return r;
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint32_t *status)
{
    const bool ok = mbar_wait(bar, parity, status);
    return __all_sync(0xffffffffu, ok);
}

// True on every softmax thread if `pred` holds on any of them (also a
// barrier of the softmax warps).
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

// R consecutive fp32 columns of this thread's TMEM lane.
template <int R>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[R])
{
    static_assert(R == 16 || R == 24 || R == 32, "column count");
    if constexpr (R == 16) {
        tmem_ld16(taddr, r);
    } else if constexpr (R == 24) {
        tmem_ld24(taddr, r);
    } else {
        tmem_ld32(taddr, r);
    }
}

// What the softmax warps share about the CTA's work.
struct TnWork {
    uint8_t *smem;
    uint32_t sbase, tmem;
    int b, ctx, ntiles, key_begin, key_lim, nsplit, slot, h;
};

// The epilogue of one softmax warp, once the row sums are in `red`: O^T / l
// for rows r0 .. r0 + R - 1 (thread = output element d), or the split's FP32
// partial.  Not inlined: nothing it computes stays live across the tile loop.
template <int KVT>
__device__ __noinline__ void tn_epilogue(const DecodeParams &p, const TnWork wk, uint64_t *pv_done,
                                         int r0, int R, int warp, int lane, int sel, bool ok)
{
    const int quad = warp & 3;
    const uint32_t tl = wk.tmem + ((uint32_t)(32 * quad) << 16);
    const float *red = reinterpret_cast<const float *>(wk.smem + kOffRed);
    const float *m_arr = reinterpret_cast<const float *>(wk.smem + kOffM);
    const int G = p.group;
    const float *mfin = m_arr + sel * kN;
    const int jl = wk.ntiles - 1;
    const bool have_o = ok && wk.ntiles > 0 && warp_wait(pv_done, jl & 1, p.status);
    if (have_o)
        tc_fence_after();
    const int d = 32 * quad + lane;   // TMEM lane of O^T = output element d
    float vfac = 1.0f;
    if constexpr (kv_has_head_scale(KVT))
        vfac = __ldg(p.v_scale + wk.h * p.scale_stride);
#pragma unroll 1
    for (int c = 0; c < R; c += 8) {
        uint32_t o[8];
        if (have_o)   // warp-uniform
            tmem_ld8(tl + kTmO + r0 + c, o);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + c + j;
            if (r >= p.rows)
                break;
            const float lsum = red[r] + red[kN + r] + red[2 * kN + r] + red[3 * kN + r];
            const bool has = have_o && lsum > 0.0f;
            const float mrow = has ? mfin[r] : -INFINITY;
            if (wk.nsplit == 1) {
                const int tq = r / G, gq = r % G;
                const size_t qrow =
                    ((size_t)wk.b * p.q_len + tq) * p.num_q_heads + (size_t)wk.h * G + gq;
                const float y = has ? __uint_as_float(o[j]) * (vfac / lsum) : 0.0f;
                p.out[qrow * kHeadDim + d] = __float2half_rn(y);
                if (d == 0 && p.lse)
                    p.lse[qrow] = has ? (mrow + log2f(lsum)) * kLn2 : -INFINITY;
            } else {
                // FP32 partial: unnormalised O, max (log2 units) and sum
                const size_t wrow = ((size_t)wk.h * p.num_splits + wk.slot) * p.rows_per_cta + r;
                p.ws_o[wrow * kHeadDim + d] = has ? __uint_as_float(o[j]) : 0.0f;
                if (d == 0)
                    *reinterpret_cast<float2 *>(p.ws_ml + wrow * 2) =
                        has ? make_float2(mrow, lsum) : make_float2(-INFINITY, 0.0f);
            }
        }
    }
}

// The softmax role of one warp: R rows starting at r0 (of nr), keys of
// quadrant warp % 4.  Every softmax thread takes the same barrier steps, whatever its
// waits returned (the votes would otherwise never complete).
template <int KVT, int NP, int R>
__device__ __forceinline__ void softmax_role(const DecodeParams &p, const TnWork &wk,
                                             const Bars &bars, int r0, int nr, int warp, int lane)
{
    uint8_t *smem = wk.smem;
    const int tid = threadIdx.x;
    const int quad = warp & 3;
    const int key_in_tile = 32 * quad + lane;
    const uint32_t tl = wk.tmem + ((uint32_t)(32 * quad) << 16);
    float *red = reinterpret_cast<float *>(smem + kOffRed);   // [4][kN]
    int *pos_row = reinterpret_cast<int *>(smem + kOffPos);   // [kN]
    int *lo_row = pos_row + kN;                               // [kN]
    float *m_arr = reinterpret_cast<float *>(smem + kOffM);   // [2][kN]
    float *corr_row = reinterpret_cast<float *>(smem + kOffCorr);   // [kN]
    const int G = p.group;
    const int ctx = wk.ctx, key_lim = wk.key_lim;
    constexpr uint32_t kIdescO = idesc_f16_f32(128, NP, true, true);

    // Q rows -> shared memory (K-major B operand), zeros for padding rows;
    // each row's visible key range; P^T columns no thread writes stay 0
    for (int c = tid; c < kN * 16; c += kSoftmaxThreads) {
        const int r = c >> 4, dc = c & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < p.rows) {
            const int tq = r / G, gq = r % G;
            const size_t qrow =
                ((size_t)wk.b * p.q_len + tq) * p.num_q_heads + (size_t)wk.h * G + gq;
            v = __ldg(reinterpret_cast<const uint4 *>(p.q + qrow * kHeadDim) + dc);
        }
        *reinterpret_cast<uint4 *>(smem + kOffQ + (dc >> 3) * 8192 + sw128_off(r, dc & 7)) = v;
    }
    for (int c = tid; c < kKT * 8; c += kSoftmaxThreads)
        *reinterpret_cast<uint4 *>(smem + kOffP + c * 16) = make_uint4(0u, 0u, 0u, 0u);
    if (tid < kN) {
        const int r = tid;
        const bool valid = r < p.rows;
        const int ps = valid ? min(ctx - 1, query_position(p, wk.b, ctx, r / G)) : ctx - 1;
        pos_row[r] = ps;
        lo_row[r] = p.window > 0 && valid ? ps - p.window + 1 : INT_MIN;
        // padding rows see every key with m = 0: finite P, never written out
        m_arr[r] = valid ? kMInit : 0.0f;
        m_arr[kN + r] = m_arr[r];
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
        kfac_head *= __ldg(p.k_scale + wk.h * p.scale_stride);

    // partial sums of this key's rows live in tensor memory (lane = key)
    {
        uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int c = 0; c < R; c += 8)
            tmem_st8(tl + kTmL + r0 + c, z);
        tmem_st_wait();
    }
    int sel = 0;
    bool ok = true;
    for (int t = 0; t < wk.ntiles; ++t) {
        const int bj = t & 1;
        ok = warp_wait(&bars.s_full[bj], (t >> 1) & 1, p.status) && ok;
        // the per-key factors were written before the buffers were released
        if constexpr (KVT == kKvInt8)
            ok = ok && warp_wait(&bars.kfull[bj], (t >> 1) & 1, p.status);
        ok = ok && warp_wait(&bars.vfull[bj], (t >> 1) & 1, p.status);
        tc_fence_after();
        float kf = kfac_head, vf = 1.0f;
        if constexpr (KVT == kKvInt8) {
            kf = reinterpret_cast<const float *>(smem + kOffKsf)[bj * kKT + key_in_tile];
            vf = reinterpret_cast<const float *>(smem + kOffVsf)[bj * kKT + key_in_tile];
        }
        const int key0 = wk.key_begin + t * kKT;
        const int key = key0 + key_in_tile;
        const bool masked = key0 + kKT - 1 > pos_lo || key0 + kKT > key_lim || key0 < lo_hi;
        const uint32_t scol = tl + kTmS + bj * kN + r0;
        // scaled, masked scores of this thread's rows (log2 units); the
        // mask is gathered as a bit set, so that no per-row bounds stay live
        auto scores = [&](float (&x)[R]) {
            uint32_t u[R];
            if (ok)
                ld_cols<R>(scol, u);
#pragma unroll
            for (int i = 0; i < R; ++i)
                x[i] = ok ? __uint_as_float(u[i]) * kf : -INFINITY;
            if (masked) {
                uint32_t vis = 0u;
#pragma unroll 1
                for (int i = 0; i < R; ++i) {
                    const int r = r0 + i;
                    if (key <= pos_row[r] && key < key_lim && key >= lo_row[r])
                        vis |= 1u << i;
                }
#pragma unroll
                for (int i = 0; i < R; ++i)
                    if (!((vis >> i) & 1u))
                        x[i] = -INFINITY;
            }
        };
        float x[R];
        scores(x);
        float mx = -INFINITY;
        {
            const float *mc = m_arr + sel * kN + r0;
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(mc + i);
                x[i] -= m4.x;
                x[i + 1] -= m4.y;
                x[i + 2] -= m4.z;
                x[i + 3] -= m4.w;
                mx = fmaxf(mx, fmaxf(fmaxf(x[i], x[i + 1]), fmaxf(x[i + 2], x[i + 3])));
            }
        }
        if (softmax_any(mx > kRescaleLog2 || !ok)) {
            if (softmax_any(!ok)) {
                ok = false;
            } else {
                // move every row's reference to the running maximum: the
                // tile's row maxima across keys (lanes, then quadrants; one
                // thread per row), then each thread rescales its own rows
                scores(x);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    float v = x[i];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    if (lane == 0)
                        red[quad * kN + r0 + i] = v;
                }
                softmax_sync();
                if (tid < nr) {
                    const int r = tid;
                    const float mt = fmaxf(fmaxf(red[r], red[kN + r]),
                                           fmaxf(red[2 * kN + r], red[3 * kN + r]));
                    const float m_old = m_arr[sel * kN + r];
                    const float m_new = fmaxf(m_old, mt);
                    m_arr[(sel ^ 1) * kN + r] = m_new;
                    corr_row[r] = fast_exp2(m_old - m_new);
                }
                softmax_sync();
                sel ^= 1;
                // O^T is rescaled once every P V issued so far has completed
                if (t > 0)
                    ok = warp_wait(bars.pv_done, (t - 1) & 1, p.status) && ok;
                tc_fence_after();
                const float *mn = m_arr + sel * kN + r0;
                const float *cr = corr_row + r0;
#pragma unroll
                for (int c = 0; c < R; c += 8) {
                    float crc[8];
#pragma unroll
                    for (int j = 0; j < 8; j += 4) {
                        const float4 c4 = *reinterpret_cast<const float4 *>(cr + c + j);
                        const float4 m4 = *reinterpret_cast<const float4 *>(mn + c + j);
                        crc[j] = c4.x;
                        crc[j + 1] = c4.y;
                        crc[j + 2] = c4.z;
                        crc[j + 3] = c4.w;
                        x[c + j] -= m4.x;
                        x[c + j + 1] -= m4.y;
                        x[c + j + 2] -= m4.z;
                        x[c + j + 3] -= m4.w;
                    }
                    if (ok) {
                        uint32_t lv[8];
                        tmem_ld8(tl + kTmL + r0 + c, lv);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            lv[j] = __float_as_uint(__uint_as_float(lv[j]) * crc[j]);
                        tmem_st8(tl + kTmL + r0 + c, lv);
                    }
                    if (t > 0 && ok) {
                        uint32_t o[8];
                        tmem_ld8(tl + kTmO + r0 + c, o);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) * crc[j]);
                        tmem_st8(tl + kTmO + r0 + c, o);
                    }
                }
                tmem_st_wait();
            }
        }
        // S^T and the K factors of this tile are no longer needed
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars.s_free[bj]);
        // P^T row of this key, 8 rows at a time: fp16 2^(s - m) (times the
        // INT8 V scale's mantissa).  P^T is single-buffered: P V of the
        // previous tile (issued at its end) must be done first.
        if (t > 0)
            ok = warp_wait(bars.pv_done, (t - 1) & 1, p.status) && ok;
        uint8_t *prow = smem + kOffP + key_in_tile * 128;
#pragma unroll
        for (int c = 0; c < R / 8; ++c) {
            uint32_t lv[8], pk[4];
            if (ok)
                tmem_ld8(tl + kTmL + r0 + 8 * c, lv);
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const int i = 8 * c + j;
                const float e0 = fast_exp2(x[i]), e1 = fast_exp2(x[i + 1]);
                lv[j] = __float_as_uint(__uint_as_float(lv[j]) + e0);
                lv[j + 1] = __float_as_uint(__uint_as_float(lv[j + 1]) + e1);
                pk[j / 2] = pack_half2(e0 * vf, e1 * vf);
            }
            if (ok)
                tmem_st8(tl + kTmL + r0 + 8 * c, lv);
            const int chunk = r0 / 8 + c;   // 8 rows of this key
            *reinterpret_cast<uint4 *>(prow + ((chunk ^ (key_in_tile & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before();
        // every P^T store of the tile is in shared memory: warp 0 issues P V
        ok = !softmax_any(!ok);
        if (warp == 0 && ok) {
            tc_fence_after();
            const uint32_t vb = wk.sbase + kOffV + bj * kHatBuf;
            const uint64_t vd0 = desc_sw128(vb, kKVHalf, 1024);
            const uint64_t pd0 = desc_sw128(wk.sbase + kOffP, 8192, 1024);
#pragma unroll
            for (int ks = 0; ks < kKT / 16; ++ks)
                mma_f16_ss_elect(wk.tmem + kTmO, vd0 + (uint64_t)((ks * 2048) >> 4),
                                 pd0 + (uint64_t)((ks * 2048) >> 4), kIdescO,
                                 (t > 0 || ks > 0) ? 1u : 0u);
            mma_commit_elect(bars.pv_done);
            mma_commit_elect(&bars.vempty[bj]);
        }
    }

    // ---- epilogue: row sums across keys, then O^T / l ----
#pragma unroll 1
    for (int c = 0; c < R; c += 8) {
        uint32_t lv[8];
        tmem_ld8(tl + kTmL + r0 + c, lv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float s = __uint_as_float(lv[j]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0)
                red[quad * kN + r0 + c + j] = s;
        }
    }
    softmax_sync();
    tn_epilogue<KVT>(p, wk, bars.pv_done, r0, R, warp, lane, sel, ok);
    if (warp == 0) {   // every P V this warp issued has completed
        mma_commit_elect(bars.pv_drain);
        warp_wait(bars.pv_drain, 0, nullptr);
    }
}

template <int KVT, int BS, int NR>
__global__ void __launch_bounds__(kThreads, 1) decode_tn_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int kBPH = kHT / BS;     // cache blocks per code stage
    constexpr int kBPT = kKT / BS;     // cache blocks per tile
    constexpr int NP = (NR + 15) / 16 * 16;          // the MMAs' N
    constexpr int R0 = NR == 40 ? 24 : NR / 2;       // rows of softmax warps 0-3
    constexpr int R1 = NR - R0;                      // rows of softmax warps 4-7
    static_assert(NR % 8 == 0 && NR <= kN && R0 % 8 == 0 && R1 % 8 == 0, "row split");
    static_assert((kPrefetchStages + 1) * kBPH <= 32 && (kPrefetchStages / 2 + 1) * kBPT <= 32,
                  "prefetches stay in the table window");
    constexpr uint32_t kIdescS = idesc_f16_f32(kKT, NP, false, false);
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
        // K^ / V^ buffers: three dequant warps each, one arrival per code
        // stage (FP16: per tile)
        constexpr uint32_t kHatArrivals = 3 * (KVT == kKvFp16 ? 1 : 2);
        mbar_init(bars.q_full, kSoftmaxWarps);
        for (int s = 0; s < kCodeStages; ++s) {
            mbar_init(&bars.code_full[s], 32);   // one cp.async arrival per producer lane
            mbar_init(&bars.code_empty[s], kDequantWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.kfull[i], kHatArrivals);
            mbar_init(&bars.vfull[i], kHatArrivals);
            mbar_init(&bars.vempty[i], 1);
            mbar_init(&bars.kv_tma[i], 32);
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.s_free[i], kSoftmaxWarps);
        }
        mbar_init(bars.pv_done, 1);
        mbar_init(bars.mma_done, 1);
        mbar_init(bars.pv_drain, 1);
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

    if (warp == kWarpMma) {
        tmem_alloc(taddr_smem, kTmCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_smem;

    if (warp == kWarpCopy) {
        // ---------------------------------------------- copy producer --
        // 16-byte cp.async copies by all 32 lanes; each lane arrives on the
        // stage's barrier once its own copies have landed.  The stages up to
        // kPrefetchStages past the one being loaded are first fetched into
        // L2, so that several times the ring's bytes are in flight.
        const CacheView cv{p.k_cache, p.v_cache, p.k_scale_tok, p.v_scale_tok, p.num_kv_heads,
                           p.num_blocks, p.status};
        BlockWindow w;
        // every index stays inside the table row, even for a context longer
        // than the row can address (a caller error: those keys read block 0)
        w.init(p.block_table + (size_t)b * p.max_blocks_per_seq + blk_begin,
               min(nblk, p.max_blocks_per_seq - blk_begin), lane);
        if constexpr (KVT == kKvFp16) {
            // a whole 128-key tile straight into K^ / V^ buffers t % 2
            int pf_next = 2;
            for (int t = 0; t < ntiles; ++t) {
                for (; pf_next < ntiles && pf_next <= t + kPrefetchStages / 2; ++pf_next)
                    prefetch_blocks<BS, KVT>(cv, h, w, pf_next * kBPT,
                                             min(kBPT, nblk - pf_next * kBPT), lane);
                const int bj = t & 1;
                if (t >= 2 && !(warp_wait(&bars.s_free[bj], ((t - 2) >> 1) & 1, p.status) &&
                                warp_wait(&bars.vempty[bj], ((t - 2) >> 1) & 1, p.status)))
                    break;
                const int blk0 = t * kBPT;
                const int nb = min(kBPT, nblk - blk0);
                copy_fp16_rows<BS>(sbase + kOffK + bj * kHatBuf, sbase + kOffV + bj * kHatBuf,
                                   kKVHalf, cv, h, w, blk0, nb, kKT, lane);
                cp_async_mbar_arrive(&bars.kv_tma[bj]);
                if (t + 1 < ntiles)
                    w.slide(blk0 + nb, lane);
            }
        } else {
            // 64-key code stages; an odd last tile gets an empty stage
            int pf_next = kCodeStages;
            for (int u = 0; u < 2 * ntiles; ++u) {
                for (; pf_next < 2 * ntiles && pf_next <= u + kPrefetchStages; ++pf_next)
                    prefetch_blocks<BS, KVT>(cv, h, w, pf_next * kBPH,
                                             max(0, min(kBPH, nblk - pf_next * kBPH)), lane);
                const int s = u % kCodeStages;
                if (u >= kCodeStages &&
                    !warp_wait(&bars.code_empty[s], ((u - kCodeStages) / kCodeStages) & 1,
                               p.status))
                    break;
                const int blk0 = u * kBPH;
                const int nb = max(0, min(kBPH, nblk - blk0));
                const uint32_t dst = sbase + kOffCodes + s * kCodeStage;
                copy_code_rows<BS>(dst, dst + 8192, cv, h, w, blk0, nb, kHT, lane);
                if constexpr (KVT == kKvInt8) {
                    const uint32_t sd = sbase + kOffScl + s * 256;
                    copy_int8_scales<BS>(sd, sd + 128, cv, h, w, blk0, nb, lane);
                }
                cp_async_mbar_arrive(&bars.code_full[s]);
                if (u + 1 < 2 * ntiles)
                    w.slide(blk0 + nb, lane);
            }
        }
        // copies this warp issued land before it exits
        cp_async_wait_all();
    } else if (warp == kWarpMma) {
        // ----------------------------------------------- Q K^T issuer --
        // S(t) goes into the S^T buffer of S(t-2) and reads K^ buffer t % 2:
        // both are free once the softmax has finished with tile t - 2.
        if (ntiles > 0) {
            bool ok = warp_wait(bars.q_full, 0, p.status);
            const uint64_t qd0 = desc_sw128(sbase + kOffQ, 16, 1024);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int bj = t & 1;
                ok = warp_wait(&bars.kfull[bj], (t >> 1) & 1, p.status);
                if (ok && t >= 2)
                    ok = warp_wait(&bars.s_free[bj], ((t - 2) >> 1) & 1, p.status);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t kb = sbase + kOffK + bj * kHatBuf;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * kKVHalf + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_f16_ss_elect(tmem + kTmS + bj * kN, desc_sw128(kb + off, 16, 1024),
                                     qd0 + (uint64_t)(qoff >> 4), kIdescS, ks > 0 ? 1u : 0u);
                }
                mma_commit_elect(&bars.s_full[bj]);
            }
            mma_commit_elect(bars.mma_done);
            warp_wait(bars.mma_done, 0, p.status);
        }
    } else if (warp >= kDequantWarp0) {
        // ------------------------------------------------------ dequant --
        const int dw = warp - kDequantWarp0;
        const bool wide = dw == 2 || dw == 3;     // rows 0-31, all of d
        const int isv = dw & 1;                   // K: dw 0, 2, 4; V: dw 1, 3, 5
        const int row = wide ? lane : 32 + lane;  // key row of this thread in a code stage
        const int c0 = dw >= 4 ? 4 : 0;           // first 16-byte code chunk of the row
        const int nch = wide ? 8 : 4;             // chunks this thread converts
        const float kfac = p.scale_log2;
        uint64_t *full = isv ? bars.vfull : bars.kfull;
        const int hat_off = isv ? kOffV : kOffK;
        for (int u = 0; u < 2 * ntiles; ++u) {
            const int t = u >> 1, hk = u & 1, bj = t & 1;
            const int krow = hk * kHT + row;      // key row within the tile
            const int key = key_begin + t * kKT + krow;
            const bool live = key < ctx && key < key_lim;
            uint8_t *hat = smem + hat_off + bj * kHatBuf;
            if constexpr (KVT == kKvFp16) {
                if (hk == 0 && !warp_wait(&bars.kv_tma[bj], (t >> 1) & 1, p.status))
                    break;
                if (!live) {   // this warp's chunks of the row
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    for (int cc = c0; cc < c0 + nch; ++cc) {
                        uint8_t *dst = hat + (cc >> 2) * kKVHalf;
                        *reinterpret_cast<uint4 *>(dst + sw128_off(krow, (2 * cc) & 7)) = z;
                        *reinterpret_cast<uint4 *>(dst + sw128_off(krow, (2 * cc + 1) & 7)) = z;
                    }
                }
                if (hk == 1) {
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&full[bj]);
                }
                continue;
            }
            const int s = u % kCodeStages;
            if (!warp_wait(&bars.code_full[s], (u / kCodeStages) & 1, p.status))
                break;
            if (hk == 0 && t >= 2) {
                // K^: the softmax is done with tile t - 2; V^: its P V completed
                uint64_t *bar = isv ? &bars.vempty[bj] : &bars.s_free[bj];
                if (!warp_wait(bar, ((t - 2) >> 1) & 1, p.status))
                    break;
            }
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
                    wv[i] = *reinterpret_cast<const uint4 *>(codes + sw128_off(row, c0 + i));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i >= nch)
                    break;
                const int cc = c0 + i;   // 16-byte code chunk: d 16cc .. 16cc+15
                const uint4 cw = wv[i];
                uint32_t hv[8];
                if constexpr (KVT == kKvInt8) {
                    if (isv && !big) {
                        s8x4_to_half2x2_scaled(cw.x, p2, nb2, hv[0], hv[1]);
                        s8x4_to_half2x2_scaled(cw.y, p2, nb2, hv[2], hv[3]);
                        s8x4_to_half2x2_scaled(cw.z, p2, nb2, hv[4], hv[5]);
                        s8x4_to_half2x2_scaled(cw.w, p2, nb2, hv[6], hv[7]);
                    } else {
                        cvt4<KVT>(cw.x, hv[0], hv[1]);
                        cvt4<KVT>(cw.y, hv[2], hv[3]);
                        cvt4<KVT>(cw.z, hv[4], hv[5]);
                        cvt4<KVT>(cw.w, hv[6], hv[7]);
                        if (isv) {   // scales of 2^8 and above: code * s in fp16
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                __half2 xh = __hmul2(*reinterpret_cast<__half2 *>(&hv[e]),
                                                     *reinterpret_cast<const __half2 *>(&s2));
                                hv[e] = *reinterpret_cast<uint32_t *>(&xh);
                            }
                        }
                    }
                } else {
                    cvt4<KVT>(cw.x, hv[0], hv[1]);
                    cvt4<KVT>(cw.y, hv[2], hv[3]);
                    cvt4<KVT>(cw.z, hv[4], hv[5]);
                    cvt4<KVT>(cw.w, hv[6], hv[7]);
                }
                if (!live) {   // past the context or the split: codes may be anything
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        hv[e] = 0u;
                }
                uint8_t *dst = hat + (cc >> 2) * kKVHalf;
                *reinterpret_cast<uint4 *>(dst + sw128_off(krow, (2 * cc) & 7)) =
                    make_uint4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<uint4 *>(dst + sw128_off(krow, (2 * cc + 1) & 7)) =
                    make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
            if constexpr (KVT == kKvInt8) {
                if (c0 == 0 && !isv) {   // per-key score factor: softmax scale * log2(e) * K scale
                    float *ksf = reinterpret_cast<float *>(smem + kOffKsf) + bj * kKT;
                    ksf[krow] = live ? kfac * __half2float(__ushort_as_half(scl[row])) : 0.0f;
                }
                if (c0 == 0 && isv) {    // the mantissa of the V scale, applied to P
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
                mbar_arrive(&full[bj]);
            }
        }
    } else {
        // ------------------------------------------------------ softmax --
        const TnWork wk{smem, sbase, tmem, b, ctx, ntiles, key_begin, key_lim, si.nsplit, slot, h};
        if (warp < 4)
            softmax_role<KVT, NP, R0>(p, wk, bars, 0, NR, warp, lane);
        else
            softmax_role<KVT, NP, R1>(p, wk, bars, R0, NR, warp, lane);
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmCols);
    }
}

template <int KVT, int BS, int NR>
cudaError_t launch_tn(const DecodeParams &p, cudaStream_t stream)
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
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int KVT, int BS>
cudaError_t launch_tn_rows(const DecodeParams &p, cudaStream_t stream)
{
    if (p.rows <= 32)
        return launch_tn<KVT, BS, 32>(p, stream);
    if (p.rows <= 40)
        return launch_tn<KVT, BS, 40>(p, stream);
    if (p.rows <= 48)
        return launch_tn<KVT, BS, 48>(p, stream);
    return launch_tn<KVT, BS, 64>(p, stream);
}

}  // namespace

cudaError_t launch_decode_tn(const DecodeParams &p, int kv_dtype, cudaStream_t stream)
{
    switch (kv_dtype * 100 + p.block_size) {
#define PKVQ_TN_CASE(T, B) \
    case T * 100 + B: return launch_tn_rows<T, B>(p, stream);
        PKVQ_TN_CASE(kKvFp8, 16) PKVQ_TN_CASE(kKvFp8, 32) PKVQ_TN_CASE(kKvFp8, 64)
        PKVQ_TN_CASE(kKvInt8, 16) PKVQ_TN_CASE(kKvInt8, 32) PKVQ_TN_CASE(kKvInt8, 64)
        PKVQ_TN_CASE(kKvE5m2, 16) PKVQ_TN_CASE(kKvE5m2, 32) PKVQ_TN_CASE(kKvE5m2, 64)
        PKVQ_TN_CASE(kKvFp16, 16) PKVQ_TN_CASE(kKvFp16, 32) PKVQ_TN_CASE(kKvFp16, 64)
#undef PKVQ_TN_CASE
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkvq
