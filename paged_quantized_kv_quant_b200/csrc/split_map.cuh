// Length-proportional split map of the decode kernels ("1Cat-LLM" README,
// "Layer 2": Split-KV over the cached tokens of each sequence).
//
// A decode launch gives every (row group, KV head) the same number C of CTA
// slots.  The host knows only max_context_len; the context lengths live on
// the device.  So each CTA maps its slot to a (sequence, split) pair itself:
// sequence b gets nsplit_b = max(1, ceil(n_b / bpc)) consecutive slots, where
// n_b is its number of cache blocks that any of its queries can see and
// bpc = split_blocks(...) below, which keeps the total within C.  Sequences of
// different lengths then still give every CTA about the same number of
// blocks.  The merge kernel recomputes the same map to find a sequence's
// partials.
//
// Visible blocks: a sequence's keys end at its context length; with a
// sliding window w they start at the first query's position - w + 1 ("1Cat-LLM"
// README, "DFlash2 Long-Context Decay": the paged loop starts at the window's
// first tile), so blocks below it are neither read nor given a split.
#pragma once

#include "internal.h"

namespace pkvq {

// Blocks per split for C slots over `batch` sequences holding `total` blocks,
// the longest holding `longest`: a multiple of `gran`, at least `min_blocks`.
// With C > batch, any bpc >= total / (C - batch) keeps
//   sum_b max(1, ceil(n_b / bpc)) <= total / bpc + batch <= C;
// with C == batch every sequence gets one split.
__host__ __device__ inline int split_blocks(long long total, int C, int batch, int longest,
                                            int min_blocks, int gran)
{
    long long v;
    if (C <= batch) {
        v = longest > 1 ? longest : 1;
    } else {
        v = (total + (C - batch) - 1) / (C - batch);
        if (v < min_blocks)
            v = min_blocks;
    }
    v = (v + gran - 1) / gran * gran;
    return (int)v;
}

struct SplitInfo {
    int b;        // sequence (-1: a slot past the last split)
    int split;    // split of that sequence
    int nsplit;   // splits of that sequence
    int first;    // slot of its first split
    int ctx;      // its context length
    int bpc;      // blocks per split
    int blk0;     // its first visible block (splits start at blk0 + split * bpc)
};

// Position of query token t of sequence b among the call's keys.
__device__ __forceinline__ int query_position(const DecodeParams &p, int b, int ctx, int t)
{
    return p.query_pos ? p.query_pos[(size_t)b * p.q_len + t] : ctx - p.q_len + t;
}

// First block any query of sequence i can see (0 without a sliding window).
template <int BS>
__device__ __forceinline__ int seq_first_block(const DecodeParams &p, int i, int ctx)
{
    if (p.window <= 0)
        return 0;
    int lo = query_position(p, i, ctx, 0);
    for (int t = 1; t < p.q_len; ++t)
        lo = min(lo, query_position(p, i, ctx, t));
    return max(0, lo - p.window + 1) / BS;
}

// Visible blocks of sequence i (0 for i >= batch).
template <int BS>
__device__ __forceinline__ int seq_blocks(const DecodeParams &p, int i)
{
    if (i >= p.batch)
        return 0;
    const int ctx = max(p.context_lens[i], 0);
    const int end = (ctx + BS - 1) / BS;
    return max(0, end - seq_first_block<BS>(p, i, ctx));
}

// Computed by one whole warp (result warp-uniform).  slot >= 0: the
// (sequence, split) owning that slot; slot < 0: where sequence `seq` is.
template <int BS>
__device__ SplitInfo find_split(const DecodeParams &p, int slot, int seq)
{
    const int lane = threadIdx.x & 31;
    long long total = 0;
    int longest = 0;
    const int n0 = seq_blocks<BS>(p, lane);   // kept: most batches have at most 32 sequences
    for (int base = 0; base < p.batch; base += 32) {
        const int n = base == 0 ? n0 : seq_blocks<BS>(p, base + lane);
        total += n;
        longest = max(longest, n);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, o);
        longest = max(longest, __shfl_xor_sync(0xffffffffu, longest, o));
    }
    SplitInfo r{-1, 0, 0, 0, 0,
                split_blocks(total, p.num_splits, p.batch, longest, p.split_min_blocks,
                             p.split_gran),
                0};
    int run = 0;   // slots taken by the sequences before this chunk
    for (int base = 0; base < p.batch; base += 32) {
        const int i = base + lane;
        const int n = base == 0 ? n0 : seq_blocks<BS>(p, i);
        const int ns = i < p.batch ? max(1, (n + r.bpc - 1) / r.bpc) : 0;
        int incl = ns;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += v;
        }
        const int first = run + incl - ns;
        const bool hit =
            i < p.batch && (slot >= 0 ? (slot >= first && slot < first + ns) : i == seq);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            r.b = base + src;
            r.first = __shfl_sync(0xffffffffu, first, src);
            r.nsplit = __shfl_sync(0xffffffffu, ns, src);
            r.split = slot >= 0 ? slot - r.first : 0;
            r.ctx = max(p.context_lens[r.b], 0);
            r.blk0 = seq_first_block<BS>(p, r.b, r.ctx);
            break;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    return r;
}

}  // namespace pkvq
