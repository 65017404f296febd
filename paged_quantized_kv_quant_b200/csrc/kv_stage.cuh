// Producer-side copies of paged-cache blocks into shared-memory stages for
// the tensor-core attention kernels: a sliding window over the split's
// block-table row, 16-byte cp.async copies of K/V rows into the 128-byte-
// swizzled stage layout, and L2 prefetches of the blocks ahead.
//
// Why per-lane copies: a cache block of 16 tokens holds 2 KB of K (8-bit
// codes) per KV head, scattered over the pool.  One bulk-tensor copy per block
// (plus two for the INT8 scales) is a descriptor-driven operation issued by a
// single thread; at a few hundred cycles of issue each, a 64-key stage of
// INT8 K/V took ~2,300 cycles to request.  A warp of cp.async copies moves 4
// rows x 128 bytes per instruction with no per-block setup.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkvq {

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled tile
// (the layout the tensor-core descriptors with SWIZZLE_128B read).
__device__ __forceinline__ uint32_t sw128_off(int r, int c)
{
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// The cache as the producer sees it.
struct CacheView {
    const uint8_t *k, *v;          // [blocks][Hkv][block_size][row bytes]
    const uint16_t *ks, *vs;       // INT8: per-(block, head, token) fp16 scales
    int num_kv_heads, num_blocks;
    uint32_t *status;
};

// A producer warp's window over one block-table row: entries [wbase,
// wbase + 64) in two registers per lane.  Every index read stays below `n`
// (entries past it read as block 0).
struct BlockWindow {
    const int32_t *row;
    int n, wbase, w0, w1;

    __device__ __forceinline__ void init(const int32_t *r, int nread, int lane)
    {
        row = r;
        n = nread;
        wbase = 0;
        w0 = lane < n ? __ldg(r + lane) : 0;
        w1 = 32 + lane < n ? __ldg(r + 32 + lane) : 0;
    }

    // Physical block of entry bi, bi in [wbase, wbase + 64).  Warp-collective:
    // every lane calls it (bi may differ between lanes).
    __device__ __forceinline__ int id(int bi, const CacheView &cv) const
    {
        const int a = __shfl_sync(0xffffffffu, w0, bi & 31);
        const int c = __shfl_sync(0xffffffffu, w1, bi & 31);
        int phys = (bi - wbase) < 32 ? a : c;
#ifdef PKVQ_BOUNDS_CHECK
        if (phys < 0 || phys >= cv.num_blocks) {
            atomicOr(cv.status, kStatusBadBlock);
            phys = 0;
        }
#endif
        return phys;
    }

    // Moves the window so that entry `next` lies in [wbase, wbase + 32).
    __device__ __forceinline__ void slide(int next, int lane)
    {
        while (next >= wbase + 32) {
            wbase += 32;
            w0 = w1;
            w1 = wbase + 32 + lane < n ? __ldg(row + wbase + 32 + lane) : 0;
        }
    }
};

// 8-bit codes of `rows` keys (a multiple of 4): the nb blocks from window
// entry blk0.  Row r of the stage lands at kdst / vdst + sw128_off(r, c);
// rows past nb blocks are not written.
template <int BS>
__device__ __forceinline__ void copy_code_rows(uint32_t kdst, uint32_t vdst, const CacheView &cv,
                                               int h, const BlockWindow &w, int blk0, int nb,
                                               int rows, int lane)
{
    int cur = -1, phys = 0;
    for (int k = 0; k < rows / 4; ++k) {
        const int r = 4 * k + (lane >> 3), c = lane & 7;
        const int i = (4 * k) / BS;   // warp-uniform block
        if (i >= nb)
            break;
        if (i != cur) {
            phys = w.id(blk0 + i, cv);
            cur = i;
        }
        const size_t g = (((size_t)phys * cv.num_kv_heads + h) * BS + r % BS) * 128 + c * 16;
        cp_async_16(kdst + sw128_off(r, c), cv.k + g);
        cp_async_16(vdst + sw128_off(r, c), cv.v + g);
    }
}

// INT8 scales of the same keys: 8 keys per 16-byte copy, K scales of stage
// key j at kdst + 2 j, V scales at vdst + 2 j.
template <int BS>
__device__ __forceinline__ void copy_int8_scales(uint32_t kdst, uint32_t vdst, const CacheView &cv,
                                                 int h, const BlockWindow &w, int blk0, int nb,
                                                 int lane)
{
    const int nck = nb * BS / 8;   // copies per K (and per V); at most 16 in all
    const int q = lane < nck ? lane : lane - nck;
    const int phys = w.id(blk0 + min((8 * q) / BS, max(nb - 1, 0)), cv);   // all lanes
    if (lane < 2 * nck) {
        const size_t y = ((size_t)phys * cv.num_kv_heads + h) * BS + (8 * q) % BS;
        cp_async_16((lane < nck ? kdst : vdst) + q * 16, (lane < nck ? cv.ks : cv.vs) + y);
    }
}

// FP16 rows (256 bytes) of `rows` keys (a multiple of 2) into [d half][row]
// [64 d] tiles: chunk c of row r at dst + (c / 8) * half_bytes +
// sw128_off(r, c % 8).
template <int BS>
__device__ __forceinline__ void copy_fp16_rows(uint32_t kdst, uint32_t vdst, uint32_t half_bytes,
                                               const CacheView &cv, int h, const BlockWindow &w,
                                               int blk0, int nb, int rows, int lane)
{
    int cur = -1, phys = 0;
    for (int k = 0; k < rows / 2; ++k) {
        const int r = 2 * k + (lane >> 4), c = lane & 15;
        const int i = (2 * k) / BS;
        if (i >= nb)
            break;
        if (i != cur) {
            phys = w.id(blk0 + i, cv);
            cur = i;
        }
        const size_t g = (((size_t)phys * cv.num_kv_heads + h) * BS + r % BS) * 256 + c * 16;
        const uint32_t o = (c >> 3) * half_bytes + sw128_off(r, c & 7);
        cp_async_16(kdst + o, cv.k + g);
        cp_async_16(vdst + o, cv.v + g);
    }
}

// L2 prefetch of nb blocks from window entry blk0 (K and V rows, and the
// INT8 scales), one 128-byte line per lane and instruction.
template <int BS, int KVT>
__device__ __forceinline__ void prefetch_blocks(const CacheView &cv, int h, const BlockWindow &w,
                                                int blk0, int nb, int lane)
{
    constexpr int kLines = BS * kv_elem_bytes(KVT);   // lines per K (or V) block
    for (int i = 0; i < nb; ++i) {
        const int phys = w.id(blk0 + i, cv);
        const size_t y = ((size_t)phys * cv.num_kv_heads + h) * BS;
        const size_t base = y * 128 * kv_elem_bytes(KVT);
#pragma unroll
        for (int j = lane; j < 2 * kLines; j += 32)
            prefetch_l2((j < kLines ? cv.k : cv.v) + base + (size_t)(j % kLines) * 128);
        if constexpr (KVT == kKvInt8) {
            if (lane < 2)
                prefetch_l2((lane ? cv.vs : cv.ks) + y);
        }
    }
}

}  // namespace pkvq
