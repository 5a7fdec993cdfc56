// Pieces shared by the tensor-core decode kernels (pa_decode_tc.cu,
// pa_decode_umma.cu): TMA wrappers, the block-stream schedule, and the host
// helpers that build tensor maps, size grids and launch the merge.
#pragma once
#include <cudaTypedefs.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// One contiguous run of blocks of one (sequence, KV head) row.
struct Seg {
    int b, kvh, L, nb;  // row: sequence, KV head, tokens, blocks
    int j0, j1;         // this segment: blocks [j0, j1) of the row
    int fr;             // index of the row's first block in the concatenated stream
    int ch;             // chunk that holds the segment (-1: whole-row mode)
    int ncol;           // the row's real (not padding) columns
};

// Walks the ranges of one warp and cuts them into segments at row boundaries.
struct SegIter {
    int k;              // range counter
    int f, fend;        // position and end in the concatenated stream
    int ch;
    bool done;
};

// Consecutive table entries of one segment, read 32 at a time (lane l holds
// entry o + l as a TMA row coordinate, -2 for a block id outside the pool).
struct Win {
    Seg sg;
    int o, n;
    int kc;  // the cache's KV head of the window's row
    bool valid;
};

// Chunks of the concatenated block stream: n chunks of c blocks (the last one
// shorter); warp w takes chunks w, w + W, w + 2W, ...
#ifndef PA_TC_GAMMA
#define PA_TC_GAMMA 2
#endif
// Chunks are cut in a virtual stream in which every non-empty row is followed by
// gam extra units (the cost of finishing one segment and starting the next, in
// blocks), so a chunk that holds several row ends holds fewer blocks.  cum[b] /
// cumv[b]: blocks / virtual units of the rows of sequences before b.
struct Chunks {
    int total, vtotal, c, n, gam, Hkv;
    const int *cum, *cumv;
    // virtual position of block j of row (b, kvh) of nb blocks
    __device__ int vpos(int b, int kvh, int nb, int j) const { return cumv[b] + kvh * (nb + gam) + j; }
    // actual stream position of the first block at or after virtual position v
    __device__ int at(int v) const {
        if (v >= vtotal) return total;
        int l = 0, h = nseq;  // largest b with cumv[b] <= v: sequence b is not empty
        while (h - l > 1) {
            const int mid = (l + h) >> 1;
            if (cumv[mid] <= v) l = mid; else h = mid;
        }
        const int nb = cum[l + 1] - cum[l];
        const int off = v - cumv[l], rl = nb + gam;
        const int kvh = off / rl, j = off - kvh * rl;
        return cum[l] * Hkv + kvh * nb + (j < nb ? j : nb);
    }
    int nseq;
    __device__ int start(int ch) const { return at(ch * c); }
    __device__ int end(int ch) const { return at((ch + 1) * c); }
    // chunk of block j of row (b, kvh)
    __device__ int of(int b, int kvh, int nb, int j) const { return vpos(b, kvh, nb, j) / c; }
    // whether the row (b, kvh) begins after its first chunk's first block, i.e. the
    // block before it (the previous row's last) lies in the same chunk
    __device__ bool mid_start(int b, int kvh, int nb) const {
        const int fr = cum[b] * Hkv + kvh * nb;
        return fr > 0 && (vpos(b, kvh, nb, 0) - gam - 1) / c == vpos(b, kvh, nb, 0) / c;
    }
};


// Host side (pa_decode_tc.cu).
// 2-D TMA map over a cache [rows][D] (128-byte boxes of 16 rows, 128-byte swizzle;
// 4-bit: one unswizzled box per row), cached by (base, rows, D, dtype).
bool tc_cache_tensor_map(CUtensorMap *m, const void *base, int64_t rows, int D, int dtype);
// SMs and resident CTAs per SM of a kernel at this block size and shared memory.
bool tc_launch_shape(const void *kernel, int threads, int smem, int *sms, int *per_sm);
// merge_tc_kernel over rows of GC = a2.G columns (16, 32 or 64; no multi-query mapping),
// the decode grid's workers a2.tc_W being CTAs that each walk whole chunks.
int launch_merge_rows(const DecodeArgs &a2, int sms, cudaStream_t st);

}  // namespace pa
