// Paged decode attention, tensor-core kernel family (fp16 / bf16, int8 and 4-bit
// KV; up to 8 (query token, head) columns per row, larger groups as several rows).
//
// Same computation as the CUDA-core kernel (lqnn.cn/news/235768 sections 1.2,
// 2.2, 3.2, 4.2; chanyi.net.cn/article/49 section 四):
//   out[b][h] = sum_t softmax_t(scale * q[b][h] . K[b][t]) V[b][t]
// with fp32 online softmax and fp32 accumulation.  The GQA group's Q.K^T and
// P.V products are small dense contractions, so they run as mma.sync
// m16n8k16 with the group padded to n = 8:
//   S^T[16 tokens x 8 heads] = K[16 x d] . Q^T[d x 8]      (A = K tile, B = q)
//   O^T[d x 8 heads]        += V^T[d x 16] . P^T[16 x 8]   (A = V tile^T, B = p)
// which keeps the per-token instruction count low enough that the kernel is
// bound by HBM, not by issue.
//
// Data movement: the cache tile of one (block, KV head) is 16 rows x d, rows
// contiguous.  A 2-D tensor map over the cache ([rows = blocks*H_kv*16][d])
// with 128-byte swizzle brings each tile into shared memory with TMA
// (cp.async.bulk.tensor, 64-element boxes), so the ldmatrix reads of 8 rows x
// 16 bytes hit 8 different bank groups.
//
// Scheduling: a persistent grid; every warp is an independent worker with its
// own ring of (K tile, V tile) stages (a fixed byte depth: two stages of fp16 at
// d = 128, more for smaller tiles) and its own mbarriers.  The
// (sequence, KV head) rows are laid end to end as one stream of blocks (row
// order: sequence, then KV head; total = sum_b ceil(L_b / 16) * H_kv blocks).
// With partition_size == 0 warp w takes whole rows w, w + W, ... (W = warps in
// the grid).  Otherwise the stream is cut into chunks -- by default W' =
// min(W, 2048) chunks of equal cost, the cost of a chunk being its blocks plus
// PA_TC_GAMMA for every row that ends in it (the work of finishing a segment and
// starting the next, measured at about 1.4 blocks' time), so every warp has the
// same work whatever the length mix; partition_size > 0 fixes chunks of
// partition/16 blocks -- and warp w takes chunks w, w + W, ...  A chunk is
// walked segment by segment (a segment = the part of one row inside the chunk);
// the producer side of the warp keeps issuing TMA for the next blocks across
// segment and chunk ends, so the copy stream does not drain.  A segment that is
// a whole row writes the output directly.  A cut segment is a partial: its
// normalised output and log2-sum-exp go to workspace slot 2*chunk (first segment
// of the chunk) or 2*chunk + 1 (last).  merge_tc_kernel, launched right after
// with programmatic dependent launch, merges every cut row:
//   out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M).
// No warp ever waits for another.  (Merging inside the decode kernel, by the
// warp that finished a row's last partial, put those merges at the end of the
// slowest warps: a separate merge kernel measured 7% faster on the ragged trace.)
//
// Groups of 16, 32 or 64 query heads per KV head run in decode_coop_kernel
// (one CTA per chunk of cache rows, its warps sharing each staged tile, with
// the heads on the M side of the MMA).
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>
#include <unordered_map>

#include "pa_common.cuh"
#include "pa_internal.h"
#include "pa_tc_shared.cuh"

namespace pa {

PA_ERROR_WORD_ACCESSOR(error_word_decode_tc)

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
template <typename T> struct Mma;
template <> struct Mma<__half> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    // d = a . b (a zero accumulator)
    static __device__ __forceinline__ void mma0(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
    }
};
template <> struct Mma<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ void mma0(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
    }
};

// ---------------------------------------------------------------------------
// configuration
// ---------------------------------------------------------------------------
#ifndef PA_TC_WARPS
#define PA_TC_WARPS 4
#endif
// Cache bytes each warp keeps in flight.  A warp's ring stage holds one block's
// K and V tiles, so the stage count is this over the stage size: two stages of
// fp16 at d = 128 (three measured slower on the ragged trace: more bytes in
// flight per warp only lengthen the DRAM queues), and proportionally more for
// the smaller int8, 4-bit and d = 64 tiles, which otherwise leave the warps
// latency-bound at a fraction of the bandwidth.
#ifndef PA_TC_INFLIGHT
#define PA_TC_INFLIGHT (16 * 1024)
#endif
// shared memory for the rings and q slots of one CTA; two CTAs fit on an SM
#ifndef PA_TC_RING_BUDGET
#define PA_TC_RING_BUDGET (96 * 1024)
#endif
// int8 and 4-bit caches: consume the blocks of a segment two at a time (their
// conversion-heavy fragment work interleaves), with the ring twice as deep
#ifndef PA_TC_PAIRS
#define PA_TC_PAIRS 1
#endif
#ifndef PA_TC_HOIST_V
#define PA_TC_HOIST_V 1
#endif
#ifndef PA_TC_MIN_CTAS
#define PA_TC_MIN_CTAS 1
#endif


// TKV: the cache element: the q/out type T, int8_t, or U4x2 (two 4-bit values
// per byte).  fp16/bf16 and int8 tile rows come as 128-byte boxes (64 or 128
// elements) with 128-byte swizzle; a 4-bit tile row is D / 2 bytes, one box, no
// swizzle.
struct U4x2 {
    uint8_t v;
};
template <typename TKV, int D, int G>
struct TcCfg {
    static constexpr bool I4 = std::is_same<TKV, U4x2>::value;
    // warps (independent workers) per CTA, and CTAs per SM the registers are sized
    // for.  A head_dim-256 stage is 16 KB (K and V tiles of 8 KB), so two stages per
    // warp and three warps per CTA keep two CTAs (six warps, 192 KB in flight) on an SM.
    static constexpr int NW = D == 256 ? 3 : PA_TC_WARPS;
    // 4-bit tiles are 2 KB: their conversion chains keep a warp busy far longer than its
    // copies take, so three CTAs (twelve warps, 168 registers) share an SM
    static constexpr int MIN_CTAS = D == 256 ? 2 : (I4 ? 3 : PA_TC_MIN_CTAS);
    static constexpr int BUDGET = MIN_CTAS >= 3 ? 200 * 1024 / MIN_CTAS - 8 * 1024 : PA_TC_RING_BUDGET;
    static constexpr int THREADS = NW * 32;
    static constexpr int ROW_BYTES = I4 ? D / 2 : 128;              // bytes per box row
    static constexpr int BOXW = I4 ? D / 2 : 128 / (int)sizeof(TKV);  // TMA elements per box row
    static constexpr int BOXES = I4 ? 1 : D / BOXW;                  // boxes per tile row
    static constexpr int BOX_BYTES = 16 * ROW_BYTES;                 // one box of a tile
    static constexpr int TILE = BOXES * BOX_BYTES;
    static constexpr int STAGE = 2 * TILE;        // K tile, then V tile
    static constexpr int QSLOT = G * D * 2;       // q rows of a segment's G heads
    static constexpr int stages() {
        int s = PA_TC_INFLIGHT / STAGE;
        s = s < 2 ? 2 : (s > 8 ? 8 : s);
        while (s > 2 && NW * s * (STAGE + QSLOT) > BUDGET) --s;
        return s;
    }
    static constexpr int S = stages();            // ring stages per warp
    static constexpr int KSTEPS = D / 16;         // QK k-steps
    static constexpr int MTILES = D / 16;         // PV m-tiles
    static constexpr int DPL = D / 32;            // dims per lane in the merge
    static constexpr int RING = NW * S * STAGE;
    static constexpr int QRING_OFF = RING;        // [NW][S] q slots, one per stage
    static constexpr int BAR_OFF = QRING_OFF + NW * S * QSLOT;
    static constexpr int OK_OFF = BAR_OFF + NW * S * 8;
    static constexpr int SC_OFF = OK_OFF + NW * S * 4;    // float [NW][S][2]: int8 K, V scales
    // pa_decode_append (fp16 / bf16 caches): a row end's new K and V rows, and the cache
    // slot its warp writes
    static constexpr int PATCH = std::is_same<TKV, __half>::value || std::is_same<TKV, __nv_bfloat16>::value ? 2 * D * 2 : 0;
    static constexpr int PATCH_OFF = (SC_OFF + NW * S * 8 + 15) / 16 * 16;
    static constexpr int PSLOT_OFF = PATCH_OFF + NW * S * PATCH;  // int [NW][S], -1: none
    static constexpr int CUM_OFF = PSLOT_OFF + NW * S * 4;
    static int smem_bytes(int B) { return 1024 + CUM_OFF + (3 * B + 3) * 4; }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int N> struct FVec;
template <> struct FVec<4> {
    using type = float4;
    static __device__ __forceinline__ float4 ld(const float *p) { return __ldcg(reinterpret_cast<const float4 *>(p)); }
    static __device__ __forceinline__ float get(const float4 &v, int e) { return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w; }
};
template <> struct FVec<8> {
    struct type {
        float4 a, b;
    };
    static __device__ __forceinline__ type ld(const float *p) {
        return {__ldcg(reinterpret_cast<const float4 *>(p)), __ldcg(reinterpret_cast<const float4 *>(p) + 1)};
    }
    static __device__ __forceinline__ float get(const type &v, int e) {
        const float4 &h = e < 4 ? v.a : v.b;
        const int f = e & 3;
        return f == 0 ? h.x : f == 1 ? h.y : f == 2 ? h.z : h.w;
    }
};
template <> struct FVec<2> {
    using type = float2;
    static __device__ __forceinline__ float2 ld(const float *p) { return __ldcg(reinterpret_cast<const float2 *>(p)); }
    static __device__ __forceinline__ float get(const float2 &v, int e) { return e == 0 ? v.x : v.y; }
};

// ---------------------------------------------------------------------------
// int8 tiles -> fp16 MMA fragments
// ---------------------------------------------------------------------------
// Two int8 values -> two fp16 values, exactly.  u holds the bytes biased by 128
// (word ^ 0x80808080); the byte permute builds the fp16 bit patterns 0x64xx =
// 1024 + (x + 128) for the two bytes picked by `sel`, and subtracting 1152
// (0x6480) leaves x.  Every value involved is an integer below 2048, so fp16
// holds all of them exactly.
__device__ __forceinline__ uint32_t i8x2_to_h2(uint32_t u, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(u), "r"(0x64646464u), "r"(sel));
    asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(r) : "r"(0x64806480u));
    return r;
}
constexpr uint32_t kLoPair = 0x5140u;  // bytes 0, 1 -> low, high half
constexpr uint32_t kHiPair = 0x5342u;  // bytes 2, 3 -> low, high half

__device__ __forceinline__ void lds_v4(uint32_t (&w)[4], uint32_t addr) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr)
                 : "memory");
}
// 16-byte chunk `ch` of row `r` of a 128-byte-row tile written by TMA with
// 128-byte swizzle
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int ch) { return tile + r * 128 + ((ch ^ (r & 7)) << 4); }

// K (A operand of S^T = K . Q^T; m = tokens, k = dims) from an int8 tile of 16
// tokens x 128 dims.  The contraction runs over the dims in the order that lets
// a thread read its own 32 contiguous bytes: in k-step ks, thread column c holds
// the dims 32c + 4ks .. 32c + 4ks + 3 (k slots 2c, 2c+1 <- dims +0, +1; k slots
// 2c+8, 2c+9 <- dims +2, +3), and q is read in the same order.  kload_i8 reads
// the raw words (biased by 128), kfrag_i8 converts the fragment of one k-step.
__device__ __forceinline__ void kload_i8(uint32_t (&w)[2][8], uint32_t tile, int g, int c) {
    lds_v4(*reinterpret_cast<uint32_t(*)[4]>(&w[0][0]), swz(tile, g, 2 * c));
    lds_v4(*reinterpret_cast<uint32_t(*)[4]>(&w[0][4]), swz(tile, g, 2 * c + 1));
    lds_v4(*reinterpret_cast<uint32_t(*)[4]>(&w[1][0]), swz(tile, g + 8, 2 * c));
    lds_v4(*reinterpret_cast<uint32_t(*)[4]>(&w[1][4]), swz(tile, g + 8, 2 * c + 1));
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j) w[r][j] ^= 0x80808080u;
}
__device__ __forceinline__ void kfrag_i8(const uint32_t (&w)[2][8], int ks, uint32_t (&a)[4]) {
    a[0] = i8x2_to_h2(w[0][ks], kLoPair);  // token g, k slots 2c, 2c+1
    a[1] = i8x2_to_h2(w[1][ks], kLoPair);  // token g + 8
    a[2] = i8x2_to_h2(w[0][ks], kHiPair);  // token g, k slots 2c+8, 2c+9
    a[3] = i8x2_to_h2(w[1][ks], kHiPair);
}

// V^T (A operand of O^T += V^T . P^T; m = dims, k = tokens) from an int8 tile.
// Thread row g owns the 16 dims 16g .. 16g + 15: m-tile i, row g is dim
// 16g + i and row g + 8 is dim 16g + 8 + i.  The k slots are the tokens
// themselves (2c, 2c+1 and 2c+8, 2c+9), as the P^T fragments expect.  vload_i8
// reads the four token rows' 16 bytes (biased by 128), vfrag_i8 converts the
// fragment of m-tile i: byte i % 4 of word i / 4 (row g) or 2 + i / 4 (row
// g + 8) of each token, paired by token.
__device__ __forceinline__ void vload_i8(uint32_t (&r)[4][4], uint32_t tile, int g, int c) {
    lds_v4(r[0], swz(tile, 2 * c, g));
    lds_v4(r[1], swz(tile, 2 * c + 1, g));
    lds_v4(r[2], swz(tile, 2 * c + 8, g));
    lds_v4(r[3], swz(tile, 2 * c + 9, g));
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) r[t][j] ^= 0x80808080u;
}
__device__ __forceinline__ void vfrag_i8(const uint32_t (&r)[4][4], int i, uint32_t (&a)[4]) {
    const uint32_t sel = (uint32_t)(i & 3) | ((uint32_t)(4 + (i & 3)) << 4);  // byte i%4 of both tokens
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // register q: token pair q / 2, dims row (q & 1 ? g + 8 : g)
        const int p = q >> 1, w = ((q & 1) << 1) + (i >> 2);
        uint32_t t;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(r[2 * p][w]), "r"(r[2 * p + 1][w]), "r"(sel));
        a[q] = i8x2_to_h2(t, kLoPair);
    }
}

// ---------------------------------------------------------------------------
// 4-bit tiles -> fp16 MMA fragments
// ---------------------------------------------------------------------------
// A 4-bit tile row is D / 2 bytes (64 at D = 128), unswizzled; byte k holds
// element 2k in its low four bits and 2k+1 in its high four, each as q + 8, so
// nibble t of a 32-bit word (bits 4t .. 4t+3) is element 8w + t of that word w.
// Two nibbles in bits 0-3 and 16-19 become an fp16 pair exactly: OR-ing
// 0x6400 gives 1024 + n, and subtracting 1032 (0x6408) leaves n - 8 = q.
__device__ __forceinline__ uint32_t u4pair_to_h2(uint32_t x) {  // x: nibbles in bits 0-3, 16-19
    uint32_t r = (x & 0x000f000fu) | 0x64006400u;
    asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(r) : "r"(0x64086408u));
    return r;
}
__device__ __forceinline__ void lds_v2(uint32_t (&w)[2], uint32_t addr) {
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr) : "memory");
}

// K from a 4-bit tile (D = 128): thread column c reads the 16 bytes (32 dims
// 32c .. 32c + 31) of tokens g and g + 8.  The contraction runs over the dims in
// the order the nibble pairs give: in k-step ks (word w = ks / 2, t0 = 2 (ks % 2),
// t1 = t0 + 1) k slots 2c, 2c+1 are dims 32c + 8w + t0 and + t0 + 4, k slots 2c+8,
// 2c+9 dims 32c + 8w + t1 and + t1 + 4; q is read in the same order.
__device__ __forceinline__ void kload_i4(uint32_t (&w)[2][4], uint32_t tile, int g, int c) {
    lds_v4(w[0], tile + g * 64 + c * 16);
    lds_v4(w[1], tile + (g + 8) * 64 + c * 16);
}
__device__ __forceinline__ void kfrag_i4(const uint32_t (&w)[2][4], int ks, uint32_t (&a)[4]) {
    const int wi = ks >> 1, t0 = 2 * (ks & 1);
    a[0] = u4pair_to_h2(w[0][wi] >> (4 * t0));        // token g
    a[1] = u4pair_to_h2(w[1][wi] >> (4 * t0));        // token g + 8
    a[2] = u4pair_to_h2(w[0][wi] >> (4 * t0 + 4));
    a[3] = u4pair_to_h2(w[1][wi] >> (4 * t0 + 4));
}

// V^T from a 4-bit tile: thread row g owns dims 16g .. 16g + 15 (8 bytes of each
// token row), as in the int8 path; the tokens are 2c, 2c+1 and 2c+8, 2c+9.
__device__ __forceinline__ void vload_i4(uint32_t (&r)[4][2], uint32_t tile, int g, int c) {
    lds_v2(r[0], tile + (2 * c) * 64 + g * 8);
    lds_v2(r[1], tile + (2 * c + 1) * 64 + g * 8);
    lds_v2(r[2], tile + (2 * c + 8) * 64 + g * 8);
    lds_v2(r[3], tile + (2 * c + 9) * 64 + g * 8);
}
__device__ __forceinline__ void vfrag_i4(const uint32_t (&r)[4][2], int i, uint32_t (&a)[4]) {
    // byte i / 2 of both tokens' words into bytes 0 and 2, then nibble i % 2 of each
    const uint32_t sel = (uint32_t)(i >> 1) | ((uint32_t)(4 + (i >> 1)) << 8);
    const int sh = 4 * (i & 1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // register q: token pair q / 2, word q % 2 (dim 16g + 8 (q % 2) + i)
        const int p = q >> 1, wi = q & 1;
        uint32_t y;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(y) : "r"(r[2 * p][wi]), "r"(r[2 * p + 1][wi]), "r"(sel));
        a[q] = u4pair_to_h2(y >> sh);
    }
}

// MQ: the general column mapping (several new tokens per sequence, causal among
// them, or padding columns); without it every row's G columns are the G query
// heads of one single-token decode, and the kernel keeps the plain addressing.
template <typename T, typename TKV, int D, int G, bool MQ, bool APP>
__global__ void __launch_bounds__(TcCfg<TKV, D, G>::THREADS, TcCfg<TKV, D, G>::MIN_CTAS)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const DecodeArgs a) {
    using C = TcCfg<TKV, D, G>;
    constexpr int NW = C::NW, S = C::S;
    constexpr bool SPLIT_P = sizeof(T) == 2 && !std::is_same<T, __half>::value;  // bf16: P = hi + lo
    constexpr bool kI8 = std::is_same<TKV, int8_t>::value;
    constexpr bool kI4 = C::I4;
    constexpr bool kQz = kI8 || kI4;  // quantised cache: per-(block, KV head) scales
    static_assert(!kQz || (std::is_same<T, __half>::value && (D == 128 || (kI8 && D == 256))),
                  "int8 caches: fp16 q, head_dim 128 or 256; 4-bit caches: fp16 q, head_dim 128");
    // APP (pa_decode_append): single-token rows of an fp16 / bf16 cache
    static_assert(!APP || (!MQ && !kQz), "the fused append takes single-token fp16 / bf16 rows");
    constexpr bool app = APP;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    int *stage_ok = reinterpret_cast<int *>(smem + C::OK_OFF);
    float *stage_sc = reinterpret_cast<float *>(smem + C::SC_OFF);
    int *cum = reinterpret_cast<int *>(smem + C::CUM_OFF);  // [B + 1] blocks before sequence b
    int *lens = cum + a.B + 1;                                // [B] effective lengths
    int *cumv = lens + a.B;                                   // [B + 1] virtual units before b

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = a.B, Hkv = a.Hkv;
    const int Hc = Hkv / a.ngroups;  // the cache's KV heads
    if (tid == 0) {  // bring the two tensor maps into the SM's descriptor cache before the first copy
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    // Without PA_DECODE_INPUTS_READY nothing is read before the previous kernel
    // on the stream has finished; with it, the lengths, the block tables and q
    // are read first (the caller guarantees that kernel does not write them) and
    // the wait comes just before the first cache tile is requested.
    if (!a.early) {
        pdl_wait();
        pdl_release_dependents();
    }

    // ---- effective lengths and blocks per sequence -> exclusive prefix sum cum[0..B] ----
    {
        __shared__ int wsum[NW];
        const int per = (B + C::THREADS - 1) / C::THREADS;
        const int lo = min(B, tid * per), hi = min(B, lo + per);
        __shared__ int wsumv[NW];
        const int gam = a.tc_chunk == 0 ? PA_TC_GAMMA : 0;
        int s = 0, sv = 0;
        for (int b = lo; b < hi; ++b) {
            const int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            lens[b] = L;
            const int nb = L > 0 ? (L + kBlockSize - 1) / kBlockSize : 0;
            s += nb;
            sv += nb > 0 ? (nb + gam) * Hkv : 0;
        }
        int x = s, xv = sv;  // inclusive warp scans
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o), yv = __shfl_up_sync(0xffffffffu, xv, o);
            if (lane >= o) {
                x += y;
                xv += yv;
            }
        }
        if (lane == 31) {
            wsum[warp] = x;
            wsumv[warp] = xv;
        }
        __syncthreads();
        int run = x - s, runv = xv - sv;
        for (int w = 0; w < warp; ++w) {
            run += wsum[w];
            runv += wsumv[w];
        }
        for (int b = lo; b < hi; ++b) {
            cum[b] = run;
            cumv[b] = runv;
            const int L = lens[b];
            const int nb = L > 0 ? (L + kBlockSize - 1) / kBlockSize : 0;
            run += nb;
            runv += nb > 0 ? (nb + gam) * Hkv : 0;
        }
        if (tid == C::THREADS - 1) {
            cum[B] = run;
            cumv[B] = runv;
        }
        __syncthreads();
    }
    // blocks of all rows: the host sends this family only streams below 2^31 blocks
    const int total = cum[B] * Hkv;
    const int gw = blockIdx.x * NW + warp;
    const int W = gridDim.x * NW;
    const bool rows_mode = a.tc_chunk < 0;
    // Columns: column j of row kvh is the (query token, head) pair jg = (kvh % ngroups) * G
    // + j of cache KV head kvh / ngroups; pairs from gcols on are padding.
    // Without MQ, column j of row kvh is query head kvh * G + j of a [B][Hq] q.
    auto col_jg = [&](int kvh, int j) { return (kvh % a.ngroups) * G + j; };
    auto ncol_of = [&](int kvh) { return MQ ? min(G, a.gcols - (kvh % a.ngroups) * G) : G; };
    auto col_row = [&](int b, int kvh, int j) -> size_t {  // row of q / out [B][qlen][Hq]
        if constexpr (!MQ) return (size_t)b * a.Hq + (size_t)kvh * G + j;
        const int jg = col_jg(kvh, j);
        const int i = jg / a.Greal, h = jg - i * a.Greal;
        return ((size_t)b * a.qlen + i) * a.Hq + (size_t)(kvh / a.ngroups) * a.Greal + h;
    };

    // Static schedule: by default one chunk of ceil(total / W) blocks (at least
    // kTcMinChunk) per warp, so every warp reads the same number of blocks;
    // partition_size > 0 fixes the chunk length instead.
    Chunks ck{total, cumv[B], 1, 0, a.tc_chunk == 0 ? PA_TC_GAMMA : 0, Hkv, cum, cumv, B};
    if (!rows_mode) {
        if (a.tc_chunk > 0) {
            ck.c = a.tc_chunk;
        } else {
            const int wc = min(W, kTcMaxChunks);
            const int c = (ck.vtotal + wc - 1) / wc;
            ck.c = c > kTcMinChunk ? c : kTcMinChunk;
        }
        ck.n = (ck.vtotal + ck.c - 1) / ck.c;
    }


    auto locate = [&](int f, Seg &sg) {
        int lo = 0, hi = B;  // largest b with cum[b] * Hkv <= f
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid] * Hkv <= f) lo = mid; else hi = mid;
        }
        sg.b = lo;
        sg.nb = cum[lo + 1] - cum[lo];
        const int off = f - cum[lo] * Hkv;
        sg.kvh = (int)(off / sg.nb);
        sg.j0 = off - sg.kvh * sg.nb;
        sg.fr = cum[lo] * Hkv + sg.kvh * sg.nb;
        sg.L = lens[lo];
    };

    // ---- range schedule: rows w, w+W, ... (one pass) or chunks w, w+W, ...
    auto set_range = [&](SegIter &it, int ch) {
        it.f = ck.start(ch);
        it.fend = ck.end(ch);
        it.ch = (int)ch;
    };
    auto range = [&](SegIter &it) -> bool {
        if (rows_mode) {
            for (;; ++it.k) {
                const int r = gw + it.k * W;
                if (r >= B * Hkv) return false;
                const int b = (int)(r / Hkv), kvh = (int)(r % Hkv);
                const int nb = cum[b + 1] - cum[b];
                if (nb > 0) {
                    it.f = cum[b] * Hkv + kvh * nb;
                    it.fend = it.f + nb;
                    it.ch = -1;
                    return true;
                }
            }
        }
        const int ch = gw + it.k * W;
        if (ch >= ck.n) return false;
        set_range(it, ch);
        return true;
    };
    auto next_seg = [&](SegIter &it, Seg &sg) -> bool {
        if (it.done) return false;
        if (it.f >= it.fend) {
            ++it.k;
            if (!range(it)) {
                it.done = true;
                return false;
            }
        }
        locate(it.f, sg);
        const int end = min(it.fend, sg.fr + sg.nb);
        sg.j1 = sg.j0 + (int)(end - it.f);
        sg.ch = it.ch;
        sg.ncol = ncol_of(sg.kvh);
        it.f = end;
        return true;
    };

    uint64_t *my_bars = bars + warp * S;
    const uint32_t qring = smem_addr(smem) + C::QRING_OFF + warp * S * C::QSLOT;
    int *my_ok = stage_ok + warp * S;
    const uint32_t ring = smem_addr(smem) + warp * S * C::STAGE;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // ---- producer: TMA for the warp's block stream, S blocks ahead of the consumer ----
    SegIter pit{0, 0, 0, -1, false};
    pit.done = !range(pit);
    auto win_first = [&](Win &w) {
        Seg sg;
        w.valid = next_seg(pit, sg);
        if (w.valid) {
            w.sg = sg;
            w.o = 0;
            w.n = min(32, sg.j1 - sg.j0);
            w.kc = sg.kvh / a.ngroups;
        }
    };
    auto win_after = [&](const Win &cur, Win &w) {
        if (!cur.valid) {
            w.valid = false;
            return;
        }
        const int len = cur.sg.j1 - cur.sg.j0;
        if (cur.o + 32 < len) {
            w = cur;
            w.o = cur.o + 32;
            w.n = min(32, len - w.o);
        } else {
            win_first(w);
        }
    };
    // lane l: the physical block of the window's entry l, loaded a window ahead
    // of its use and checked against the pool only when its copy is issued, so
    // that the table load never holds the warp (-1: no entry).  Quantised caches
    // also load the block's K and V scales, which need the block id at once: an
    // id outside the pool is marked -2 there.
    float p_ks = 0.f, p_vs = 0.f, p_ks_next = 0.f, p_vs_next = 0.f;
    // pa_decode_append: the lane holding a row's last block also loads the sequence's
    // new-token slot (as an int: this family's pools hold fewer than 2^31 slots, so a
    // larger slot is marked 2^31 - 1, outside the pool)
    int p_sn = -1, p_sn_next = -1;
    auto win_load = [&](const Win &w, float &ks, float &vs, int &sn) -> int {
        if (!w.valid || lane >= w.n) return -1;
        const int pb = a.tables[(size_t)w.sg.b * a.mbps + w.sg.j0 + w.o + lane];
        if (app && w.sg.j0 + w.o + lane == w.sg.nb - 1) {
            const long long s64 = a.slot_new[w.sg.b];
            sn = s64 > 0x7fffffffLL ? 0x7fffffff : (int)s64;
        }
        if constexpr (kQz) {
            if (pb < 0 || (int64_t)pb >= a.N) return -2;
            ks = a.ks[(size_t)pb * Hc + w.kc];
            vs = a.vs[(size_t)pb * Hc + w.kc];
        }
        return pb;
    };
    Win pc, pn;
    win_first(pc);
    win_after(pc, pn);
    int p_y = win_load(pc, p_ks, p_vs, p_sn), p_y_next = win_load(pn, p_ks_next, p_vs_next, p_sn_next);
    int p_i = 0, p_k = 0;
    float *my_sc = stage_sc + warp * S * 2;
    const uint32_t my_patch = smem_addr(smem) + C::PATCH_OFF + warp * S * C::PATCH;
    int *my_pslot = reinterpret_cast<int *>(smem + C::PSLOT_OFF) + warp * S;
    auto refill = [&]() {
        if (!pc.valid) return;
        const int pb = __shfl_sync(0xffffffffu, p_y, p_i);
        // TMA row of the block's tile for the cache's KV head, -1 for an id outside the pool
        const int y = (pb < 0 || (int64_t)pb >= a.N) ? -1 : (pb * Hc + pc.kc) * kBlockSize;
        float ksv = 0.f, vsv = 0.f;
        if constexpr (kQz) {
            ksv = __shfl_sync(0xffffffffu, p_ks, p_i);
            vsv = __shfl_sync(0xffffffffu, p_vs, p_i);
        }
        // pa_decode_append, a row's last block: the new token is patched into the staged
        // tile when its slot is the slot of the row's last decoded position (then the
        // append before the decode would have put it exactly there); the row's warp
        // writes it to its cache slot (one warp per cache KV head) in any case
        bool patch = false;
        int psn = -1;
        if (app && pc.sg.j0 + pc.o + p_i == pc.sg.nb - 1) {
            const int sn = __shfl_sync(0xffffffffu, p_sn, p_i);
            const bool inpool = sn >= 0 && (int64_t)sn < a.N * kBlockSize;
            patch = y >= 0 && sn == pb * kBlockSize + (pc.sg.L - 1) % kBlockSize;
            const bool writer = pc.sg.kvh % a.ngroups == 0;
            psn = inpool && writer ? sn : -1;
            if (lane == 0 && writer && sn >= 0 && !inpool) raise_flag(PA_EFLAG_BAD_SLOT);
        }
        if (lane == 0) {
            const int s = p_k % S;
            uint64_t *bar = &my_bars[s];
            // a segment's first block also brings the segment's q rows into the
            // stage's q slot (even when the block itself is skipped)
            const bool seg_first = pc.o == 0 && p_i == 0;
            const int ncol = seg_first ? pc.sg.ncol : 0;
            const bool fetch_new = patch || psn >= 0;
            const uint32_t tx = (y < 0 ? 0u : (uint32_t)C::STAGE) + (uint32_t)(ncol * D * (int)sizeof(T)) +
                                (fetch_new ? (uint32_t)C::PATCH : 0u);
            my_ok[s] = (y >= 0 ? 1 : 0) | (patch ? 2 : 0);
            if (app) my_pslot[s] = psn;
            if constexpr (kQz) {
                my_sc[2 * s] = ksv;  // released to the consumer by the arrive below
                my_sc[2 * s + 1] = vsv;
            }
            if (y < 0) raise_flag(PA_EFLAG_BAD_BLOCK);
            // the failure-path self-test leaves one stage's copies unissued, so that the
            // consumer's bounded wait for it runs out (never set in a normal call)
            const bool stall = gw == 0 && p_k == a.stall_at;
            // Relaxed arrival: a releasing one would first wait for this lane's
            // outstanding loads (the next window's table entries).  The stage's tiles
            // and q rows are published by the transaction count; the flag and scales
            // stored above reach the other lanes through the __syncwarp that every
            // consumer iteration runs before this stage is read again.
            if (tx == 0) {
                mbar_arrive_relaxed(bar);
            } else {
                mbar_arrive_expect_tx_relaxed(bar, tx);
            }
            if (y >= 0 && !stall) {
                const uint32_t dst = ring + s * C::STAGE;
#pragma unroll
                for (int bx = 0; bx < C::BOXES; ++bx) {
                    tma_load_2d(dst + bx * C::BOX_BYTES, &tmK, bx * C::BOXW, y, smem_addr(bar));
                    tma_load_2d(dst + C::TILE + bx * C::BOX_BYTES, &tmV, bx * C::BOXW, y, smem_addr(bar));
                }
            }
            if (fetch_new && !stall) {
                const size_t kh = (size_t)(pc.sg.kvh / a.ngroups) * D;
                const T *kn = reinterpret_cast<const T *>(a.k_new) + (size_t)pc.sg.b * a.kn_stride + kh;
                const T *vn = reinterpret_cast<const T *>(a.v_new) + (size_t)pc.sg.b * a.vn_stride + kh;
                bulk_g2s_u32(my_patch + s * C::PATCH, kn, D * 2, smem_addr(bar));
                bulk_g2s_u32(my_patch + s * C::PATCH + D * 2, vn, D * 2, smem_addr(bar));
            }
            if (stall) {
            } else if (!MQ && seg_first) {
                bulk_g2s_u32(qring + s * C::QSLOT, reinterpret_cast<const T *>(a.q) + col_row(pc.sg.b, pc.sg.kvh, 0) * D,
                             G * D * (int)sizeof(T), smem_addr(bar));
            } else if (seg_first) {
                // the segment's q rows: runs of columns that are consecutive heads of one
                // query token, each one bulk copy
                for (int j = 0; j < ncol;) {
                    const int h = col_jg(pc.sg.kvh, j) % a.Greal;
                    const int run = min(ncol - j, a.Greal - h);
                    const T *qsrc = reinterpret_cast<const T *>(a.q) + col_row(pc.sg.b, pc.sg.kvh, j) * D;
                    bulk_g2s_u32(qring + s * C::QSLOT + j * D * (int)sizeof(T), qsrc,
                                 run * D * (int)sizeof(T), smem_addr(bar));
                    j += run;
                }
            }
        }
        ++p_k;
        if (++p_i == pc.n) {
            p_i = 0;
            pc = pn;
            p_y = p_y_next;
            p_ks = p_ks_next;
            p_vs = p_vs_next;
            p_sn = p_sn_next;
            win_after(pc, pn);
            p_y_next = win_load(pn, p_ks_next, p_vs_next, p_sn_next);
        }
    };
    if (a.early) {
        pdl_wait();
        pdl_release_dependents();
    }
    // rows of sequences with no token produce zeros (and, for pa_decode_append, still
    // write their new token, if any, to its slot)
    for (int r = gw; r < B * Hkv; r += W) {
        const int b = r / Hkv;
        if (cum[b + 1] == cum[b]) {
            const int kvh = r % Hkv, ncol = ncol_of(kvh);
            for (int j = 0; j < ncol; ++j)
                for (int i = lane; i < D; i += 32) store_out<T>(a.out, a.out_f32, col_row(b, kvh, j) * D + i, 0.f);
            if (app && kvh % a.ngroups == 0) {
                const long long sn = a.slot_new[b];
                if (sn >= a.N * kBlockSize) {
                    if (lane == 0) raise_flag(PA_EFLAG_BAD_SLOT);
                } else if (sn >= 0) {
                    const int kc = kvh / a.ngroups;
                    const size_t drow = (((size_t)(sn / kBlockSize) * Hc + kc) * kBlockSize + sn % kBlockSize) * D;
                    for (int q = lane; q < D / 4; q += 32) {
                        const bool isv = q >= D / 8;
                        const int ch = isv ? q - D / 8 : q;
                        const T *src = reinterpret_cast<const T *>(isv ? a.v_new : a.k_new) +
                                       (size_t)b * (isv ? a.vn_stride : a.kn_stride) + (size_t)kc * D;
                        T *dst = reinterpret_cast<T *>(const_cast<void *>(isv ? a.vc : a.kc)) + drow;
                        reinterpret_cast<uint4 *>(dst)[ch] = reinterpret_cast<const uint4 *>(src)[ch];
                    }
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < S; ++i) refill();
    __syncwarp();

    // ---- consumer ------------------------------------------------------------------------
    const int g = lane >> 2, c = lane & 3;  // mma fragment coordinates
    // O^T row (m-tile i, row g; row g + 8 is dim + 8) -> head dim: m-tile i holds
    // dims 16i .. 16i + 15 for fp16/bf16 tiles; the int8 path gives thread row g
    // the 16 dims 16g .. 16g + 15 instead (see vfrag_i8)
    // (head_dim 256: m-tiles 8 .. 15 are the second 128-dim box, in the same order)
    auto dmap = [&](int i, int gg) -> int { return kQz ? (i >> 3) * 128 + 16 * gg + (i & 7) : 16 * i + gg; };
    const int h0 = 2 * c, h1 = 2 * c + 1;  // heads of this thread's S^T / O^T columns
    // B fragments of q (n = heads, k = dims) from the q slot of stage s.  The
    // int8 path orders the contraction's dims differently (see kfrag_i8): k-step
    // ks, thread column c covers dims 32c + 4ks .. 32c + 4ks + 3.
    auto load_q = [&](int s, uint32_t (&bq)[C::KSTEPS][2], int ncol) {
        const uint32_t qs = qring + s * C::QSLOT + (kQz ? (g * D + 32 * c) * 2 : (g * D + 2 * c) * 2);
        if constexpr (kI4) {
            // the 4-bit order (see kfrag_i4): k-step ks pairs dims 8w + t and 8w + t + 4
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS; ++ks) {
                const int w8 = 8 * (ks >> 1), t0 = 2 * (ks & 1);
                if (g < ncol) {
                    bq[ks][0] = lds_u16(qs + (w8 + t0) * 2) | (lds_u16(qs + (w8 + t0 + 4) * 2) << 16);
                    bq[ks][1] = lds_u16(qs + (w8 + t0 + 1) * 2) | (lds_u16(qs + (w8 + t0 + 5) * 2) << 16);
                } else {
                    bq[ks][0] = bq[ks][1] = 0u;
                }
            }
            return;
        }
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
            if (g < ncol) {
                // (int8 at head_dim 256: k-steps 8 .. 15 are dims 128 .. 255, in the same order)
                bq[ks][0] = lds_u32(qs + (kI8 ? (ks >> 3) * 256 + (ks & 7) * 8 : ks * 32));
                bq[ks][1] = lds_u32(qs + (kI8 ? (ks >> 3) * 256 + (ks & 7) * 8 + 4 : ks * 32 + 16));
            } else {
                bq[ks][0] = bq[ks][1] = 0u;
            }
        }
    };
    // per-lane ldmatrix offsets inside a stage (128-byte swizzle): K as the A
    // operand of S^T (chunk 2i + hi of row r), V^T as the A operand of O^T; the
    // box of k-step ks is ks / 4
    const int mi = lane >> 3, r8 = lane & 7;
    uint32_t koff[4], voff[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kr = r8 + ((mi & 1) << 3), kc = 2 * i + (mi >> 1);
        koff[i] = kr * 128 + (((kc & 7) ^ (kr & 7)) << 4);
        const int vr = r8 + ((mi >> 1) << 3), vc = 2 * i + (mi & 1);
        voff[i] = C::TILE + vr * 128 + (((vc & 7) ^ (vr & 7)) << 4);
    }

    SegIter cit{0, 0, 0, -1, false};
    cit.done = !range(cit);
    Seg cs;
    bool have = next_seg(cit, cs);
    uint32_t bq[C::KSTEPS][2];
    int c_k = 0;
    bool alive = true, drained = false;
    while (have) {
        const int len = cs.j1 - cs.j0;
        const int ntok_last = cs.L - (cs.nb - 1) * kBlockSize;  // tokens in the row's last block
        // causal limits: column (query token i) sees positions < L - qlen + 1 + i;
        // padding columns see none
        const int ncol = cs.ncol;
        const int lim0 = h0 < ncol ? cs.L - a.qlen + 1 + col_jg(cs.kvh, h0) / a.Greal : -1;
        const int lim1 = h1 < ncol ? cs.L - a.qlen + 1 + col_jg(cs.kvh, h1) / a.Greal : -1;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[C::MTILES][4];
#pragma unroll
        for (int i = 0; i < C::MTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

        for (int j = 0; alive && j < len; ++j) {
            if constexpr (kQz && PA_TC_PAIRS && D == 128) {
                if (j + 1 < len) {
                    // ---- two blocks (stages sA, sB) at once: one max/sum reduction and
                    // one rescale for both, two independent MMA streams
                    const int sA = c_k % S, sB = (c_k + 1) % S;
                    const bool okw = __all_sync(0xffffffffu, mbar_wait(&my_bars[sA], (c_k / S) & 1, a.wait_ns) &&
                                                                 mbar_wait(&my_bars[sB], ((c_k + 1) / S) & 1, a.wait_ns));
                    if (!okw) {
                        alive = false;
                        break;
                    }
                    if (j == 0) load_q(sA, bq, ncol);
                    // block j is not the row's last block (block j + 1 follows it)
                    const int ntokB = (cs.j0 + j + 1 == cs.nb - 1) ? ntok_last : kBlockSize;
                    const bool okA = my_ok[sA] != 0, okB = my_ok[sB] != 0;
                    if (okA || okB) {
                        const uint32_t tA = ring + sA * C::STAGE, tB = ring + sB * C::STAGE;
                        const float slA = a.scale_log2 * my_sc[2 * sA], slB = a.scale_log2 * my_sc[2 * sB];
                        const float vsA = my_sc[2 * sA + 1], vsB = my_sc[2 * sB + 1];
                        uint32_t kwA[kI8 ? 2 : 1][8], kwB[kI8 ? 2 : 1][8], vwA[kI8 ? 4 : 1][4], vwB[kI8 ? 4 : 1][4];
                        uint32_t k4A[kI4 ? 2 : 1][4], k4B[kI4 ? 2 : 1][4], v4A[kI4 ? 4 : 1][2], v4B[kI4 ? 4 : 1][2];
                        if constexpr (kI4) {
                            kload_i4(k4A, tA, g, c);
                            kload_i4(k4B, tB, g, c);
                            vload_i4(v4A, tA + C::TILE, g, c);
                            vload_i4(v4B, tB + C::TILE, g, c);
                        } else {
                            kload_i8(kwA, tA, g, c);
                            kload_i8(kwB, tB, g, c);
                            vload_i8(vwA, tA + C::TILE, g, c);
                            vload_i8(vwB, tB + C::TILE, g, c);
                        }
                        // ---- S^T of both blocks, NCH accumulator chains each (two where the
                        // general column mapping leaves too few registers for four)
                        constexpr int NCH = (MQ && kI8) ? 2 : 4;
                        float sa[2][NCH][4];
#pragma unroll
                        for (int u = 0; u < NCH; ++u)
#pragma unroll
                            for (int e = 0; e < 4; ++e) sa[0][u][e] = sa[1][u][e] = 0.f;
#pragma unroll
                        for (int ks = 0; ks < C::KSTEPS; ++ks) {
                            uint32_t fa[4], fb[4];
                            if constexpr (kI4) {
                                kfrag_i4(k4A, ks, fa);
                                kfrag_i4(k4B, ks, fb);
                            } else {
                                kfrag_i8(kwA, ks, fa);
                                kfrag_i8(kwB, ks, fb);
                            }
                            Mma<T>::mma(sa[0][ks % NCH], fa, bq[ks][0], bq[ks][1]);
                            Mma<T>::mma(sa[1][ks % NCH], fb, bq[ks][0], bq[ks][1]);
                        }
                        // ---- scores: block A is full, block B may end the row; a skipped
                        // block (id outside the pool) sees no token
                        float sp[2][4];
#pragma unroll
                        for (int bb = 0; bb < 2; ++bb) {
                            float sc[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                sc[e] = sa[bb][0][e] + sa[bb][1][e];
                                if constexpr (NCH == 4) sc[e] += sa[bb][2][e] + sa[bb][3][e];
                            }
                            const bool okb = bb ? okB : okA;
                            const float sl = bb ? slB : slA;
                            if constexpr (MQ) {
                                const int pos = (cs.j0 + j + bb) * kBlockSize + g;
                                sp[bb][0] = okb && pos < lim0 ? sc[0] * sl : -INFINITY;
                                sp[bb][1] = okb && pos < lim1 ? sc[1] * sl : -INFINITY;
                                sp[bb][2] = okb && pos + 8 < lim0 ? sc[2] * sl : -INFINITY;
                                sp[bb][3] = okb && pos + 8 < lim1 ? sc[3] * sl : -INFINITY;
                            } else {
                                const int nt = okb ? (bb ? ntokB : kBlockSize) : 0;
                                const bool v0 = g < nt, v1 = g + 8 < nt;
                                sp[bb][0] = v0 ? sc[0] * sl : -INFINITY;
                                sp[bb][1] = v0 ? sc[1] * sl : -INFINITY;
                                sp[bb][2] = v1 ? sc[2] * sl : -INFINITY;
                                sp[bb][3] = v1 ? sc[3] * sl : -INFINITY;
                            }
                        }
                        float mx0 = fmaxf(fmaxf(sp[0][0], sp[0][2]), fmaxf(sp[1][0], sp[1][2]));
                        float mx1 = fmaxf(fmaxf(sp[0][1], sp[0][3]), fmaxf(sp[1][1], sp[1][3]));
#pragma unroll
                        for (int msk = 4; msk < 32; msk <<= 1) {
                            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
                            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
                        }
                        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                        // as for one block: without MQ one of the two blocks holds a token of
                        // every column, so m is finite
                        const float mc0 = (MQ && mn0 == -INFINITY) ? 0.f : mn0;
                        const float mc1 = (MQ && mn1 == -INFINITY) ? 0.f : mn1;
                        const float al0 = (MQ && m0 == -INFINITY) ? 1.f : fast_exp2(m0 - mc0);
                        const float al1 = (MQ && m1 == -INFINITY) ? 1.f : fast_exp2(m1 - mc1);
                        float pp[2][4];
#pragma unroll
                        for (int bb = 0; bb < 2; ++bb) {
                            pp[bb][0] = fast_exp2(sp[bb][0] - mc0);
                            pp[bb][1] = fast_exp2(sp[bb][1] - mc1);
                            pp[bb][2] = fast_exp2(sp[bb][2] - mc0);
                            pp[bb][3] = fast_exp2(sp[bb][3] - mc1);
                        }
                        l0 = l0 * al0 + ((pp[0][0] + pp[0][2]) + (pp[1][0] + pp[1][2]));
                        l1 = l1 * al1 + ((pp[0][1] + pp[0][3]) + (pp[1][1] + pp[1][3]));
                        m0 = mn0;
                        m1 = mn1;
                        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                            for (int i = 0; i < C::MTILES; ++i) {
                                o[i][0] *= al0;
                                o[i][1] *= al1;
                                o[i][2] *= al0;
                                o[i][3] *= al1;
                            }
                        }
                        // ---- P^T fragments of both blocks, each carrying its block's V scale
                        const uint32_t pa0 = movm_t(Mma<T>::pack(pp[0][0] * vsA, pp[0][1] * vsA));
                        const uint32_t pa1 = movm_t(Mma<T>::pack(pp[0][2] * vsA, pp[0][3] * vsA));
                        const uint32_t pb0 = movm_t(Mma<T>::pack(pp[1][0] * vsB, pp[1][1] * vsB));
                        const uint32_t pb1 = movm_t(Mma<T>::pack(pp[1][2] * vsB, pp[1][3] * vsB));
                        // ---- O^T += V_A^T . P_A^T + V_B^T . P_B^T (no V mask: quantised slots
                        // past the end are finite and weighted 0)
#pragma unroll
                        for (int i = 0; i < C::MTILES; ++i) {
                            uint32_t fa[4], fb[4];
                            if constexpr (kI4) {
                                vfrag_i4(v4A, i, fa);
                                vfrag_i4(v4B, i, fb);
                            } else {
                                vfrag_i8(vwA, i, fa);
                                vfrag_i8(vwB, i, fb);
                            }
                            Mma<T>::mma(o[i], fa, pa0, pa1);
                            Mma<T>::mma(o[i], fb, pb0, pb1);
                        }
                    }
                    __syncwarp();
                    refill();
                    refill();
                    c_k += 2;
                            ++j;  // with the loop's own increment: two blocks
                    continue;
                }
            }
            const int s = c_k % S;
            const uint32_t parity = (c_k / S) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&my_bars[s], parity, a.wait_ns))) {
                alive = false;
                break;
            }
            if (j == 0) load_q(s, bq, ncol);  // the segment's q came with its first block
            const bool row_end = cs.j0 + j == cs.nb - 1;
            const int ntok = row_end ? ntok_last : kBlockSize;
            const uint32_t tK = ring + s * C::STAGE;
            if (app && row_end) {
                // pa_decode_append: the new token's K and V rows, staged with this block,
                // replace tile row ntok - 1 (its slot) and go to their cache slot
                const int okw = my_ok[s];
                const int psn = my_pslot[s];
                // a new token written elsewhere although this row's length counts it: the
                // slot is not its position's (rare: looked up only here)
                if (!(okw & 2) && psn >= 0 && lane == 0 && a.lens[cs.b] == cs.L) raise_flag(PA_EFLAG_APPEND_SLOT);
                if ((okw & 2) || psn >= 0) {
                    const int r = ntok - 1;
                    const int kc = cs.kvh / a.ngroups;
                    const size_t drow =
                        psn >= 0 ? (((size_t)(psn / kBlockSize) * Hc + kc) * kBlockSize + psn % kBlockSize) * D : 0;
                    for (int q = lane; q < D / 4; q += 32) {
                        const bool isv = q >= D / 8;
                        const int ch = isv ? q - D / 8 : q;  // 16-byte chunk of the row
                        uint32_t w4[4];
                        lds_v4(w4, my_patch + s * C::PATCH + q * 16);
                        if (okw & 2) {
                            const uint32_t dst = tK + (isv ? C::TILE : 0) + (ch >> 3) * C::BOX_BYTES + r * 128 +
                                                 (((ch & 7) ^ (r & 7)) << 4);
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w4[0]),
                                         "r"(w4[1]), "r"(w4[2]), "r"(w4[3])
                                         : "memory");
                        }
                        if (psn >= 0) {
                            T *cache = reinterpret_cast<T *>(const_cast<void *>(isv ? a.vc : a.kc)) + drow;
                            reinterpret_cast<uint4 *>(cache)[ch] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                    __syncwarp();
                }
            }
            if (my_ok[s] & 1) {
                // Slots past the sequence end hold stale data (in fp16/bf16 caches possibly
                // NaN/Inf); their probabilities are 0, and fp16/bf16 V values are masked
                // to 0 in the fragments so that they add exactly 0.  V^T fragment registers 0, 1
                // hold tokens 2c, 2c+1 and registers 2, 3 tokens 2c+8, 2c+9 (low half
                // = even token).
                const uint32_t vm_lo = (2 * c < ntok ? 0x0000ffffu : 0u) | (2 * c + 1 < ntok ? 0xffff0000u : 0u);
                const uint32_t vm_hi = (2 * c + 8 < ntok ? 0x0000ffffu : 0u) | (2 * c + 9 < ntok ? 0xffff0000u : 0u);
                // ---- fragments: K (A of S^T), then V^T (A of O^T), all issued up front
                // fragments of a head_dim-256 tile are loaded just before their MMAs (all
                // of them at once would take 128 more registers)
                constexpr bool kHoist = PA_TC_HOIST_V && !kQz && D <= 128;
                constexpr bool kHoistK = !kQz && D <= 128;
                uint32_t kf[kHoistK ? C::KSTEPS : 1][4], vf[kHoist ? C::MTILES : 1][4];
                uint32_t kw[kI8 ? 2 : 1][8], vw[kI8 ? 4 : 1][4];  // raw int8 words
                uint32_t kw4[kI4 ? 2 : 1][4], vw4[kI4 ? 4 : 1][2];  // raw 4-bit words
                float slog = a.scale_log2, vsc = 1.f;
                if constexpr (kI4) {
                    slog *= my_sc[2 * s];
                    vsc = my_sc[2 * s + 1];
                    kload_i4(kw4, tK, g, c);
                    vload_i4(vw4, tK + C::TILE, g, c);
                } else if constexpr (kI8) {
                    // int8 tiles (128-byte rows, 128-byte swizzle), converted exactly to fp16 in
                    // registers fragment by fragment; the block's K scale goes into the score
                    // scale, its V scale into the probabilities fed to P.V (the softmax sum
                    // keeps the unscaled ones)
                    slog *= my_sc[2 * s];
                    vsc = my_sc[2 * s + 1];
                    // (head_dim 256: the second box's words are read when its k-steps and
                    // m-tiles come up)
                    kload_i8(kw, tK, g, c);
                    vload_i8(vw, tK + C::TILE, g, c);
                } else if constexpr (kHoistK) {
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) ldsm_x4(kf[ks], tK + koff[ks & 3] + (ks >> 2) * C::BOX_BYTES);
                if constexpr (kHoist) {
#pragma unroll
                    for (int i = 0; i < C::MTILES; ++i) ldsm_x4_t(vf[i], tK + voff[i & 3] + (i >> 2) * C::BOX_BYTES);
#pragma unroll
                    for (int i = 0; i < C::MTILES; ++i) {
                        vf[i][0] &= vm_lo;
                        vf[i][1] &= vm_lo;
                        vf[i][2] &= vm_hi;
                        vf[i][3] &= vm_hi;
                    }
                }
                }
                // ---- S^T = K . Q^T, four independent accumulator chains
                float sa[4][4];
                // the first product of each chain starts from a zero accumulator
                auto qk = [&](int ks, const uint32_t (&f)[4]) {
                    if (ks < 4)
                        Mma<T>::mma0(sa[ks & 3], f, bq[ks][0], bq[ks][1]);
                    else
                        Mma<T>::mma(sa[ks & 3], f, bq[ks][0], bq[ks][1]);
                };
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) {
                    if constexpr (kI4) {
                        kfrag_i4(kw4, ks, kf[0]);
                        qk(ks, kf[0]);
                    } else if constexpr (kI8) {
                        if (C::BOXES > 1 && ks == 8) kload_i8(kw, tK + C::BOX_BYTES, g, c);
                        kfrag_i8(kw, ks & 7, kf[0]);
                        qk(ks, kf[0]);
                    } else if constexpr (kHoistK) {
                        qk(ks, kf[ks]);
                    } else {
                        ldsm_x4(kf[0], tK + koff[ks & 3] + (ks >> 2) * C::BOX_BYTES);
                        qk(ks, kf[0]);
                    }
                }
                float sc[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[e] = (sa[0][e] + sa[1][e]) + (sa[2][e] + sa[3][e]);
                // ---- online softmax (log2 domain): rows g, g+8 are tokens, columns heads
                float s0, s1, s2, s3;
                if constexpr (MQ) {
                    const int pos = (cs.j0 + j) * kBlockSize + g;  // token of rows g; g + 8 is pos + 8
                    s0 = pos < lim0 ? sc[0] * slog : -INFINITY;
                    s1 = pos < lim1 ? sc[1] * slog : -INFINITY;
                    s2 = pos + 8 < lim0 ? sc[2] * slog : -INFINITY;
                    s3 = pos + 8 < lim1 ? sc[3] * slog : -INFINITY;
                } else {
                    // every column sees the same tokens; padding columns (h >= G) hold
                    // zero q rows and score 0, which keeps them finite
                    const bool v0 = g < ntok, v1 = g + 8 < ntok;
                    s0 = v0 ? sc[0] * slog : -INFINITY;
                    s1 = v0 ? sc[1] * slog : -INFINITY;
                    s2 = v1 ? sc[2] * slog : -INFINITY;
                    s3 = v1 ? sc[3] * slog : -INFINITY;
                }
                float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
                for (int msk = 4; msk < 32; msk <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
                }
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                // A column with no visible token so far keeps m = -inf: its l and o are 0, so
                // it needs no rescale (al = 1, which also keeps padding columns from forcing
                // the rescale below), and its p are measured from 0 (exp2(-inf) = 0).
                // (Without MQ every column sees a token in every block, so m is finite.)
                const float mc0 = (MQ && mn0 == -INFINITY) ? 0.f : mn0;
                const float mc1 = (MQ && mn1 == -INFINITY) ? 0.f : mn1;
                const float al0 = (MQ && m0 == -INFINITY) ? 1.f : fast_exp2(m0 - mc0);
                const float al1 = (MQ && m1 == -INFINITY) ? 1.f : fast_exp2(m1 - mc1);
                const float p0 = fast_exp2(s0 - mc0), p1 = fast_exp2(s1 - mc1);
                const float p2 = fast_exp2(s2 - mc0), p3 = fast_exp2(s3 - mc1);
                l0 = l0 * al0 + (p0 + p2);
                l1 = l1 * al1 + (p1 + p3);
                m0 = mn0;
                m1 = mn1;
                if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                    for (int i = 0; i < C::MTILES; ++i) {
                        o[i][0] *= al0;
                        o[i][1] *= al1;
                        o[i][2] *= al0;
                        o[i][3] *= al1;
                    }
                }
                // ---- P^T fragments (k = tokens, n = heads): transpose the S^T layout
                const uint32_t ph01 = Mma<T>::pack(p0 * vsc, p1 * vsc), ph23 = Mma<T>::pack(p2 * vsc, p3 * vsc);
                const uint32_t pb0 = movm_t(ph01);  // tokens 0-7
                const uint32_t pb1 = movm_t(ph23);  // tokens 8-15
                uint32_t pl0 = 0, pl1 = 0;
                if constexpr (SPLIT_P) {
                    // bf16 keeps 8 significant bits; the remainder p - hi goes in a second
                    // bf16 operand so that P enters the product to ~16 bits
                    const float r0 = __uint_as_float(ph01 << 16), r1 = __uint_as_float(ph01 & 0xffff0000u);
                    const float r2 = __uint_as_float(ph23 << 16), r3 = __uint_as_float(ph23 & 0xffff0000u);
                    pl0 = movm_t(Mma<T>::pack(p0 * vsc - r0, p1 * vsc - r1));
                    pl1 = movm_t(Mma<T>::pack(p2 * vsc - r2, p3 * vsc - r3));
                }
                // ---- O^T += V^T . P^T
#pragma unroll
                for (int i = 0; i < C::MTILES; ++i) {
                    const int vi = kHoist ? i : 0;
                    if constexpr (kQz) {
                        if constexpr (kI4) {
                            vfrag_i4(vw4, i, vf[0]);
                        } else {
                            if (C::BOXES > 1 && i == 8) vload_i8(vw, tK + C::TILE + C::BOX_BYTES, g, c);
                            vfrag_i8(vw, i & 7, vf[0]);
                        }
                        // no mask: an int8 or 4-bit slot past the sequence end holds a finite
                        // value, and its probability is exactly 0
                    } else if constexpr (!kHoist) {
                        ldsm_x4_t(vf[vi], tK + voff[i & 3] + (i >> 2) * C::BOX_BYTES);
                        vf[vi][0] &= vm_lo;
                        vf[vi][1] &= vm_lo;
                        vf[vi][2] &= vm_hi;
                        vf[vi][3] &= vm_hi;
                    }
                    Mma<T>::mma(o[i], vf[vi], pb0, pb1);
                    if constexpr (SPLIT_P) Mma<T>::mma(o[i], vf[vi], pl0, pl1);
                }
            }
            __syncwarp();
            refill();
            ++c_k;
        }
        if (!alive) {
            // A copy did not land within the limit (PA_EFLAG_WAIT_TIMEOUT is raised).
            // First wait, bounded again, for the warp's copies still in flight, so that
            // none lands in shared memory after the warp has moved on or exited.  Then
            // this segment and every later one of the warp finish without data: a whole
            // row writes zeros, a partial writes an empty result (o = 0, lse = -inf,
            // weight 0 in the merge), so every slot the merge kernel reads is written.
            if (!drained) {
                if (lane == 0)
                    for (int k = c_k; k < p_k; ++k) mbar_wait(&my_bars[k % S], (k / S) & 1, a.wait_ns);
                __syncwarp();
                drained = true;
            }
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
#pragma unroll
            for (int i = 0; i < C::MTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        }

        // ---- finish the segment
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, msk);
            l1 += __shfl_xor_sync(0xffffffffu, l1, msk);
        }
        // l == 0 only when every block of the segment was skipped (bad table entries)
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
        if (cs.j0 == 0 && cs.j1 == cs.nb) {  // the whole row: final output
            const size_t out0 = col_row(cs.b, cs.kvh, h0) * D, out1 = col_row(cs.b, cs.kvh, h1) * D;
#pragma unroll
            for (int i = 0; i < C::MTILES; ++i) {
                const int d0 = dmap(i, g), d1 = d0 + 8;
                if (h0 < ncol) {
                    store_out<T>(a.out, a.out_f32, out0 + d0, o[i][0] * inv0);
                    store_out<T>(a.out, a.out_f32, out0 + d1, o[i][2] * inv0);
                }
                if (h1 < ncol) {
                    store_out<T>(a.out, a.out_f32, out1 + d0, o[i][1] * inv1);
                    store_out<T>(a.out, a.out_f32, out1 + d1, o[i][3] * inv1);
                }
            }
        } else {
            // Partial of a row cut by chunk boundaries: chunk ch holds at most two
            // partial segments, its first (slot 2ch) and its last (slot 2ch+1).
            const int ch_first = ck.of(cs.b, cs.kvh, cs.nb, 0);
            auto slot_of = [&](int ch) -> int {
                return (int)(2 * ch + ((ch == ch_first && ck.mid_start(cs.b, cs.kvh, cs.nb)) ? 1 : 0));
            };
            const int sl = slot_of(cs.ch);
#pragma unroll
            for (int i = 0; i < C::MTILES; ++i) {
                const int d0 = dmap(i, g), d1 = d0 + 8;
                if (h0 < G) {
                    float *w = a.ws_o + ((size_t)sl * G + h0) * D;
                    w[d0] = o[i][0] * inv0;
                    w[d1] = o[i][2] * inv0;
                }
                if (h1 < G) {
                    float *w = a.ws_o + ((size_t)sl * G + h1) * D;
                    w[d0] = o[i][1] * inv1;
                    w[d1] = o[i][3] * inv1;
                }
            }
            if (g == 0) {
                if (h0 < G) a.ws_lse[(size_t)sl * G + h0] = m0 + log2f(l0);
                if (h1 < G) a.ws_lse[(size_t)sl * G + h1] = m1 + log2f(l1);
            }
        }
        have = next_seg(cit, cs);
    }
}

// ---------------------------------------------------------------------------
// log-sum-exp merge of the rows the decode kernel cut into partial segments
// ---------------------------------------------------------------------------
// Launched right after decode_tc_kernel (programmatic dependent launch): the
// prologue (effective lengths, blocks per sequence, their prefix sum) runs
// while the decode kernel finishes; then every warp takes (row, column) items
// whose row the decode's schedule cut into several segments and merges
//   out = sum_i 2^(lse_i - M) o_i / sum_i 2^(lse_i - M),  M = max_i lse_i
// over the row's segments i (lse in the log2 domain), all of the row's partial
// loads issued before their use.  Rows that one segment covered were written
// by the decode kernel and are skipped.
template <typename T, int D, int G, bool MQ>
__global__ void __launch_bounds__(256) merge_tc_kernel(const DecodeArgs a) {
    constexpr int NWM = 8, DPL = D / 32;
    extern __shared__ int mcum[];  // [B + 1] blocks, then [B + 1] virtual units
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = a.B, Hkv = a.Hkv;
    {
        __shared__ int wsum[NWM];
        const int per = (B + NWM * 32 - 1) / (NWM * 32);
        const int lo = min(B, tid * per), hi = min(B, lo + per);
        __shared__ int wsumv[NWM];
        const int gam = a.tc_chunk == 0 ? PA_TC_GAMMA : 0;
        int s = 0, sv = 0;
        for (int b = lo; b < hi; ++b) {
            const int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            const int nb = L > 0 ? (L + kBlockSize - 1) / kBlockSize : 0;
            s += nb;
            sv += nb > 0 ? (nb + gam) * Hkv : 0;
        }
        int x = s, xv = sv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o), yv = __shfl_up_sync(0xffffffffu, xv, o);
            if (lane >= o) {
                x += y;
                xv += yv;
            }
        }
        if (lane == 31) {
            wsum[warp] = x;
            wsumv[warp] = xv;
        }
        __syncthreads();
        int run = x - s, runv = xv - sv;
        for (int w = 0; w < warp; ++w) {
            run += wsum[w];
            runv += wsumv[w];
        }
        for (int b = lo; b < hi; ++b) {
            mcum[b] = run;
            mcum[B + 1 + b] = runv;
            const int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            const int nb = L > 0 ? (L + kBlockSize - 1) / kBlockSize : 0;
            run += nb;
            runv += nb > 0 ? (nb + gam) * Hkv : 0;
        }
        if (tid == NWM * 32 - 1) {
            mcum[B] = run;
            mcum[2 * B + 1] = runv;
        }
        __syncthreads();
    }
    // the decode kernel's chunks (same rule, same numbers)
    const int total = mcum[B] * Hkv;
    Chunks ck{total, mcum[2 * B + 1], 1, 0, a.tc_chunk == 0 ? PA_TC_GAMMA : 0, Hkv, mcum, mcum + B + 1, B};
    if (a.tc_chunk > 0) {
        ck.c = a.tc_chunk;
    } else {
        const int wc = min(a.tc_W, kTcMaxChunks);
        const int c = (ck.vtotal + wc - 1) / wc;
        ck.c = c > kTcMinChunk ? c : kTcMinChunk;
    }
    ck.n = (ck.vtotal + ck.c - 1) / ck.c;
    pdl_wait();  // the decode kernel's partial results
    pdl_release_dependents();
    const int items = B * Hkv * G;
    for (int it = blockIdx.x * NWM + warp; it < items; it += gridDim.x * NWM) {
        const int r = it / G, h = it - r * G;
        const int b = r / Hkv, kvh = r - b * Hkv;
        const int nb = mcum[b + 1] - mcum[b];
        if (nb == 0) continue;
        const int fr = mcum[b] * Hkv + kvh * nb;
        const int ch_first = ck.of(b, kvh, nb, 0), ch_last = ck.of(b, kvh, nb, nb - 1);
        if (ch_first == ch_last) continue;  // written by the decode kernel
        const int ncol = MQ ? min(G, a.gcols - (kvh % a.ngroups) * G) : G;
        if (h >= ncol) continue;
        const int nseg = ch_last - ch_first + 1;
        auto slot_of = [&](int i) -> int {
            const int ch = ch_first + i;
            return 2 * ch + ((i == 0 && ck.mid_start(b, kvh, nb)) ? 1 : 0);
        };
        // weights: lane i holds segment i's lse (32 segments per round)
        constexpr int NBM = DPL >= 8 ? 4 : 8;  // segments per round, loads issued together
        // The first round's partial outputs do not depend on the weights: they are
        // loaded together with the lse values, so a row of up to NBM segments costs one
        // round trip.  Lane i holds segment i's lse (32 per round).
        float v[NBM][DPL];
#pragma unroll
        for (int j = 0; j < NBM; ++j) {
            if (j < nseg) {
                // DPL = 2, 4 or 8 consecutive floats of this lane, naturally aligned
                const typename FVec<DPL>::type x = FVec<DPL>::ld(a.ws_o + ((size_t)slot_of(j) * G + h) * D + lane * DPL);
#pragma unroll
                for (int e = 0; e < DPL; ++e) v[j][e] = FVec<DPL>::get(x, e);
            }
        }
        const float x0 = lane < nseg ? __ldcg(a.ws_lse + (size_t)slot_of(lane) * G + h) : -INFINITY;
        float mx = x0, sm = x0 == -INFINITY ? 0.f : 1.f;
        for (int i0 = 32; i0 < nseg; i0 += 32) {
            const float x = i0 + lane < nseg ? __ldcg(a.ws_lse + (size_t)slot_of(i0 + lane) * G + h) : -INFINITY;
            const float mn = fmaxf(mx, x);
            sm = (mx == -INFINITY ? 0.f : sm * fast_exp2(mx - mn)) + (x == -INFINITY ? 0.f : fast_exp2(x - mn));
            mx = mn;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, mx, o), so = __shfl_xor_sync(0xffffffffu, sm, o);
            const float mn = fmaxf(mx, mo);
            sm = (mx == -INFINITY ? 0.f : sm * fast_exp2(mx - mn)) + (mo == -INFINITY ? 0.f : so * fast_exp2(mo - mn));
            mx = mn;
        }
        const float inv = sm > 0.f ? 1.f / sm : 0.f;
        const float w0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - mx) * inv;  // weight of segment lane
        float acc[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
        for (int i0 = 0; i0 < nseg; i0 += NBM) {
            float wl = 0.f;
            if (i0 > 0) {
#pragma unroll
                for (int j = 0; j < NBM; ++j) {
                    if (i0 + j < nseg) {
                        const typename FVec<DPL>::type x =
                            FVec<DPL>::ld(a.ws_o + ((size_t)slot_of(i0 + j) * G + h) * D + lane * DPL);
#pragma unroll
                        for (int e = 0; e < DPL; ++e) v[j][e] = FVec<DPL>::get(x, e);
                    }
                }
                // segments past the first 32: their weights from their lse, lane j < NBM
                if (i0 >= 32 && lane < NBM && i0 + lane < nseg) {
                    const float x = __ldcg(a.ws_lse + (size_t)slot_of(i0 + lane) * G + h);
                    wl = x == -INFINITY ? 0.f : fast_exp2(x - mx) * inv;
                }
            }
#pragma unroll
            for (int j = 0; j < NBM; ++j) {
                const float w = i0 < 32 ? __shfl_sync(0xffffffffu, w0, i0 + j) : __shfl_sync(0xffffffffu, wl, j);
                if (i0 + j < nseg) {
#pragma unroll
                    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, v[j][e], acc[e]);
                }
            }
        }
        // output row of column h
        size_t orow;
        if constexpr (!MQ) {
            orow = (size_t)b * a.Hq + (size_t)kvh * G + h;
        } else {
            const int jg = (kvh % a.ngroups) * G + h;
            const int qi = jg / a.Greal, hh = jg - qi * a.Greal;
            orow = ((size_t)b * a.qlen + qi) * a.Hq + (size_t)(kvh / a.ngroups) * a.Greal + hh;
        }
#pragma unroll
        for (int e = 0; e < DPL; ++e) store_out<T>(a.out, a.out_f32, orow * D + lane * DPL + e, acc[e]);
    }
}

// ---------------------------------------------------------------------------
// CTA-cooperative decode for groups of 16, 32 or 64 query heads per KV head
// ---------------------------------------------------------------------------
// With G = 16 * NG query heads per cache KV head (MQA-like groups) the group is
// wide enough to fill the M side of the MMA, so the contraction is laid out the
// other way round from decode_tc_kernel, with the heads as rows:
//   S[16 heads x 16 tokens]  = Q[16 x d] . K^T[d x 16]   (A = q, kept in registers
//                                                          for the whole segment)
//   O[16 heads x d]         += P[16 x 16] . V[16 x d]     (A = P, taken straight from
//                                                          the S accumulators)
// so one ldmatrix of K or V feeds 16 heads and P needs no transpose.  One CTA of
// NG warps takes each cache row once: its tiles go through one ring of S shared
// stages, warp w computes the 16 heads 16w .. 16w + 15, and only lane 0 of warp 0
// issues copies.  A stage is refilled once all NG warps have released it (an
// mbarrier with NG arrivals); with NG > 1 warp 0 refills the stage of block k - 1
// right after its own block k (a warp that lags by one block does not hold it
// up), so the ring runs S - 1 blocks ahead of it.  Chunks of the cache-row stream
// go to CTAs (not warps); cut rows leave partial results for merge_tc_kernel,
// with GC = 16 NG columns per cache row.
//
// The running maximum moves only when a block's scores exceed it by more than
// kLazyMax (in log2 units): until then the probabilities are taken against the
// old maximum (at most 2^kLazyMax, exact in fp32 and rounded to the same
// relative precision in fp16/bf16), and O and l need no rescale.  The result
// is the same softmax: numerator and denominator share the reference point.
template <typename T, int D, int NG>
struct CoopCfg {
    static constexpr int NW = NG;
    static constexpr int THREADS = NW * 32;
    // ten to twelve warps per SM (O, 64 registers at d = 128, stays in registers; q is
    // read from shared memory)
    static constexpr int MIN_CTAS = NG == 1 ? 10 : (NG == 2 ? 6 : 3);
    static constexpr int BOXW = 128 / (int)sizeof(T);
    static constexpr int BOXES = D / BOXW;
    static constexpr int BOX_BYTES = 16 * 128;
    static constexpr int TILE = BOXES * BOX_BYTES;
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING_BYTES = NG == 1 ? 16 * 1024 : (NG == 2 ? 24 * 1024 : 48 * 1024);
    static constexpr int S = RING_BYTES / STAGE;
    static constexpr int LAG = NG == 1 ? 0 : 1;  // blocks the refill trails the consumer by
    static constexpr int KSTEPS = D / 16, NT = D / 8;
    static constexpr int QSLOT = 16 * D * 2;            // a warp's 16 q rows (16-byte chunks swizzled)
    static constexpr int Q_OFF = S * STAGE;
    static constexpr int BAR_OFF = Q_OFF + NW * QSLOT;  // full[S], then empty[S]
    static constexpr int OK_OFF = BAR_OFF + 2 * S * 8;  // int [S]: the stage's block is in the pool
    static constexpr int CUM_OFF = OK_OFF + S * 4;
    static int smem_bytes(int B) { return 1024 + CUM_OFF + (3 * B + 3) * 4; }
};
constexpr float kLazyMax = 8.f;

template <typename T, int D, int NG>
__global__ void __launch_bounds__(CoopCfg<T, D, NG>::THREADS, CoopCfg<T, D, NG>::MIN_CTAS)
    decode_coop_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeArgs a) {
    using C = CoopCfg<T, D, NG>;
    constexpr int S = C::S, GC = NG * 16;
    constexpr bool SPLIT_P = !std::is_same<T, __half>::value;  // bf16: P = hi + lo
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + S;
    int *stage_ok = reinterpret_cast<int *>(smem + C::OK_OFF);
    int *cum = reinterpret_cast<int *>(smem + C::CUM_OFF);  // [B + 1]
    int *lens = cum + a.B + 1;                                // [B]
    int *cumv = lens + a.B;                                   // [B + 1]
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = a.B, Hc = a.Hkv;  // the launcher passes the cache's KV heads
    if (tid == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        abort_flag = 0;
    }
    if (!a.early) {
        pdl_wait();
        pdl_release_dependents();
    }
    const int gam = a.tc_chunk == 0 ? PA_TC_GAMMA : 0;
    {
        __shared__ int wsum[NG], wsumv[NG];
        const int per = (B + C::THREADS - 1) / C::THREADS;
        const int lo = min(B, tid * per), hi = min(B, lo + per);
        int s = 0, sv = 0;
        for (int b = lo; b < hi; ++b) {
            const int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            lens[b] = L;
            const int nb = L > 0 ? (L + kBlockSize - 1) / kBlockSize : 0;
            s += nb;
            sv += nb > 0 ? (nb + gam) * Hc : 0;
        }
        int x = s, xv = sv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o), yv = __shfl_up_sync(0xffffffffu, xv, o);
            if (lane >= o) {
                x += y;
                xv += yv;
            }
        }
        if (lane == 31) {
            wsum[warp] = x;
            wsumv[warp] = xv;
        }
        __syncthreads();
        int run = x - s, runv = xv - sv;
        for (int w = 0; w < warp; ++w) {
            run += wsum[w];
            runv += wsumv[w];
        }
        for (int b = lo; b < hi; ++b) {
            cum[b] = run;
            cumv[b] = runv;
            const int nb = lens[b] > 0 ? (lens[b] + kBlockSize - 1) / kBlockSize : 0;
            run += nb;
            runv += nb > 0 ? (nb + gam) * Hc : 0;
        }
        if (tid == C::THREADS - 1) {
            cum[B] = run;
            cumv[B] = runv;
        }
        if (tid == 0) {
            for (int s2 = 0; s2 < S; ++s2) {
                mbar_init(&full[s2], 1);
                mbar_init(&empty[s2], NG);
            }
            fence_mbar_init();
        }
        __syncthreads();
    }
    const int total = cum[B] * Hc;
    Chunks ck{total, cumv[B], 1, 0, gam, Hc, cum, cumv, B};
    {
        if (a.tc_chunk > 0) {
            ck.c = a.tc_chunk;
        } else {
            const int wc = min((int)gridDim.x, kTcMaxChunks);
            const int c = (ck.vtotal + wc - 1) / wc;
            ck.c = c > kTcMinChunk ? c : kTcMinChunk;
        }
        ck.n = (ck.vtotal + ck.c - 1) / ck.c;
    }
    auto locate = [&](int f, Seg &sg) {
        int lo = 0, hi = B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid] * Hc <= f) lo = mid; else hi = mid;
        }
        sg.b = lo;
        sg.nb = cum[lo + 1] - cum[lo];
        const int off = f - cum[lo] * Hc;
        sg.kvh = off / sg.nb;
        sg.j0 = off - sg.kvh * sg.nb;
        sg.fr = cum[lo] * Hc + sg.kvh * sg.nb;
        sg.L = lens[lo];
    };
    auto range = [&](SegIter &it) -> bool {
        const int ch = blockIdx.x + it.k * gridDim.x;
        if (ch >= ck.n) return false;
        it.f = ck.start(ch);
        it.fend = ck.end(ch);
        it.ch = ch;
        return true;
    };
    auto next_seg = [&](SegIter &it, Seg &sg) -> bool {
        if (it.done) return false;
        while (it.f >= it.fend) {
            ++it.k;
            if (!range(it)) {
                it.done = true;
                return false;
            }
        }
        locate(it.f, sg);
        const int end = min(it.fend, sg.fr + sg.nb);
        sg.j1 = sg.j0 + (end - it.f);
        sg.ch = it.ch;
        sg.ncol = GC;
        it.f = end;
        return true;
    };

    // ---- producer (warp 0): the CTA's block stream, table entries a window ahead ----
    SegIter pit{0, 0, 0, -1, false};
    Win pc{}, pn{};
    int p_y = -1, p_y_next = -1, p_i = 0, p_k = 0;
    int p_s = 0;         // stage of block p_k (p_k % S)
    uint32_t p_ph = 0;   // (p_k / S) & 1
    bool p_alive = true;
    auto win_first = [&](Win &w) {
        Seg sg;
        w.valid = next_seg(pit, sg);
        if (w.valid) {
            w.sg = sg;
            w.o = 0;
            w.n = min(32, sg.j1 - sg.j0);
            w.kc = sg.kvh;
        }
    };
    auto win_after = [&](const Win &cur, Win &w) {
        if (!cur.valid) {
            w.valid = false;
            return;
        }
        const int len = cur.sg.j1 - cur.sg.j0;
        if (cur.o + 32 < len) {
            w = cur;
            w.o = cur.o + 32;
            w.n = min(32, len - w.o);
        } else {
            win_first(w);
        }
    };
    auto win_load = [&](const Win &w) -> int {
        if (!w.valid || lane >= w.n) return -1;
        return a.tables[(size_t)w.sg.b * a.mbps + w.sg.j0 + w.o + lane];
    };
    // issue the copy of the next block of the stream into its stage (warp 0, all lanes)
    auto refill = [&]() {
        if (!pc.valid || !p_alive) return;
        const int s = p_s;
        if (p_k >= S) {  // the stage's previous block must be released by every warp
            int ok = lane == 0 ? (int)mbar_wait(&empty[s], p_ph ^ 1u, a.wait_ns) : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                p_alive = false;
                if (lane == 0) atomicExch(&abort_flag, 1);
                return;
            }
        }
        const int pb = __shfl_sync(0xffffffffu, p_y, p_i);
        const int y = (pb < 0 || (int64_t)pb >= a.N) ? -1 : (pb * Hc + pc.kc) * kBlockSize;
        if (lane == 0) {
            stage_ok[s] = y >= 0;
            if (y < 0) raise_flag(PA_EFLAG_BAD_BLOCK);
            const bool stall = p_k == a.stall_at && blockIdx.x == 0;
            // a releasing arrival: stage_ok is read by the other warps after their wait
            if (y < 0) {
                mbar_arrive(&full[s]);
            } else {
                mbar_arrive_expect_tx(&full[s], (uint32_t)C::STAGE);
                if (!stall) {
                    const uint32_t dst = smem_addr(smem) + s * C::STAGE;
#pragma unroll
                    for (int bx = 0; bx < C::BOXES; ++bx) {
                        tma_load_2d(dst + bx * C::BOX_BYTES, &tmK, bx * C::BOXW, y, smem_addr(&full[s]));
                        tma_load_2d(dst + C::TILE + bx * C::BOX_BYTES, &tmV, bx * C::BOXW, y, smem_addr(&full[s]));
                    }
                }
            }
        }
        ++p_k;
        if (++p_s == S) {
            p_s = 0;
            p_ph ^= 1u;
        }
        if (++p_i == pc.n) {
            p_i = 0;
            pc = pn;
            p_y = p_y_next;
            win_after(pc, pn);
            p_y_next = win_load(pn);
        }
    };
    if (warp == 0) {
        pit.done = !range(pit);
        win_first(pc);
        win_after(pc, pn);
        p_y = win_load(pc);
        p_y_next = win_load(pn);
    }
    if (a.early) {
        pdl_wait();
        pdl_release_dependents();
    }
    // rows of sequences with no token produce zeros
    for (int r = blockIdx.x * NG + warp; r < B * Hc; r += gridDim.x * NG) {
        const int b = r / Hc;
        if (cum[b + 1] == cum[b]) {
            const int kvh = r % Hc;
            for (int j = 0; j < GC; ++j)
                for (int i = lane; i < D; i += 32)
                    store_out<T>(a.out, a.out_f32, ((size_t)b * a.Hq + (size_t)kvh * GC + j) * D + i, 0.f);
        }
    }
    if (warp == 0)
        for (int i = 0; i < S; ++i) refill();

    // ---- consumers: every warp, heads 16 warp .. 16 warp + 15 of each row ----
    // Fragment coordinates: thread (g, c) holds rows (heads) g and g + 8 and
    // columns 2c, 2c + 1 (+ 8) of every 16 x 16 / 16 x 8 tile.
    const int g = lane >> 2, c = lane & 3;
    // ldmatrix lane addresses (128-byte swizzle): matrix mi = lane / 8 is token
    // rows 8 (mi >> 1) .. + 7 and the 16-byte chunk 2i + (mi & 1) of the row.
    // Non-transposed on K this gives the B fragments of S for both 8-token halves
    // of k-step i; transposed on V, those of O for dims 16i .. 16i + 15.
    const int mi = lane >> 3, r8 = lane & 7;
    uint32_t moff[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r8 + ((mi >> 1) << 3), ch = 2 * i + (mi & 1);
        moff[i] = r * 128 + (((ch & 7) ^ (r & 7)) << 4);
    }
    // q rows in the warp's slot: row r, 16-byte chunk ch at r * 2D + ((ch ^ (r & 7)) << 4), so
    // that the ldmatrix of 8 rows at one chunk hits 8 different bank groups; A fragment of
    // k-step ks: matrix mi = lane / 8 is rows 8 (mi & 1) .. + 7, chunk 2 ks + (mi >> 1)
    const uint32_t qslot = smem_addr(smem) + C::Q_OFF + warp * C::QSLOT;
    const int qr = r8 + ((mi & 1) << 3);
    auto qaddr = [&](int ks) -> uint32_t { return qslot + qr * (2 * D) + (((2 * ks + (mi >> 1)) ^ (qr & 7)) << 4); };
    SegIter cit{0, 0, 0, -1, false};
    cit.done = !range(cit);
    Seg cs;
    bool have = next_seg(cit, cs);
    int c_k = 0, c_s = 0;  // blocks consumed; stage of block c_k
    uint32_t c_ph = 0;     // (c_k / S) & 1
    bool alive = true;
    const int row0 = warp * 16;  // this warp's first column (head) of the row
    // Scores stay unscaled: p = 2^((s - m) |scale| log2 e) with m the (lazy) maximum of
    // the unscaled scores, kLazyMax of slack in log2 units being lazy_raw unscaled.
    // (a zero scale is taken as 1e-30: every probability 1 to within 1e-26 relative,
    // and the slots past a row's end still weigh exactly 0)
    const float sl = fmaxf(fabsf(a.scale_log2), 1e-30f);
    const float lazy_raw = kLazyMax / sl;
    while (have) {
        const int len = cs.j1 - cs.j0;
        const int ntok_last = cs.L - (cs.nb - 1) * kBlockSize;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads g, g + 8
        float o[C::NT][4];
#pragma unroll
        for (int i = 0; i < C::NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        if (alive) {
            // the segment's q rows (heads row0 .. row0 + 15, consecutive in q) into the slot
            const uint4 *qg = reinterpret_cast<const uint4 *>(a.q) +
                              ((size_t)cs.b * a.Hq + (size_t)cs.kvh * GC + row0) * (D / 8);
            __syncwarp();  // the previous segment's fragment reads are done
            // a negative scale goes into q (sign bits flipped, exact), so that the scores
            // below are scaled by |scale| and their maximum is taken before scaling
            const uint32_t sflip = a.scale_log2 < 0.f ? 0x80008000u : 0u;
#pragma unroll
            for (int i = 0; i < 16 * D / 8 / 32; ++i) {
                const int id = i * 32 + lane, r = id / (D / 8), ch = id % (D / 8);
                uint4 v = __ldg(qg + id);
                v.x ^= sflip;
                v.y ^= sflip;
                v.z ^= sflip;
                v.w ^= sflip;
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(qslot + r * (2 * D) + ((ch ^ (r & 7)) << 4)),
                             "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                             : "memory");
            }
            __syncwarp();
        }
        for (int j = 0; alive && j < len; ++j) {
            const int s = c_s;
            const uint32_t parity = c_ph;
            // every lane polls the stage's barrier; the CTA's abort flag (the producer gave
            // up) is looked at every 16 blocks and after a failed wait
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], parity, a.wait_ns));
            if (!ok || ((c_k & 15) == 15 && *reinterpret_cast<volatile int *>(&abort_flag))) {
                if (lane == 0) atomicExch(&abort_flag, 1);
                alive = false;
                break;
            }
            const int ntok = (cs.j0 + j == cs.nb - 1) ? ntok_last : kBlockSize;
            const uint32_t tK = smem_addr(smem) + s * C::STAGE, tV = tK + C::TILE;
            if (stage_ok[s]) {
                // ---- S = Q . K^T: n-tiles of tokens 0-7 and 8-15, two chains each
                float sa[2][2][4];
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) {
                    uint32_t kb[4], qa[4];
                    ldsm_x4(qa, qaddr(ks));
                    ldsm_x4(kb, tK + moff[ks & 3] + (ks >> 2) * C::BOX_BYTES);
                    if (ks < 2) {
                        Mma<T>::mma0(sa[0][ks & 1], qa, kb[0], kb[1]);
                        Mma<T>::mma0(sa[1][ks & 1], qa, kb[2], kb[3]);
                    } else {
                        Mma<T>::mma(sa[0][ks & 1], qa, kb[0], kb[1]);
                        Mma<T>::mma(sa[1][ks & 1], qa, kb[2], kb[3]);
                    }
                }
                // x[nt][e]: head g (e < 2) or g + 8, token 8 nt + 2c + (e & 1), unscaled
                float x[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[nt][e] = sa[nt][0][e] + sa[nt][1][e];
                if (ntok < kBlockSize) {  // the row's last block: slots past the end see nothing
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (8 * nt + 2 * c + (e & 1) >= ntok) x[nt][e] = -INFINITY;
                }
                float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
                float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                // move the reference point only when a score exceeds it by more than
                // kLazyMax (always on the segment's first block: m = -inf)
                if (__any_sync(0xffffffffu, mx0 > m0 + lazy_raw || mx1 > m1 + lazy_raw)) {
                    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                    const float al0 = fast_exp2((m0 - mn0) * sl), al1 = fast_exp2((m1 - mn1) * sl);
                    l0 *= al0;
                    l1 *= al1;
#pragma unroll
                    for (int i = 0; i < C::NT; ++i) {
                        o[i][0] *= al0;
                        o[i][1] *= al0;
                        o[i][2] *= al1;
                        o[i][3] *= al1;
                    }
                    m0 = mn0;
                    m1 = mn1;
                }
                float p[2][4];
                const float ms0 = m0 * sl, ms1 = m1 * sl;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    p[nt][0] = fast_exp2(fmaf(x[nt][0], sl, -ms0));
                    p[nt][1] = fast_exp2(fmaf(x[nt][1], sl, -ms0));
                    p[nt][2] = fast_exp2(fmaf(x[nt][2], sl, -ms1));
                    p[nt][3] = fast_exp2(fmaf(x[nt][3], sl, -ms1));
                }
                l0 += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
                l1 += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
                // ---- A fragments of P (rows heads, k = tokens) straight from S's layout
                uint32_t pa[4], pl[4];
                pa[0] = Mma<T>::pack(p[0][0], p[0][1]);
                pa[1] = Mma<T>::pack(p[0][2], p[0][3]);
                pa[2] = Mma<T>::pack(p[1][0], p[1][1]);
                pa[3] = Mma<T>::pack(p[1][2], p[1][3]);
                if constexpr (SPLIT_P) {
                    // bf16 keeps 8 significant bits: the remainder goes in a second operand
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float hi0 = __uint_as_float(pa[r] << 16), hi1 = __uint_as_float(pa[r] & 0xffff0000u);
                        pl[r] = Mma<T>::pack(p[r >> 1][2 * (r & 1)] - hi0, p[r >> 1][2 * (r & 1) + 1] - hi1);
                    }
                }
                // ---- O += P . V, V fragments masked on the row's last block (stale slots
                // may hold NaN or Inf; registers 0/1 hold tokens 2c, 2c + 1, 2/3 tokens + 8)
                const uint32_t vm_lo = ntok < kBlockSize ? (2 * c < ntok ? 0x0000ffffu : 0u) |
                                                               (2 * c + 1 < ntok ? 0xffff0000u : 0u)
                                                         : 0xffffffffu;
                const uint32_t vm_hi = ntok < kBlockSize ? (2 * c + 8 < ntok ? 0x0000ffffu : 0u) |
                                                               (2 * c + 9 < ntok ? 0xffff0000u : 0u)
                                                         : 0xffffffffu;
#pragma unroll
                for (int i = 0; i < C::KSTEPS; ++i) {
                    uint32_t vb[4];
                    ldsm_x4_t(vb, tV + moff[i & 3] + (i >> 2) * C::BOX_BYTES);
                    if (ntok < kBlockSize) {
                        vb[0] &= vm_lo;
                        vb[1] &= vm_lo;
                        vb[2] &= vm_hi;
                        vb[3] &= vm_hi;
                    }
                    Mma<T>::mma(o[2 * i], pa, vb[0], vb[2]);
                    Mma<T>::mma(o[2 * i + 1], pa, vb[1], vb[3]);
                    if constexpr (SPLIT_P) {
                        Mma<T>::mma(o[2 * i], pl, vb[0], vb[2]);
                        Mma<T>::mma(o[2 * i + 1], pl, vb[1], vb[3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
            ++c_k;
            if (++c_s == S) {
                c_s = 0;
                c_ph ^= 1u;
            }
            if (warp == 0) {
                // keep the ring S - LAG blocks ahead of warp 0
                while (p_alive && pc.valid && p_k < c_k - C::LAG + S) refill();
            }
        }
        if (!alive) {
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
#pragma unroll
            for (int i = 0; i < C::NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
        if (cs.j0 == 0 && cs.j1 == cs.nb) {
            const size_t out0 = ((size_t)cs.b * a.Hq + (size_t)cs.kvh * GC + row0 + g) * D + 2 * c;
            const size_t out1 = out0 + 8 * D;
#pragma unroll
            for (int i = 0; i < C::NT; ++i) {
                store_out2<T>(a.out, a.out_f32, out0 + 8 * i, o[i][0] * inv0, o[i][1] * inv0);
                store_out2<T>(a.out, a.out_f32, out1 + 8 * i, o[i][2] * inv1, o[i][3] * inv1);
            }
        } else {
            const int ch_first = ck.of(cs.b, cs.kvh, cs.nb, 0);
            const int slot = 2 * cs.ch + ((cs.ch == ch_first && ck.mid_start(cs.b, cs.kvh, cs.nb)) ? 1 : 0);
            float *w0 = a.ws_o + ((size_t)slot * GC + row0 + g) * D + 2 * c;
            float *w1 = w0 + 8 * D;
#pragma unroll
            for (int i = 0; i < C::NT; ++i) {
                *reinterpret_cast<float2 *>(w0 + 8 * i) = make_float2(o[i][0] * inv0, o[i][1] * inv0);
                *reinterpret_cast<float2 *>(w1 + 8 * i) = make_float2(o[i][2] * inv1, o[i][3] * inv1);
            }
            if (c == 0) {
                a.ws_lse[(size_t)slot * GC + row0 + g] = m0 * sl + log2f(l0);
                a.ws_lse[(size_t)slot * GC + row0 + g + 8] = m1 * sl + log2f(l1);
            }
        }
        have = next_seg(cit, cs);
    }
    // no copy may land after the CTA exits: warp 0 waits (bounded) for the ones it issued
    if (warp == 0 && lane == 0)
        for (int k = max(0, p_k - S); k < p_k; ++k) mbar_wait(&full[k % S], (k / S) & 1, a.wait_ns);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over a cache viewed as [rows = N*H_kv*16][D] with boxes of 16 rows
// of 128 bytes (64 fp16/bf16 or 128 int8 elements) and 128-byte swizzle.  Encoded maps are cached by (address,
// rows, D, dtype): the encode is a host call of a few microseconds.
bool tc_cache_tensor_map(CUtensorMap *m, const void *base, int64_t rows, int D, int dtype) {
    struct Key {
        const void *p;
        int64_t rows;
        int D, dt;
        bool operator==(const Key &o) const { return p == o.p && rows == o.rows && D == o.D && dt == o.dt; }
    };
    struct Hash {
        size_t operator()(const Key &k) const {
            return std::hash<const void *>()(k.p) ^ (std::hash<int64_t>()(k.rows) * 31) ^ (k.D * 131) ^ k.dt;
        }
    };
    static std::mutex mu;
    static std::unordered_map<Key, CUtensorMap, Hash> cache;
    const Key key{base, rows, D, dtype};
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *m = it->second;
            return true;
        }
    }
    auto fn = encode_fn();
    if (!fn) return false;
    // 4-bit caches: rows of D / 2 bytes, one unswizzled box per tile row
    const bool i4 = dtype == PA_I4;
    const int esize = (dtype == PA_I8 || i4) ? 1 : 2;
    const int width = i4 ? D / 2 : D;  // TMA elements per cache row
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)width * esize};
    cuuint32_t box[2] = {(cuuint32_t)(i4 ? width : 128 / esize), 16};  // 128-byte (4-bit: D/2-byte) box rows
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = dtype == PA_BF16                  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : (dtype == PA_I8 || i4)          ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    i4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() > 256) cache.clear();
    cache.emplace(key, *m);
    return true;
}

// SM count and resident CTAs per SM for (kernel, device, dynamic shared memory),
// queried once: the occupancy query costs microseconds of host time per call.
bool tc_launch_shape(const void *kernel, int threads, int smem, int *sms, int *per_sm) {
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, int>, std::pair<int, int>> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const auto key = std::make_tuple(kernel, dev, smem);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *sms = it->second.first;
            *per_sm = it->second.second;
            return true;
        }
    }
    int s = 0, p = 0;
    if (cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p, kernel, threads, smem) != cudaSuccess)
        return false;
    p = p < 1 ? 1 : p;
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = {s, p};
    *sms = s;
    *per_sm = p;
    return true;
}

bool decode_tc_supported(int q_dtype, int kv_dtype, int D, int G, int B) {
    const bool same = (q_dtype == PA_F16 || q_dtype == PA_BF16) && kv_dtype == q_dtype &&
                      (D == 64 || D == 128 || D == 256);
    const bool quant = q_dtype == PA_F16 &&
                       ((kv_dtype == PA_I8 && (D == 128 || D == 256)) || (kv_dtype == PA_I4 && D == 128));
    return (same || quant) && (G == 1 || G == 2 || G == 4 || G == 8) && B <= kTcMaxB;
}

template <typename T, typename TKV, int D, int G, bool MQ>
static int launch_tc(const DecodeArgs &a, cudaStream_t st) {
    using C = TcCfg<TKV, D, G>;
    auto kern = decode_tc_kernel<T, TKV, D, G, MQ, false>;
    if constexpr (!MQ && std::is_same<T, TKV>::value) {
        if (a.append) kern = decode_tc_kernel<T, TKV, D, G, MQ, true>;
    }
    if (a.append && kern == decode_tc_kernel<T, TKV, D, G, MQ, false>) return PA_ERR_UNSUPPORTED;
    const int smem = C::smem_bytes(a.B);
    if (!set_smem_attr_once(reinterpret_cast<const void *>(kern), C::smem_bytes(kTcMaxB))) return PA_ERR_CUDA;
    if ((uintptr_t)a.q % 16) return PA_ERR_ALIGN;  // q rows are read as aligned 32-bit pairs
    CUtensorMap tk, tv;
    const int64_t rows = a.N * (a.Hkv / a.ngroups) * kBlockSize;  // the cache's rows
    if (!tc_cache_tensor_map(&tk, a.kc, rows, D, a.kv_dtype) || !tc_cache_tensor_map(&tv, a.vc, rows, D, a.kv_dtype))
        return PA_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (!tc_launch_shape(reinterpret_cast<const void *>(kern), C::THREADS, smem, &sms, &per_sm)) return PA_ERR_CUDA;
    // persistent grid: every resident warp is a worker, but no more warps than
    // there are blocks to read (every sequence at max_len)
    const int64_t blocks = (int64_t)a.B * a.Hkv * ((a.max_len + kBlockSize - 1) / kBlockSize);
    int64_t ctas = (int64_t)sms * per_sm;
    const int64_t need = (blocks + C::NW - 1) / C::NW;
    if (need < ctas) ctas = need;
    if (ctas < 1) ctas = 1;
    DecodeArgs a2 = a;
    a2.tc_W = (int)ctas * C::NW;
    if (launch_pdl(kern, dim3((unsigned)ctas), dim3(C::THREADS), smem, st, tk, tv, a2) != cudaSuccess)
        return PA_ERR_CUDA;
    if (a.tc_chunk < 0 || a.ws_o == nullptr) return PA_OK;  // one pass: nothing to merge
    auto mk = merge_tc_kernel<T, D, G, MQ>;
    const int msmem = 2 * (a.B + 1) * 4;
    if (!set_smem_attr_once(reinterpret_cast<const void *>(mk), 2 * (kTcMaxB + 1) * 4)) return PA_ERR_CUDA;
    const int64_t items = (int64_t)a.B * a.Hkv * G;
    int64_t mctas = (items + 7) / 8;
    if (mctas > 2 * sms) mctas = 2 * sms;
    return launch_pdl(mk, dim3((unsigned)mctas), dim3(256), msmem, st, a2) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D, int NG>
static int launch_coop(const DecodeArgs &a, cudaStream_t st) {
    using C = CoopCfg<T, D, NG>;
    auto kern = decode_coop_kernel<T, D, NG>;
    DecodeArgs a2 = a;
    a2.Hkv = a.Hkv / a.ngroups;  // cache rows; GC = 8 NG columns each
    a2.ngroups = 1;
    a2.G = NG * 16;
    a2.gcols = NG * 16;
    const int smem = C::smem_bytes(a.B);
    if (!set_smem_attr_once(reinterpret_cast<const void *>(kern), C::smem_bytes(kTcMaxB))) return PA_ERR_CUDA;
    CUtensorMap tk, tv;
    const int64_t rows = a.N * a2.Hkv * kBlockSize;
    if (!tc_cache_tensor_map(&tk, a.kc, rows, D, a.kv_dtype) || !tc_cache_tensor_map(&tv, a.vc, rows, D, a.kv_dtype))
        return PA_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (!tc_launch_shape(reinterpret_cast<const void *>(kern), C::THREADS, smem, &sms, &per_sm)) return PA_ERR_CUDA;
    const int64_t blocks = (int64_t)a.B * a2.Hkv * ((a.max_len + kBlockSize - 1) / kBlockSize);
    int64_t ctas = (int64_t)sms * per_sm;
    const int64_t need = (blocks + kTcMinChunk - 1) / kTcMinChunk;
    if (need < ctas) ctas = need;
    if (ctas < 1) ctas = 1;
    a2.tc_W = (int)ctas;
    if (launch_pdl(kern, dim3((unsigned)ctas), dim3(C::THREADS), smem, st, tk, tv, a2) != cudaSuccess)
        return PA_ERR_CUDA;
    return launch_merge_rows(a2, sms, st);
}

template <typename T, int D, int GC>
static int launch_merge_rows_t(const DecodeArgs &a2, int sms, cudaStream_t st) {
    auto mk = merge_tc_kernel<T, D, GC, false>;
    const int msmem = 2 * (a2.B + 1) * 4;
    if (!set_smem_attr_once(reinterpret_cast<const void *>(mk), 2 * (kTcMaxB + 1) * 4)) return PA_ERR_CUDA;
    const int64_t items = (int64_t)a2.B * a2.Hkv * GC;
    int64_t mctas = (items + 7) / 8;
    if (mctas > 2 * sms) mctas = 2 * sms;
    return launch_pdl(mk, dim3((unsigned)mctas), dim3(256), msmem, st, a2) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D>
static int launch_merge_rows_d(const DecodeArgs &a2, int sms, cudaStream_t st) {
    switch (a2.G) {
    case 16: return launch_merge_rows_t<T, D, 16>(a2, sms, st);
    case 32: return launch_merge_rows_t<T, D, 32>(a2, sms, st);
    case 64: return launch_merge_rows_t<T, D, 64>(a2, sms, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

int launch_merge_rows(const DecodeArgs &a2, int sms, cudaStream_t st) {
    if (a2.D != 64 && a2.D != 128) return PA_ERR_UNSUPPORTED;
    if (a2.q_dtype == PA_F16)
        return a2.D == 64 ? launch_merge_rows_d<__half, 64>(a2, sms, st) : launch_merge_rows_d<__half, 128>(a2, sms, st);
    if (a2.q_dtype == PA_BF16)
        return a2.D == 64 ? launch_merge_rows_d<__nv_bfloat16, 64>(a2, sms, st)
                          : launch_merge_rows_d<__nv_bfloat16, 128>(a2, sms, st);
    return PA_ERR_DTYPE;
}

bool decode_coop_eligible(int q_dtype, int kv_dtype, int D, int G, int ngroups, int qlen, bool padded, int part) {
    return (q_dtype == PA_F16 || q_dtype == PA_BF16) && kv_dtype == q_dtype && (D == 64 || D == 128) && G == 8 &&
           (ngroups == 2 || ngroups == 4 || ngroups == 8) && qlen == 1 && !padded && part != 0;
}

template <typename T, typename TKV, int D, bool MQ>
static int launch_tc_mq(const DecodeArgs &a, cudaStream_t st) {
    switch (a.G) {
    case 1: return launch_tc<T, TKV, D, 1, MQ>(a, st);
    case 2: return launch_tc<T, TKV, D, 2, MQ>(a, st);
    case 4: return launch_tc<T, TKV, D, 4, MQ>(a, st);
    case 8: return launch_tc<T, TKV, D, 8, MQ>(a, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T, typename TKV, int D>
static int launch_tc_g(const DecodeArgs &a, cudaStream_t st) {
    // several new tokens, or padding columns: the general column mapping
    const bool mq = a.qlen > 1 || (int64_t)a.G * a.ngroups != a.gcols;
    if constexpr (std::is_same<T, TKV>::value && D <= 128) {
        if (a.umma && a.tc_chunk >= 0) return launch_decode_umma(a, st);
        if (decode_coop_eligible(a.q_dtype, a.kv_dtype, D, a.G, a.ngroups, a.qlen, mq, a.tc_chunk < 0 ? 0 : 1)) {
            switch (a.ngroups) {
            case 2: return launch_coop<T, D, 1>(a, st);
            case 4: return launch_coop<T, D, 2>(a, st);
            default: return launch_coop<T, D, 4>(a, st);
            }
        }
    }
    return mq ? launch_tc_mq<T, TKV, D, true>(a, st) : launch_tc_mq<T, TKV, D, false>(a, st);
}

int launch_decode_tc(const DecodeArgs &a, cudaStream_t st) {
    if (a.q_dtype == PA_F16 && a.kv_dtype == PA_I8) {
        if (a.D == 256) return launch_tc_g<__half, int8_t, 256>(a, st);
        if (a.D != 128) return PA_ERR_UNSUPPORTED;
        return launch_tc_g<__half, int8_t, 128>(a, st);
    }
    if (a.q_dtype == PA_F16 && a.kv_dtype == PA_I4) {
        if (a.D != 128) return PA_ERR_UNSUPPORTED;
        return launch_tc_g<__half, U4x2, 128>(a, st);
    }
    if (a.q_dtype == PA_F16)
        return a.D == 64    ? launch_tc_g<__half, __half, 64>(a, st)
               : a.D == 128 ? launch_tc_g<__half, __half, 128>(a, st)
                            : launch_tc_g<__half, __half, 256>(a, st);
    if (a.q_dtype == PA_BF16)
        return a.D == 64    ? launch_tc_g<__nv_bfloat16, __nv_bfloat16, 64>(a, st)
               : a.D == 128 ? launch_tc_g<__nv_bfloat16, __nv_bfloat16, 128>(a, st)
                            : launch_tc_g<__nv_bfloat16, __nv_bfloat16, 256>(a, st);
    return PA_ERR_DTYPE;
}

}  // namespace pa
