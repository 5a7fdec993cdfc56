// Paged decode attention, tensor-core kernel family (fp16 / bf16 KV, G <= 8).
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
// Scheduling: a persistent grid; every warp is an independent worker.  Work
// items are (sequence, partition of `part` tokens, KV head); warp w takes
// items w, w + W, w + 2W, ... (W = warps in the grid).  Each warp owns a
// 3-stage ring, refilled one block ahead per consumed block, and the refill
// runs straight on into the warp's next item, so the copy stream does not
// drain between items.  A single-partition item writes its output directly.
// Otherwise it writes its normalised partial output and log2-sum-exp to the
// workspace and takes a ticket from a per-(sequence, KV head) counter; the
// warp that takes the last ticket merges all partitions
//   out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M)
// and resets the counter to zero (no waiting on other warps).
#include <cudaTypedefs.h>

#include <mutex>
#include <unordered_map>

#include "pa_common.cuh"
#include "pa_internal.h"

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
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

template <typename T> struct Mma;
template <> struct Mma<__half> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};
template <> struct Mma<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t r;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
        return r;
    }
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

// ---------------------------------------------------------------------------
// configuration
// ---------------------------------------------------------------------------
template <int D>
struct TcCfg {
    static constexpr int NW = 4;
    static constexpr int THREADS = NW * 32;
    static constexpr int S = 3;                   // ring stages per warp
    static constexpr int BOXES = D / 64;          // 64-element (128-byte) boxes per row
    static constexpr int BOX_BYTES = 16 * 128;    // one box of a tile
    static constexpr int TILE = BOXES * BOX_BYTES;
    static constexpr int STAGE = 2 * TILE;        // K tile, then V tile
    static constexpr int KSTEPS = D / 16;         // QK k-steps
    static constexpr int MTILES = D / 16;         // PV m-tiles
    static constexpr int RING = NW * S * STAGE;
    static constexpr int BAR_OFF = RING;
    static constexpr int BLK_OFF = BAR_OFF + NW * S * 8;
    static constexpr int CUM_OFF = BLK_OFF + NW * S * 4;
    static constexpr int MAX_B = 4096;
    static int smem_bytes(int B) { return 1024 + CUM_OFF + (B + 1) * 4; }
};

struct Item {
    int b, kvh, part, L, t0, nblk, ntok_last, nparts;
};

// Physical address of the 16-byte chunk `chunk` (0 .. D/8-1) of row `row`
// (0..15) of a swizzled tile: box = chunk / 8, and inside the 1024-byte
// aligned box the chunk index is XORed with row % 8 (128-byte swizzle).
__device__ __forceinline__ uint32_t tile_chunk(uint32_t tile, int row, int chunk) {
    return tile + (chunk >> 3) * 2048 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

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

template <typename T, int D, int G>
__global__ void __launch_bounds__(128) decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                        const __grid_constant__ CUtensorMap tmV,
                                                        const DecodeArgs a) {
    using C = TcCfg<D>;
    constexpr int NW = C::NW, S = C::S;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    int *blk_ids = reinterpret_cast<int *>(smem + C::BLK_OFF);
    int *cum = reinterpret_cast<int *>(smem + C::CUM_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = a.B;
    const int P = a.part;  // > 0: partition size; 0: one partition per sequence

    // ---- partitions per sequence -> exclusive prefix sum in cum[0..B] ------------
    {
        __shared__ int wsum[NW];
        const int per = (B + C::THREADS - 1) / C::THREADS;
        const int lo = min(B, tid * per), hi = min(B, lo + per);
        int s = 0;
        for (int b = lo; b < hi; ++b) {
            int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            s += (L <= 0 || P == 0) ? 1 : (L + P - 1) / P;
        }
        int x = s;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w) base += wsum[w];
        int run = base + x - s;
        for (int b = lo; b < hi; ++b) {
            cum[b] = run;
            int L = min(min(a.lens[b], a.max_len), a.mbps * kBlockSize);
            run += (L <= 0 || P == 0) ? 1 : (L + P - 1) / P;
        }
        if (tid == C::THREADS - 1) cum[B] = run;
        __syncthreads();
    }
    const int total_items = cum[B] * a.Hkv;

    auto item_at = [&](int it) -> Item {
        Item r;
        const int u = it / a.Hkv;
        r.kvh = it - u * a.Hkv;
        int lo = 0, hi = B;  // largest b with cum[b] <= u
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid] <= u) lo = mid; else hi = mid;
        }
        r.b = lo;
        r.part = u - cum[lo];
        r.L = min(min(a.lens[lo], a.max_len), a.mbps * kBlockSize);
        const int Pe = P > 0 ? P : max(r.L, 1);
        r.t0 = r.part * Pe;
        const int t1 = min(r.L, r.t0 + Pe);
        r.nblk = r.L > 0 ? (t1 - r.t0 + kBlockSize - 1) / kBlockSize : 0;
        r.ntok_last = r.L > 0 ? t1 - r.t0 - (r.nblk - 1) * kBlockSize : 0;
        r.nparts = r.L > 0 ? (r.L + Pe - 1) / Pe : 1;
        return r;
    };

    uint64_t *my_bars = bars + warp * S;
    int *my_blk = blk_ids + warp * S;
    const uint32_t ring = smem_addr(smem) + warp * S * C::STAGE;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < S; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const int gw = blockIdx.x * NW + warp;
    const int W = gridDim.x * NW;

    // ---- producer: the warp's stream of blocks, S blocks ahead of the consumer ----
    // Lane l holds table entry (p_j & ~31) + l of the producer's item: a
    // coalesced load of 32 entries, read out with a shuffle per block.
    int p_item = gw, p_j = 0, p_k = 0, p_tab = -1;
    Item pi{};
    auto p_load_tab = [&]() {
        const int idx = (p_j & ~31) + lane;
        p_tab = idx < pi.nblk ? a.tables[(size_t)pi.b * a.mbps + pi.t0 / kBlockSize + idx] : -1;
    };
    auto p_enter = [&]() {  // position the producer on the next item that has blocks
        while (p_item < total_items) {
            pi = item_at(p_item);
            if (pi.nblk > 0) break;
            p_item += W;
        }
        if (p_item < total_items) p_load_tab();
    };
    p_enter();
    auto refill = [&]() {
        if (p_item >= total_items) return;
        const int pb = __shfl_sync(0xffffffffu, p_tab, p_j & 31);
        if (lane == 0) {
            const int s = p_k % S;
            uint64_t *bar = &my_bars[s];
            if (pb < 0 || (int64_t)pb >= a.N) {
                my_blk[s] = -1;
                raise_flag(PA_EFLAG_BAD_BLOCK);
                mbar_arrive(bar);
            } else {
                my_blk[s] = pb;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, C::STAGE);
                const int row = (pb * a.Hkv + pi.kvh) * kBlockSize;
                const uint32_t dst = ring + s * C::STAGE;
#pragma unroll
                for (int bx = 0; bx < C::BOXES; ++bx) {
                    tma_load_2d(dst + bx * C::BOX_BYTES, &tmK, bx * 64, row, smem_addr(bar));
                    tma_load_2d(dst + C::TILE + bx * C::BOX_BYTES, &tmV, bx * 64, row, smem_addr(bar));
                }
            }
        }
        ++p_k;
        if (++p_j == pi.nblk) {
            p_j = 0;
            p_item += W;
            p_enter();
        } else if ((p_j & 31) == 0) {
            p_load_tab();
        }
    };
#pragma unroll
    for (int i = 0; i < S; ++i) refill();

    const int g = lane >> 2, c = lane & 3;  // mma fragment coordinates
    const int h0 = 2 * c, h1 = 2 * c + 1;  // the two heads of this thread's S^T / O^T columns
    int c_k = 0;
    bool alive = true;

    for (int it = gw; it < total_items && alive; it += W) {
        const Item ci = item_at(it);
        T *out = reinterpret_cast<T *>(a.out) + ((size_t)ci.b * a.Hq + (size_t)ci.kvh * G) * D;
        if (ci.L <= 0) {
            for (int i = lane; i < G * D; i += 32) out[i] = Cvt<T>::from_f(0.f);
            continue;
        }
        // B fragments of Q^T: k = dims, n = heads (rows >= G are zero padding)
        uint32_t bq[C::KSTEPS][2];
        {
            const T *qp = reinterpret_cast<const T *>(a.q) + ((size_t)ci.b * a.Hq + (size_t)ci.kvh * G) * D;
#pragma unroll
            for (int s = 0; s < C::KSTEPS; ++s) {
                if (g < G) {
                    bq[s][0] = *reinterpret_cast<const uint32_t *>(qp + g * D + 16 * s + 2 * c);
                    bq[s][1] = *reinterpret_cast<const uint32_t *>(qp + g * D + 16 * s + 2 * c + 8);
                } else {
                    bq[s][0] = bq[s][1] = 0u;
                }
            }
        }
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[C::MTILES][4];
#pragma unroll
        for (int i = 0; i < C::MTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

        for (int j = 0; j < ci.nblk; ++j) {
            const int s = c_k % S;
            const uint32_t parity = (c_k / S) & 1;
            int ok = lane == 0 ? (int)mbar_wait(&my_bars[s], parity) : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                alive = false;
                break;
            }
            if (lane != 0) mbar_wait(&my_bars[s], parity);
            const int pb = my_blk[s];
            const int ntok = (j == ci.nblk - 1) ? ci.ntok_last : kBlockSize;
            const uint32_t tK = ring + s * C::STAGE;
            const uint32_t tV = tK + C::TILE;
            if (pb >= 0) {
                if (ntok < kBlockSize) {
                    // rows past the sequence end hold stale data (possibly NaN/Inf):
                    // zero those V rows so that 0-probability tokens add exactly 0
                    unsigned char *vrow = smem + (tV - smem_addr(smem));
                    const int nrow = kBlockSize - ntok;
                    for (int i = lane; i < nrow * C::BOXES * 8; i += 32) {
                        const int r = ntok + i / (C::BOXES * 8);
                        const int rem = i % (C::BOXES * 8);
                        *reinterpret_cast<uint4 *>(vrow + (rem >> 3) * 2048 + r * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();  // before the stage is refilled by TMA
                    __syncwarp();
                }
                // ---- S^T = K . Q^T
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) {
                    uint32_t af[4];
                    const int mi = lane >> 3, r = lane & 7;
                    const int row = r + ((mi & 1) << 3);
                    const int chunk = 2 * ks + (mi >> 1);
                    ldsm_x4(af, tile_chunk(tK, row, chunk));
                    Mma<T>::mma(sc, af, bq[ks][0], bq[ks][1]);
                }
                // ---- online softmax (log2 domain); rows g and g+8 are tokens, columns heads
                const bool v0 = g < ntok, v1 = g + 8 < ntok;
                const float s0 = v0 ? sc[0] * a.scale_log2 : -INFINITY;
                const float s1 = v0 ? sc[1] * a.scale_log2 : -INFINITY;
                const float s2 = v1 ? sc[2] * a.scale_log2 : -INFINITY;
                const float s3 = v1 ? sc[3] * a.scale_log2 : -INFINITY;
                float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
                for (int msk = 4; msk < 32; msk <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
                }
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
                const float p0 = fast_exp2(s0 - mn0), p1 = fast_exp2(s1 - mn1);
                const float p2 = fast_exp2(s2 - mn0), p3 = fast_exp2(s3 - mn1);
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
                // ---- P^T fragments (k = tokens, n = heads) by transposing the S^T layout
                const uint32_t pb0 = movm_t(Mma<T>::pack(p0, p1));  // tokens 0-7
                const uint32_t pb1 = movm_t(Mma<T>::pack(p2, p3));  // tokens 8-15
                // ---- O^T += V^T . P^T
#pragma unroll
                for (int i = 0; i < C::MTILES; ++i) {
                    uint32_t af[4];
                    const int mi = lane >> 3, r = lane & 7;
                    const int row = r + ((mi >> 1) << 3);
                    const int chunk = 2 * i + (mi & 1);
                    ldsm_x4_t(af, tile_chunk(tV, row, chunk));
                    Mma<T>::mma(o[i], af, pb0, pb1);
                }
            }
            __syncwarp();
            refill();
            ++c_k;
        }
        if (!alive) break;

        // ---- finish the item
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, msk);
            l1 += __shfl_xor_sync(0xffffffffu, l1, msk);
        }
        const float inv0 = 1.f / l0, inv1 = 1.f / l1;
        if (ci.nparts == 1) {
#pragma unroll
            for (int i = 0; i < C::MTILES; ++i) {
                const int d0 = 16 * i + g, d1 = d0 + 8;
                if (h0 < G) {
                    out[h0 * D + d0] = Cvt<T>::from_f(o[i][0] * inv0);
                    out[h0 * D + d1] = Cvt<T>::from_f(o[i][2] * inv0);
                }
                if (h1 < G) {
                    out[h1 * D + d0] = Cvt<T>::from_f(o[i][1] * inv1);
                    out[h1 * D + d1] = Cvt<T>::from_f(o[i][3] * inv1);
                }
            }
            continue;
        }
        const size_t row0 = ((size_t)ci.b * a.Hq + (size_t)ci.kvh * G) * a.max_parts;
#pragma unroll
        for (int i = 0; i < C::MTILES; ++i) {
            const int d0 = 16 * i + g, d1 = d0 + 8;
            if (h0 < G) {
                float *w = a.ws_o + (row0 + (size_t)h0 * a.max_parts + ci.part) * D;
                w[d0] = o[i][0] * inv0;
                w[d1] = o[i][2] * inv0;
            }
            if (h1 < G) {
                float *w = a.ws_o + (row0 + (size_t)h1 * a.max_parts + ci.part) * D;
                w[d0] = o[i][1] * inv1;
                w[d1] = o[i][3] * inv1;
            }
        }
        if (g == 0) {
            if (h0 < G) a.ws_lse[row0 + (size_t)h0 * a.max_parts + ci.part] = m0 + log2f(l0);
            if (h1 < G) a.ws_lse[row0 + (size_t)h1 * a.max_parts + ci.part] = m1 + log2f(l1);
        }
        __threadfence();
        __syncwarp();
        int *ticket = a.counters + (size_t)ci.b * a.Hkv + ci.kvh;
        int old = 0;
        if (lane == 0) old = atomicAdd(ticket, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != ci.nparts - 1) continue;
        // ---- last partition of (b, kvh): merge every partition of its G heads
        __threadfence();
        for (int h = 0; h < G; ++h) {
            const float *lse = a.ws_lse + row0 + (size_t)h * a.max_parts;
            const float *op = a.ws_o + (row0 + (size_t)h * a.max_parts) * D;
            float M = -INFINITY;
            for (int p = lane; p < ci.nparts; p += 32) M = fmaxf(M, __ldcg(lse + p));
            M = warp_max(M);
            float Ssum = 0.f;
            for (int p = lane; p < ci.nparts; p += 32) Ssum += fast_exp2(__ldcg(lse + p) - M);
            Ssum = warp_sum(Ssum);
            const float inv = 1.f / Ssum;
            for (int d = lane; d < D; d += 32) {
                float acc = 0.f;
                for (int p = 0; p < ci.nparts; ++p)
                    acc = fmaf(fast_exp2(__ldcg(lse + p) - M), __ldcg(op + (size_t)p * D + d), acc);
                out[h * D + d] = Cvt<T>::from_f(acc * inv);
            }
        }
        if (lane == 0) *ticket = 0;  // the workspace is left as it was found
    }
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

// 2-D map over a cache viewed as [rows = N*H_kv*16][D] with 64-element boxes
// of 16 rows and 128-byte swizzle.  Encoded maps are cached by (address,
// rows, D, dtype): the encode is a host call of a few microseconds.
static bool cache_tensor_map(CUtensorMap *m, const void *base, int64_t rows, int D, int dtype) {
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
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() > 256) cache.clear();
    cache.emplace(key, *m);
    return true;
}

bool decode_tc_supported(int q_dtype, int kv_dtype, int D, int G, int B) {
    return (q_dtype == PA_F16 || q_dtype == PA_BF16) && kv_dtype == q_dtype && (D == 64 || D == 128) &&
           (G == 1 || G == 2 || G == 4 || G == 8) && B <= TcCfg<128>::MAX_B;
}

template <typename T, int D, int G>
static int launch_tc(const DecodeArgs &a, cudaStream_t st) {
    using C = TcCfg<D>;
    auto kern = decode_tc_kernel<T, D, G>;
    const int smem = C::smem_bytes(a.B);
    if (!set_smem_attr_once(reinterpret_cast<const void *>(kern), C::smem_bytes(C::MAX_B))) return PA_ERR_CUDA;
    CUtensorMap tk, tv;
    const int64_t rows = a.N * a.Hkv * kBlockSize;
    if (!cache_tensor_map(&tk, a.kc, rows, D, a.kv_dtype) || !cache_tensor_map(&tv, a.vc, rows, D, a.kv_dtype))
        return PA_ERR_CUDA;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::THREADS, smem) != cudaSuccess)
        return PA_ERR_CUDA;
    per_sm = per_sm < 1 ? 1 : per_sm;
    // an upper bound on the items: every sequence at max_len
    const int64_t parts = a.part > 0 ? a.max_parts : 1;
    const int64_t items = (int64_t)a.B * a.Hkv * parts;
    int64_t ctas = (int64_t)sms * per_sm;
    const int64_t need = (items + C::NW - 1) / C::NW;
    if (need < ctas) ctas = need;
    if (ctas < 1) ctas = 1;
    kern<<<(unsigned)ctas, C::THREADS, smem, st>>>(tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename T, int D>
static int launch_tc_g(const DecodeArgs &a, cudaStream_t st) {
    switch (a.G) {
    case 1: return launch_tc<T, D, 1>(a, st);
    case 2: return launch_tc<T, D, 2>(a, st);
    case 4: return launch_tc<T, D, 4>(a, st);
    case 8: return launch_tc<T, D, 8>(a, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

int launch_decode_tc(const DecodeArgs &a, cudaStream_t st) {
    if (a.q_dtype == PA_F16) return a.D == 64 ? launch_tc_g<__half, 64>(a, st) : launch_tc_g<__half, 128>(a, st);
    if (a.q_dtype == PA_BF16)
        return a.D == 64 ? launch_tc_g<__nv_bfloat16, 64>(a, st) : launch_tc_g<__nv_bfloat16, 128>(a, st);
    return PA_ERR_DTYPE;
}

}  // namespace pa
