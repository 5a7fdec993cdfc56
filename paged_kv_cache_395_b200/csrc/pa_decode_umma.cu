// Paged decode attention on the 5th-generation tensor cores (tcgen05, accumulators in
// tensor memory) for groups of 32 or 64 query heads per KV head (MQA-like), head_dim
// 128, fp16 / bf16.
//
// Same computation as decode_tc_kernel (lqnn.cn/news/235768 sections 1.2, 2.2, 3.2,
// 4.2):  out[b][h] = sum_t softmax_t(scale * q[b][h] . K[b][t]) V[b][t].  With 32-64
// query heads per KV head the products of a cache tile are dense contractions, so they
// run as tcgen05 MMAs over groups of n <= 8 consecutive blocks of one cache row:
//   S[64 heads x 16n tokens] = Q[64 x 128] . K^T     (M = 64, N = 16n, K = 128)
//   O[64 heads x 128 dims]  += P[64 x 16n] . V        (M = 64, N = 128, K = 16n; one MMA
//                                                      of N = 128 per block)
// S (two buffers) and O live in tensor memory (256 columns); P is written to shared
// memory by the softmax warps.  A group of 32 heads fills rows 0-31 (rows 32-63 hold zero q rows,
// computed and ignored).
//
// One CTA per SM (~195 KB of shared memory), seven warps:
// * warp 4, K producer: per group, TMA for each block's two 64-dim K boxes into two
//   box-major rings (K dims 0-63, K dims 64-127; two halves of 8 blocks), so that a
//   group's 16n token rows sit at one 128-byte pitch as the MMA descriptors want; a
//   K half is refilled as soon as the QK products that read it have finished.  It
//   also copies a new segment's q rows into one of two q slots (128-byte swizzle, the
//   same canonical K-major layout).
// * warp 6, V producer: the same for the V boxes, a V half being refilled once the
//   P.V products that read it have finished.
// * warp 5, MMA issuer (it also owns the TMEM allocation): lane 0 issues a group's 16
//   QK MMAs into S[g % 2] one group ahead, then, once the softmax has written P and
//   the group's V tiles have landed, the group's 8 P.V MMAs into O (V of a block as one
//   MN-major operand of 128 dims, its two 64-dim ring regions one leading byte offset
//   apart: an MMA costs about as much to issue at N = 64 as at 128); tcgen05.commit
//   signals S ready, K half free, P.V done, V half free and q slot free on mbarriers.
// * warps 0-3, softmax and epilogue.  An M = 64 accumulator puts rows 16w .. 16w + 15 in
//   TMEM lanes 32w .. 32w + 15 (lane tile 0) or, one tile over, 32w + 16 .. 32w + 31 (lane
//   tile 1); S takes a group's blocks 0-3 in tile 0 and 4-7 in tile 1, O all 128 dims in
//   tile 0.  Thread (w, l) so owns head row 16w + (l & 15) and 64 of its scores; one shuffle
//   joins the two halves' maxima and sums, and the threads of lane tile 0 write the row's
//   output.
//   It reads its scores, masks slots past the row's end (and blocks outside the pool), keeps the
//   online softmax with the lazy maximum of the cooperative kernel (scores unscaled, the
//   scale in the exponent, O rescaled in TMEM only when the maximum moves by more than
//   2^8), writes its P row, zeroes the stale V rows of a row's last block (0 x NaN would
//   poison the product), and at a segment's end reads its O row and writes the output or
//   the partial result.
// Every barrier completes once per use of its buffer, and no buffer is refilled before
// every wait on its previous phase has returned, so no wait can alias a later phase
// (which is why the softmax waits for S ready, not for the K tiles).
// Chunks of the cache-row stream go to CTAs as in decode_coop_kernel; cut rows leave
// partial results for merge_tc_kernel, GC columns per cache row.
#include <type_traits>

#include "pa_tc_shared.cuh"

namespace pa {

PA_ERROR_WORD_ACCESSOR(error_word_decode_umma)

namespace {

constexpr int kUD = 128;            // head_dim
constexpr int kUGroup = 8;          // blocks per MMA group
constexpr int kUThreads = 224;      // warps 0-3 softmax, 4 K producer, 5 MMA, 6 V producer
constexpr int kUBox = 16 * 128;     // one 64-dim box of one block: 16 rows x 128 bytes
constexpr int kURegion = 2 * kUGroup * kUBox;  // one box-major ring: two halves of 8 blocks
constexpr int kUQSlot = 2 * 64 * 128;          // 64 q rows x 2 boxes
constexpr int kUPBuf = 2 * 64 * 128;           // P: 64 rows x 128 tokens (2 boxes)
constexpr int kUTmemCols = 256;                // S0, S1, O (64 columns each, both lane tiles)
constexpr float kULazyMax = 8.f;

// shared memory layout (offsets from the 1024-aligned base)
constexpr int kUK0 = 0;
constexpr int kUK1 = kUK0 + kURegion;
constexpr int kUV0 = kUK1 + kURegion;
constexpr int kUV1 = kUV0 + kURegion;
constexpr int kUQ = kUV1 + kURegion;           // two q slots
constexpr int kUP = kUQ + 2 * kUQSlot;         // two P buffers
constexpr int kUBar = kUP + 2 * kUPBuf;
// barriers: full_k[2], full_v[2], empty_k[2], empty_v[2], s_ready[2], p_ready[2],
// pv_done[2], qfull[2], qempty[2]
constexpr int kUNBar = 18;
constexpr int kUMisc = kUBar + kUNBar * 8;     // tmem address, abort flag
constexpr int kUCum = kUMisc + 16;
inline int umma_smem_bytes(int B) { return 1024 + kUCum + (3 * B + 3) * 4; }

// ---- tcgen05 wrappers ----------------------------------------------------------------
// Shared-memory matrix descriptor: start, leading and stride byte offsets (16-byte
// units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16 with fp32 accumulation: A and B of type fmt
// (0 fp16, 1 bf16), A K-major, B K-major (b_mn = 0) or MN-major (1), M x N.
__device__ __forceinline__ uint32_t umma_idesc(uint32_t fmt, int M, int N, uint32_t b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 lanes x 32 columns of 32 bits (thread t: lane base + t)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
        "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
        "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
        "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
}
// 32 lanes x 64 columns of 32 bits (thread t: lane base + t)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float *v) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,"
        "%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(r[j]);
}
// A bounded mbarrier wait whose polls sleep in hardware until the phase completes (or
// 50 us pass): waiting warps issue nothing while the softmax warps on the same SM
// sub-partitions work.  Gives up after limit_ns, raising PA_EFLAG_WAIT_TIMEOUT.
__device__ __forceinline__ bool mbar_sleep_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
    const uint32_t addr = smem_addr(bar);
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(addr), "r"(parity), "r"(50000u) : "memory");
    if (ok) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok) : "r"(addr), "r"(parity), "r"(50000u) : "memory");
        if (ok) return true;
        if (global_timer_ns() - t0 > limit_ns) {
            raise_flag(PA_EFLAG_WAIT_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
// row r, 16-byte chunk c (0-7) of a 128-byte-row, 128-byte-swizzled region
__device__ __forceinline__ uint32_t swz128(uint32_t base, int r, int c) { return base + r * 128 + ((c ^ (r & 7)) << 4); }

template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One group: n <= 8 consecutive blocks j0 .. j0 + n - 1 of cache row (b, kc).
struct Grp {
    int b, kc, L, nb, j0, n;
    int ch, fr;      // chunk of the segment (partials), row start in the block stream
    int si;          // segment ordinal in this CTA
    bool seg_first, seg_last, whole;  // first / last group of its segment; the segment is the whole row
};

}  // namespace

template <typename T, int GC>
__global__ void __launch_bounds__(kUThreads, 1)
    decode_umma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeArgs a) {
    static_assert(GC == 32 || GC == 64, "groups of 32 or 64 query heads");
    constexpr uint32_t kFmt = std::is_same<T, __half>::value ? 0u : 1u;
    // bf16 keeps 8 significant bits: P goes in as hi + lo (the two P buffers of one group,
    // two products per block), so that it enters the product with ~16 bits.  fp16 P uses
    // the two buffers for consecutive groups instead.
    constexpr bool SPLIT = kFmt == 1u;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kUBar);
    uint64_t *full_k = bars, *full_v = bars + 2, *empty_k = bars + 4, *empty_v = bars + 6, *s_ready = bars + 8,
             *p_ready = bars + 10, *pv_done = bars + 12, *qfull = bars + 14, *qempty = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kUMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kUMisc + 4);
    int *cum = reinterpret_cast<int *>(smem + kUCum);  // [B + 1]
    int *lens = cum + a.B + 1;                          // [B]
    int *cumv = lens + a.B;                             // [B + 1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = a.B, Hc = a.Hkv;  // the launcher passes the cache's KV heads
    if (tid == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        *abort_flag = 0;
    }
    if (!a.early) {
        pdl_wait();
        pdl_release_dependents();
    }
    const int gam = a.tc_chunk == 0 ? PA_TC_GAMMA : 0;
    {
        __shared__ int wsum[kUThreads / 32], wsumv[kUThreads / 32];
        const int per = (B + kUThreads - 1) / kUThreads;
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
        if (tid == kUThreads - 1) {
            cum[B] = run;
            cumv[B] = runv;
        }
        if (tid == 0) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&full_k[i], 1);
                mbar_init(&full_v[i], 1);
                mbar_init(&empty_k[i], 1);
                mbar_init(&empty_v[i], 1);
                mbar_init(&s_ready[i], 1);
                mbar_init(&p_ready[i], 128);
                mbar_init(&pv_done[i], 1);
                mbar_init(&qfull[i], 1);
                mbar_init(&qempty[i], 1);
            }
            fence_mbar_init();
        }
        // q rows GC .. 63 of both slots stay zero (their S rows are computed and ignored)
        if constexpr (GC < 64) {
            constexpr int PER_BOX = (64 - GC) * 8;  // 16-byte chunks
            for (int i = tid; i < 4 * PER_BOX; i += kUThreads) {
                const int sb = i / PER_BOX, rem = i % PER_BOX;  // sb: slot * 2 + box
                sts128(swz128(sbase + kUQ + (sb >> 1) * kUQSlot + (sb & 1) * 64 * 128, GC + rem / 8, rem % 8), 0u, 0u,
                       0u, 0u);
            }
        }
        fence_async_smem();
        if (warp == 5) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                         "r"(kUTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    const uint32_t tmem = *tmem_slot;
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
    // the CTA's groups, in order: every role walks the same sequence
    struct GIt {
        SegIter it;
        Seg sg;
        bool have;
        int j, si;
    };
    auto git_init = [&](GIt &g) {
        g.it = SegIter{0, 0, 0, -1, false};
        g.it.done = !range(g.it);
        g.have = next_seg(g.it, g.sg);
        g.j = g.have ? g.sg.j0 : 0;
        g.si = 0;
    };
    auto next_group = [&](GIt &g, Grp &r) -> bool {
        if (!g.have) return false;
        r.b = g.sg.b;
        r.kc = g.sg.kvh;
        r.L = g.sg.L;
        r.nb = g.sg.nb;
        r.j0 = g.j;
        r.n = min(kUGroup, g.sg.j1 - g.j);
        r.ch = g.sg.ch;
        r.fr = g.sg.fr;
        r.si = g.si;
        r.seg_first = g.j == g.sg.j0;
        r.seg_last = g.j + r.n == g.sg.j1;
        r.whole = g.sg.j0 == 0 && g.sg.j1 == g.sg.nb;
        g.j += r.n;
        if (r.seg_last) {
            g.have = next_seg(g.it, g.sg);
            g.j = g.have ? g.sg.j0 : 0;
            ++g.si;
        }
        return true;
    };
    if (a.early) {
        pdl_wait();
        pdl_release_dependents();
    }
    const float sl = fmaxf(fabsf(a.scale_log2), 1e-30f);  // |scale| log2 e (zero taken as 1e-30)
    const float lazy_raw = kULazyMax / sl;
    bool ok_all = true;

    if (warp == 4) {
        // ================================ producer ================================
        // rows of sequences with no token produce zeros
        for (int r = blockIdx.x; r < B * Hc; r += gridDim.x) {
            const int b = r / Hc;
            if (cum[b + 1] == cum[b]) {
                const int kc = r % Hc;
                for (int j = 0; j < GC; ++j)
                    for (int i = lane; i < kUD; i += 32)
                        store_out<T>(a.out, a.out_f32, ((size_t)b * a.Hq + (size_t)kc * GC + j) * kUD + i, 0.f);
            }
        }
        GIt gi_it;
        git_init(gi_it);
        Grp cur;
        bool hc = next_group(gi_it, cur);
        int pbn = (hc && lane < cur.n) ? a.tables[(size_t)cur.b * a.mbps + cur.j0 + lane] : -1;
        const uint32_t sflip = a.scale_log2 < 0.f ? 0x80008000u : 0u;
        int gi = 0, issued_last = -1;
        while (hc && ok_all) {
            const Grp g = cur;
            const int pb = pbn;
            hc = next_group(gi_it, cur);
            pbn = (hc && lane < cur.n) ? a.tables[(size_t)cur.b * a.mbps + cur.j0 + lane] : -1;
            if (g.seg_first) {
                // q rows of the segment's GC heads into q slot si % 2, once segment si - 2 released it
                const int qs = g.si & 1;
                if (g.si >= 2) {
                    int ok = lane == 0 ? (int)mbar_sleep_wait(&qempty[qs], ((g.si >> 1) - 1) & 1, a.wait_ns) : 0;
                    if (!__shfl_sync(0xffffffffu, ok, 0)) {
                        ok_all = false;
                        break;
                    }
                }
                const uint4 *qg = reinterpret_cast<const uint4 *>(a.q) + ((size_t)g.b * a.Hq + (size_t)g.kc * GC) * (kUD / 8);
                const uint32_t qb = sbase + kUQ + qs * kUQSlot;
#pragma unroll 4
                for (int i = lane; i < GC * 16; i += 32) {
                    const int r = i >> 4, c = i & 15;
                    const uint4 v = __ldg(qg + i);
                    sts128(swz128(qb + (c >> 3) * 64 * 128, r, c & 7), v.x ^ sflip, v.y ^ sflip, v.z ^ sflip, v.w ^ sflip);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&qfull[qs]);
            }
            // K half gi % 2 is free once group gi - 2's QK products have finished (its V
            // half, refilled by warp 6, only once that group's P.V has)
            const int h = gi & 1;
            if (gi >= 2) {
                int ok = lane == 0 ? (int)mbar_sleep_wait(&empty_k[h], ((gi >> 1) - 1) & 1, a.wait_ns) : 0;
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    ok_all = false;
                    break;
                }
            }
            const bool good = lane < g.n && pb >= 0 && (int64_t)pb < a.N;
            const unsigned good_mask = __ballot_sync(0xffffffffu, good);
            const unsigned want = (g.n >= 32 ? 0xffffffffu : ((1u << g.n) - 1u));
            const unsigned bad = want & ~good_mask;
            if (lane == 0) {
                if (bad) raise_flag(PA_EFLAG_BAD_BLOCK);
                const uint32_t bytes = (uint32_t)__popc(good_mask) * 2u * (uint32_t)kUBox;
                if (bytes)
                    mbar_arrive_expect_tx(&full_k[h], bytes);
                else
                    mbar_arrive(&full_k[h]);
            }
            __syncwarp();
            const bool stall = blockIdx.x == 0 && gi == a.stall_at;
            if (good && !stall) {
                const int y = (pb * Hc + g.kc) * kBlockSize;
                const uint32_t slot = (uint32_t)((h * kUGroup + lane) * kUBox);
                const uint32_t bar = smem_addr(&full_k[h]);
                tma_load_2d(sbase + kUK0 + slot, &tmK, 0, y, bar);
                tma_load_2d(sbase + kUK1 + slot, &tmK, 64, y, bar);
            }
            issued_last = gi;
            ++gi;
        }
        if (!ok_all && lane == 0) *abort_flag = 1;
        // no copy may land after the CTA exits: wait (bounded) for the last two groups' copies
        if (lane == 0)
            for (int k = max(0, issued_last - 1); k <= issued_last; ++k)
                mbar_sleep_wait(&full_k[k & 1], (k >> 1) & 1, a.wait_ns);
    } else if (warp == 6) {
        // ============================== V producer ==============================
        // the same groups in the same order: V half gi % 2 once group gi - 2's P.V has finished
        GIt gi_it;
        git_init(gi_it);
        Grp cur;
        bool hc = next_group(gi_it, cur);
        int pbn = (hc && lane < cur.n) ? a.tables[(size_t)cur.b * a.mbps + cur.j0 + lane] : -1;
        int gi = 0, issued_last = -1;
        bool okv = true;
        while (hc) {
            const Grp g = cur;
            const int pb = pbn;
            hc = next_group(gi_it, cur);
            pbn = (hc && lane < cur.n) ? a.tables[(size_t)cur.b * a.mbps + cur.j0 + lane] : -1;
            const int h = gi & 1;
            if (gi >= 2) {
                int ok = lane == 0 ? (int)mbar_sleep_wait(&empty_v[h], ((gi >> 1) - 1) & 1, a.wait_ns) : 0;
                if (!__shfl_sync(0xffffffffu, ok, 0) || *abort_flag) {
                    okv = false;
                    break;
                }
            }
            const bool good = lane < g.n && pb >= 0 && (int64_t)pb < a.N;
            const unsigned good_mask = __ballot_sync(0xffffffffu, good);
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)__popc(good_mask) * 2u * (uint32_t)kUBox;
                if (bytes)
                    mbar_arrive_expect_tx(&full_v[h], bytes);
                else
                    mbar_arrive(&full_v[h]);
            }
            __syncwarp();
            if (good) {
                const int y = (pb * Hc + g.kc) * kBlockSize;
                const uint32_t slot = (uint32_t)((h * kUGroup + lane) * kUBox);
                const uint32_t bar = smem_addr(&full_v[h]);
                tma_load_2d(sbase + kUV0 + slot, &tmV, 0, y, bar);
                tma_load_2d(sbase + kUV1 + slot, &tmV, 64, y, bar);
            }
            issued_last = gi;
            ++gi;
        }
        if (!okv && lane == 0) *abort_flag = 1;
        if (lane == 0)
            for (int k = max(0, issued_last - 1); k <= issued_last; ++k)
                mbar_sleep_wait(&full_v[k & 1], (k >> 1) & 1, a.wait_ns);
    } else if (warp == 5) {
        // ================================ MMA issuer ================================
        GIt gi_it;
        git_init(gi_it);
        Grp cur;
        bool hc = next_group(gi_it, cur);
        const uint32_t id_qk_half = umma_idesc(kFmt, 64, 64, 0);
        const uint32_t id_pv = umma_idesc(kFmt, 64, 128, 1);
        int gi = 0, last_committed = -1, last_qk = -1;
        // QK of group k: S[k % 2] = Q . K^T over the group's 16 n tokens.  poll: only if
        // its tiles (and q) have landed already, else return false without waiting.
        auto issue_qk = [&](const Grp &g, int k, bool poll) -> bool {
            const int h = k & 1;
            int ok;
            if (poll) {
                ok = lane == 0 ? (int)(mbar_try_wait(&full_k[h], (k >> 1) & 1) &&
                                       (!g.seg_first || mbar_try_wait(&qfull[g.si & 1], (g.si >> 1) & 1)))
                               : 0;
            } else {
                ok = lane == 0 ? (int)mbar_sleep_wait(&full_k[h], (k >> 1) & 1, a.wait_ns) : 0;
                if (ok && g.seg_first && lane == 0) ok = mbar_sleep_wait(&qfull[g.si & 1], (g.si >> 1) & 1, a.wait_ns);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return false;
            tc_fence_after();
            if (lane == 0) {
                // blocks 0-3 of the group into lane tile 0 (TMEM lanes 0-15 of each quadrant),
                // blocks 4-7 into lane tile 1 (lanes 16-31)
                const uint32_t qb = sbase + kUQ + (g.si & 1) * kUQSlot;
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    const int nt = tile == 0 ? min(g.n, 4) : g.n - 4;
                    if (nt <= 0) break;
                    const uint32_t id = nt == 4 ? id_qk_half : umma_idesc(kFmt, 64, 16 * nt, 0);
                    const uint32_t kb = (uint32_t)((h * kUGroup + 4 * tile) * kUBox);
                    const uint32_t d = tmem + (uint32_t)(k & 1) * 64u + ((uint32_t)(16 * tile) << 16);
#pragma unroll
                    for (int ks = 0; ks < kUD / 16; ++ks) {
                        const uint32_t qa = qb + (ks >> 2) * 64 * 128 + (ks & 3) * 32;
                        const uint32_t ka = sbase + ((ks >> 2) ? kUK1 : kUK0) + kb + (ks & 3) * 32;
                        umma_f16(d, umma_sdesc(qa, 16, 1024), umma_sdesc(ka, 16, 1024), id, ks > 0);
                    }
                }
                umma_commit(&s_ready[k & 1]);
                umma_commit(&empty_k[h]);  // the K half may be refilled once these products finish
            }
            __syncwarp();
            last_qk = k;
            return true;
        };
        bool ok = hc ? issue_qk(cur, 0, false) : true;
        while (hc && ok) {
            const Grp g = cur;
            const int k = gi;
            hc = next_group(gi_it, cur);
            // the next group's scores while the softmax works on this one, if its tiles are
            // already in; P.V of this group never waits for the next group's copies (their
            // ring half is refilled only after an earlier P.V)
            bool qk_next = hc && issue_qk(cur, k + 1, true);
            int okp = lane == 0 ? (int)(mbar_sleep_wait(&p_ready[k & 1], (k >> 1) & 1, a.wait_ns) &&
                                        mbar_sleep_wait(&full_v[k & 1], (k >> 1) & 1, a.wait_ns))
                                : 0;
            okp = __shfl_sync(0xffffffffu, okp, 0);
            if (!okp) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t pb = sbase + kUP + (SPLIT ? 0 : (k & 1) * kUPBuf);
                for (int t = 0; t < g.n; ++t) {  // K = 16 tokens: block t of the group
                    const uint32_t pa = pb + (t >> 2) * 64 * 128 + (t & 3) * 32;
                    const uint32_t slot = (uint32_t)(((k & 1) * kUGroup + t) * kUBox);
                    const uint32_t acc = (g.seg_first && t == 0) ? 0u : 1u;
                    // block t's V as one MN-major operand of N = 128 dims: 64 dims per 128-byte
                    // swizzle atom, the atom of dims 64-127 one ring region further (the
                    // leading byte offset), 8-token groups 1024 bytes apart; O in lane tile 0
                    const uint64_t vd = umma_sdesc(sbase + kUV0 + slot, kUV1 - kUV0, 1024);
                    umma_f16(tmem + 128u, umma_sdesc(pa, 16, 1024), vd, id_pv, acc);
                    if (SPLIT) umma_f16(tmem + 128u, umma_sdesc(pa + kUPBuf, 16, 1024), vd, id_pv, 1u);
                }
                umma_commit(&pv_done[k & 1]);
                umma_commit(&empty_v[k & 1]);
                if (g.seg_last) umma_commit(&qempty[g.si & 1]);
            }
            __syncwarp();
            last_committed = k;
            ++gi;
            if (hc && !qk_next) {
                ok = issue_qk(cur, k + 1, false);
                if (!ok) break;
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
        // every MMA this warp issued has finished before the TMEM is released (a commit
        // covers all earlier MMAs of the thread; a QK issued after the last P.V has its own)
        if (lane == 0 && last_committed >= 0)
            mbar_sleep_wait(&pv_done[last_committed & 1], (last_committed >> 1) & 1, a.wait_ns);
        if (lane == 0 && last_qk > last_committed) mbar_sleep_wait(&s_ready[last_qk & 1], (last_qk >> 1) & 1, a.wait_ns);
    } else {
        // ============================ softmax and epilogue ============================
        // thread (w, l): head row 16w + (l & 15); lane tile l >> 4 holds tokens 64 (l >> 4) ..
        // + 63 of the group's S and dims 64 (l >> 4) .. + 63 of O for that row
        const int row = warp * 16 + (lane & 15);
        const int half = lane >> 4;
        const bool warp_on = warp * 16 < GC;  // the warp holds real head rows
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        GIt gi_it;
        git_init(gi_it);
        Grp g, gn;
        bool hn = next_group(gi_it, gn);
        // the group's table entries, loaded a group ahead: which of its blocks lie
        // outside the pool (their scores are masked and their V rows zeroed)
        int pbn = (hn && lane < gn.n) ? a.tables[(size_t)gn.b * a.mbps + gn.j0 + lane] : -1;
        int gi = 0;
        float m = -INFINITY, l = 0.f;  // l: this thread's half of the row's sum
        bool alive = true;
        while (hn) {
            g = gn;
            const int pbg = pbn;
            hn = next_group(gi_it, gn);
            pbn = (hn && lane < gn.n) ? a.tables[(size_t)gn.b * a.mbps + gn.j0 + lane] : -1;
            const int n = g.n;
            const unsigned want = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
            const unsigned bad = want & ~__ballot_sync(0xffffffffu, lane < n && pbg >= 0 && (int64_t)pbg < a.N);
            const int ntok_last = (g.j0 + n == g.nb) ? g.L - (g.nb - 1) * kBlockSize : kBlockSize;
            if (g.seg_first) {
                m = -INFINITY;
                l = 0.f;
            }
            const int h = gi & 1;
            if (alive) {
                // S ready implies the group's K tiles landed.  (No wait on the K barrier
                // itself: it may already have moved on to group gi + 2, whose copies start
                // as soon as this group's QK products are done.)
                const bool okf = mbar_sleep_wait(&s_ready[h], (gi >> 1) & 1, a.wait_ns);
                if (!__all_sync(0xffffffffu, okf) || *abort_flag) {
                    alive = false;
                    *abort_flag = 1;
                }
            }
            if (alive && warp_on) {
                tc_fence_after();
                float x[64];
                tmem_ld64(tmem + lane_base + (uint32_t)h * 64u, x);
                tmem_wait_ld();
                // mask tokens past the row's end, of skipped blocks and past the group
                if (n != kUGroup || bad != 0u || ntok_last != kBlockSize) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int t = 4 * half + (j >> 4);  // block of the group
                        const bool valid = t < n && !((bad >> t) & 1u) && !(t == n - 1 && (j & 15) >= ntok_last);
                        x[j] = valid ? x[j] : -INFINITY;
                    }
                }
                float mq[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    mq[q] = x[8 * q];
#pragma unroll
                    for (int j = 1; j < 8; ++j) mq[q] = fmaxf(mq[q], x[8 * q + j]);
                }
                float mx = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])),
                                 fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                // ---- lazy maximum: move it (and rescale O) only when a score exceeds it by
                // more than 2^8 in probability; O holds nothing yet on a segment's first group
                const bool grow = mx > m + lazy_raw;
                if (__any_sync(0xffffffffu, grow)) {
                    const float mn = grow ? fmaxf(m, mx) : m;
                    const float al = (grow && m != -INFINITY) ? fast_exp2((m - mn) * sl) : 1.f;
                    if (!g.seg_first) {
                        // the previous group's P.V must have finished with O
                        const int kp = gi - 1;
                        const bool okw = mbar_sleep_wait(&pv_done[kp & 1], (kp >> 1) & 1, a.wait_ns);
                        if (!__all_sync(0xffffffffu, okw)) {
                            alive = false;
                            *abort_flag = 1;
                        } else {
                            tc_fence_after();
#pragma unroll
                            for (int q = 0; q < 4; ++q) {  // O: 128 columns, rows in lane tile 0
                                float v[32];
                                tmem_ld32(tmem + lane_base + 128u + (uint32_t)q * 32u, v);
                                tmem_wait_ld();
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] *= al;
                                tmem_st32(tmem + lane_base + 128u + (uint32_t)q * 32u, v);
                            }
                            tmem_wait_st();
                        }
                    }
                    l *= al;
                    m = mn;
                }
                if (alive && gi >= (SPLIT ? 1 : 2)) {
                    // P buffer gi % 2 was last read by group gi - 2's P.V (bf16: both
                    // buffers, by group gi - 1's)
                    const int kp = gi - (SPLIT ? 1 : 2);
                    const bool okw = mbar_sleep_wait(&pv_done[kp & 1], (kp >> 1) & 1, a.wait_ns);
                    if (!__all_sync(0xffffffffu, okw)) {
                        alive = false;
                        *abort_flag = 1;
                    }
                }
                if (alive) {
                    // ---- this thread's 64 probabilities of its row, p = 2^((s - m) c)
                    const uint32_t pbuf = sbase + kUP + (SPLIT ? 0u : (uint32_t)h * kUPBuf) + (uint32_t)half * 64 * 128;
                    const float ms = m * sl;
                    if (row < GC) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {  // 16-byte chunk c: tokens 64 half + 8c .. + 7
                            float p[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float xv = x[8 * c + e];
                                p[e] = xv == -INFINITY ? 0.f : fast_exp2(fmaf(xv, sl, -ms));
                            }
                            l += ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
                            uint32_t hw[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) hw[e] = pack2<T>(p[2 * e], p[2 * e + 1]);
                            const uint32_t dst = swz128(pbuf, row, c);
                            sts128(dst, hw[0], hw[1], hw[2], hw[3]);
                            if (SPLIT) {
                                uint32_t lw[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    lw[e] = pack2<T>(p[2 * e] - __uint_as_float(hw[e] << 16),
                                                     p[2 * e + 1] - __uint_as_float(hw[e] & 0xffff0000u));
                                sts128(dst + kUPBuf, lw[0], lw[1], lw[2], lw[3]);
                            }
                        }
                    }
                }
            }
            if (alive) {
                // ---- stale V rows of the row's last block and of skipped blocks weigh 0 in
                // P; zero them, as 0 x NaN would poison the product
                if (bad != 0u || ntok_last != kBlockSize) {
                    // the V tiles must have landed before their stale rows are zeroed
                    const bool okv = mbar_sleep_wait(&full_v[h], (gi >> 1) & 1, a.wait_ns);
                    if (!__all_sync(0xffffffffu, okv)) {
                        alive = false;
                        *abort_flag = 1;
                    }
                    for (int t = 0; alive && t < n; ++t) {
                        const int r0 = ((bad >> t) & 1u) ? 0 : (t == n - 1 ? ntok_last : kBlockSize);
                        const int nz = (kBlockSize - r0) * 16;  // 16-byte chunks over both boxes
                        for (int i = tid; i < nz; i += 128) {
                            const int r = r0 + (i >> 4), c = i & 15;
                            const uint32_t vb = sbase + ((c >> 3) ? kUV1 : kUV0) + (uint32_t)((h * kUGroup + t) * kUBox);
                            sts128(swz128(vb, r, c & 7), 0u, 0u, 0u, 0u);
                        }
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&p_ready[h]);
            }
            // ---- segment end: this thread's 64 dims of its row of O to the output or the
            // workspace
            if (g.seg_last) {
                // O rows sit in lane tile 0: threads of half 0 write all 128 dims of their row,
                // 64 at a time (half 1 reads lanes that hold nothing it uses)
                float lse = -INFINITY, inv = 0.f;
                bool have_o = false;
                if (alive) {
                    const bool okw = mbar_sleep_wait(&pv_done[gi & 1], (gi >> 1) & 1, a.wait_ns);
                    if (!__all_sync(0xffffffffu, okw)) {
                        alive = false;
                        *abort_flag = 1;
                    } else if (warp_on) {
                        const float lr = l + __shfl_xor_sync(0xffffffffu, l, 16);  // the row's sum
                        inv = lr > 0.f ? 1.f / lr : 0.f;
                        lse = m * sl + log2f(lr);
                        have_o = true;
                    }
                }
                const bool writer = warp_on && row < GC && half == 0;
                size_t obase = 0;
                float *wbase = nullptr;
                if (g.whole) {
                    obase = ((size_t)g.b * a.Hq + (size_t)g.kc * GC + row) * kUD;
                } else {
                    const int ch_first = ck.of(g.b, g.kc, g.nb, 0);
                    const int slot = 2 * g.ch + ((g.ch == ch_first && ck.mid_start(g.b, g.kc, g.nb)) ? 1 : 0);
                    wbase = a.ws_o + ((size_t)slot * GC + row) * kUD;
                    if (writer) a.ws_lse[(size_t)slot * GC + row] = lse;
                }
                if (have_o) tc_fence_after();
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    float o[64];
                    if (have_o) {
                        tmem_ld64(tmem + lane_base + 128u + (uint32_t)c2 * 64u, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 64; ++j) o[j] *= inv;
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) o[j] = 0.f;
                    }
                    if (writer) {
                        if (g.whole) {
#pragma unroll
                            for (int j = 0; j < 64; j += 2)
                                store_out2<T>(a.out, a.out_f32, obase + 64 * c2 + j, o[j], o[j + 1]);
                        } else {
                            float4 *w = reinterpret_cast<float4 *>(wbase + 64 * c2);
#pragma unroll
                            for (int j = 0; j < 16; ++j) w[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                        }
                    }
                }
            }
            ++gi;
        }
    }
    // all roles done: release the tensor memory (its last MMA finished, see the issuer)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols));
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// (up to 2048 sequences: the per-CTA prefix sums share the SM's shared memory with the
// rings)
constexpr int kUMaxB = 2048;
bool decode_umma_eligible(int q_dtype, int kv_dtype, int D, int G, int ngroups, int qlen, bool padded, int part,
                          int B) {
    return (q_dtype == PA_F16 || q_dtype == PA_BF16) && kv_dtype == q_dtype && D == kUD && G == 8 &&
           (ngroups == 4 || ngroups == 8) && qlen == 1 && !padded && part != 0 && B <= kUMaxB;
}

template <typename T, int GC>
static int launch_umma(const DecodeArgs &a, cudaStream_t st) {
    auto kern = decode_umma_kernel<T, GC>;
    DecodeArgs a2 = a;
    a2.Hkv = a.Hkv / a.ngroups;  // cache rows; GC columns each
    a2.ngroups = 1;
    a2.G = GC;
    a2.gcols = GC;
    const int smem = umma_smem_bytes(a.B);
    if (a.B > kUMaxB) return PA_ERR_UNSUPPORTED;
    if (!set_smem_attr_once(reinterpret_cast<const void *>(kern), umma_smem_bytes(kUMaxB))) return PA_ERR_CUDA;
    if ((uintptr_t)a.q % 16) return PA_ERR_ALIGN;
    CUtensorMap tk, tv;
    const int64_t rows = a.N * a2.Hkv * kBlockSize;
    if (!tc_cache_tensor_map(&tk, a.kc, rows, kUD, a.kv_dtype) || !tc_cache_tensor_map(&tv, a.vc, rows, kUD, a.kv_dtype))
        return PA_ERR_CUDA;
    int sms = 0, per_sm = 0;
    if (!tc_launch_shape(reinterpret_cast<const void *>(kern), kUThreads, smem, &sms, &per_sm)) return PA_ERR_CUDA;
    const int64_t blocks = (int64_t)a.B * a2.Hkv * ((a.max_len + kBlockSize - 1) / kBlockSize);
    int64_t ctas = (int64_t)sms;  // one CTA per SM: its shared memory and TMEM take the SM
    const int64_t need = (blocks + kTcMinChunk - 1) / kTcMinChunk;
    if (need < ctas) ctas = need;
    if (ctas < 1) ctas = 1;
    a2.tc_W = (int)ctas;
    if (launch_pdl(kern, dim3((unsigned)ctas), dim3(kUThreads), smem, st, tk, tv, a2) != cudaSuccess)
        return PA_ERR_CUDA;
    return launch_merge_rows(a2, sms, st);
}

int launch_decode_umma(const DecodeArgs &a, cudaStream_t st) {
    const int GC = a.G * a.ngroups;
    if (a.q_dtype == PA_F16) return GC == 32 ? launch_umma<__half, 32>(a, st) : launch_umma<__half, 64>(a, st);
    if (a.q_dtype == PA_BF16)
        return GC == 32 ? launch_umma<__nv_bfloat16, 32>(a, st) : launch_umma<__nv_bfloat16, 64>(a, st);
    return PA_ERR_DTYPE;
}

}  // namespace pa
