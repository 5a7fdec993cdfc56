// Paged decode attention, CUDA-core ("SIMT") kernel family.
//
// What it computes (lqnn.cn/news/235768 sections 1.2, 2.2, 3.2, 4.2;
// chanyi.net.cn/article/49 section 四): for every sequence b and query head h,
//   out[b][h] = sum_t softmax_t(scale * q[b][h] . K[b][t]) V[b][t]
// over the logical tokens of b, walking its block table, one CTA per
// (partition, KV head, sequence) serving the whole GQA group of G query heads
// from one read of the K/V tiles.
//
// Structure:
//   * 4 warps; warp w takes the 16-token blocks w, w+4, w+8, ... of the
//     partition, each with a private 2-stage ring in shared memory filled by
//     bulk asynchronous copies (cp.async.bulk, one 16 x d tile of K and one of
//     V per stage, completion on an mbarrier).  A (block, KV head) tile is
//     contiguous in the cache layout, so each stage is two 16-byte-aligned
//     bulk copies issued by one lane.
//   * QK: LPT lanes share one token; each holds DPL dims of the G query rows
//     in registers (pre-scaled by scale * log2 e) and the G partial dot
//     products are reduced with a transposing butterfly (log2 LPT shuffles
//     per token group) that leaves each lane with one head's score.
//   * online softmax in the log2 domain, fp32: running max / sum per head,
//     probabilities passed to the PV step through a 16 x G buffer per warp.
//   * PV: each lane owns D/32 output dims of all G heads.
//   * the 4 warps' (m, l, o) are merged through shared memory at the end; a
//     single-partition sequence writes out directly, otherwise the normalised
//     partial output and its log2-sum-exp go to the workspace for the merge.
// int8 caches: the K scale multiplies the reduced score, the V scale the
// probabilities fed to PV; the sum l uses the unscaled probabilities.
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

PA_ERROR_WORD_ACCESSOR(error_word_decode_simt)

template <typename TKV, int D, int G>
struct SimtCfg {
    static constexpr int NW = 4;
    static constexpr int THREADS = NW * 32;
    static constexpr int STAGES = 2;
    static constexpr int E = sizeof(TKV);
    static constexpr int TILE = kBlockSize * D * E;  // bytes of one (block, head) tile
    static constexpr int STAGE_BYTES = 2 * TILE;     // K tile then V tile
    static constexpr int DPL = (G <= 4) ? 16 : 8;    // dims per lane in QK
    static constexpr int LPT = D / DPL;              // lanes per token in QK
    static constexpr int TPP = 32 / LPT;             // tokens per pass
    static constexpr int PASSES = kBlockSize / TPP;
    static constexpr int DPV = D / 32;               // dims per lane in PV
    static constexpr int RING = NW * STAGES * STAGE_BYTES;
    static constexpr int COMBINE = NW * G * (D + 2) * 4;
    static constexpr int REGION0 = RING > COMBINE ? RING : COMBINE;
    static constexpr int P_OFF = REGION0;                          // float [NW][16][G]
    static constexpr int A_OFF = P_OFF + NW * kBlockSize * G * 4;  // float [NW][G]
    static constexpr int BAR_OFF = ((A_OFF + NW * G * 4) + 7) / 8 * 8;  // u64 [NW][STAGES]
    static constexpr int BLK_OFF = BAR_OFF + NW * STAGES * 8;        // int [NW][STAGES]
    static constexpr int SMEM = BLK_OFF + NW * STAGES * 4;
    static_assert(G <= LPT, "group larger than lanes per token");
    static_assert(TILE % 16 == 0, "tile must be a multiple of 16 bytes");
};

// Head index a lane holds after reduce_heads().
template <int G, int LPT>
__device__ __forceinline__ int head_of_lane(int j) {
    int h = 0;
#pragma unroll
    for (int cnt = G, mask = LPT / 2; cnt > 1; cnt >>= 1, mask >>= 1)
        if (j & mask) h += cnt >> 1;
    return h;
}

// Sum G partial dot products over the LPT lanes of a token group; the lane
// ends with the full sum for head head_of_lane(j).  Each halving step trades
// half of the values with the partner lane, so G values cost G-1 shuffles
// plus log2(LPT/G) plain steps.
template <int G, int LPT>
__device__ __forceinline__ float reduce_heads(float (&v)[G], int j) {
#pragma unroll
    for (int cnt = G, mask = LPT / 2; cnt > 1; cnt >>= 1, mask >>= 1) {
        const int half = cnt >> 1;
        const bool up = (j & mask) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
    }
#pragma unroll
    for (int mask = LPT / (2 * G); mask >= 1; mask >>= 1)
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
    return v[0];
}

__device__ __forceinline__ int effective_len(const DecodeArgs &a, int b) {
    int L = a.lens[b];
    L = min(L, a.max_len);
    return min(L, a.mbps * kBlockSize);
}

template <typename TQ, typename TKV, int D, int G>
__global__ void __launch_bounds__(128) decode_simt_kernel(const DecodeArgs a) {
    using C = SimtCfg<TKV, D, G>;
    constexpr int NW = C::NW, STAGES = C::STAGES, TILE = C::TILE, DPL = C::DPL, LPT = C::LPT,
                  TPP = C::TPP, PASSES = C::PASSES, DPV = C::DPV;
    extern __shared__ __align__(128) unsigned char smem[];
    float *p_s = reinterpret_cast<float *>(smem + C::P_OFF);
    float *alpha_s = reinterpret_cast<float *>(smem + C::A_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    int *stage_blk = reinterpret_cast<int *>(smem + C::BLK_OFF);

    const int part = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_release_dependents();
    const int L = effective_len(a, b);
    const int P = a.part > 0 ? a.part : max(L, 1);
    const int t0 = part * P;
    const size_t out0 = ((size_t)b * a.Hq + (size_t)kvh * G) * D;  // first element of the group's rows
    if (L <= 0) {
        if (part == 0)
            for (int i = threadIdx.x; i < G * D; i += blockDim.x) store_out<TQ>(a.out, a.out_f32, out0 + i, 0.f);
        return;
    }
    if (t0 >= L) return;
    const int t1 = min(L, t0 + P);
    const int nblk = ceil_div(t1 - t0, kBlockSize);
    const int ntok_last = t1 - t0 - (nblk - 1) * kBlockSize;
    const int nparts = ceil_div(L, P);
    const int32_t *table = a.tables + (size_t)b * a.mbps + t0 / kBlockSize;

    // q rows of the group, this lane's DPL dims, scaled into the log2 domain
    const int grp = lane / LPT, j = lane % LPT;
    float qr[G][DPL];
    {
        const TQ *qp = reinterpret_cast<const TQ *>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * G) * D;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < DPL; ++i) qr[h][i] = Cvt<TQ>::to_f(qp[h * D + j * DPL + i]) * a.scale_log2;
    }

    uint64_t *my_bars = bars + warp * STAGES;
    int *my_blk = stage_blk + warp * STAGES;
    unsigned char *my_ring = smem + warp * STAGES * C::STAGE_BYTES;
    const int my_nblk = nblk > warp ? ceil_div(nblk - warp, NW) : 0;

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();

    // lane 0: start the copy of this warp's it-th block into stage it % STAGES
    int issued = 0;  // lane 0: blocks whose copy was started
    auto issue = [&](int it) {
        const int s = it % STAGES;
        issued = it + 1;
        const int pb = table[warp + it * NW];
        if (pb < 0 || (int64_t)pb >= a.N) {
            my_blk[s] = -1;
            raise_flag(PA_EFLAG_BAD_BLOCK);
            mbar_arrive(&my_bars[s]);
            return;
        }
        my_blk[s] = pb;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&my_bars[s], 2 * TILE);
        const size_t off = ((size_t)pb * (a.Hkv / a.ngroups) + (kvh / a.ngroups)) * TILE;
        bulk_g2s(my_ring + s * C::STAGE_BYTES, reinterpret_cast<const char *>(a.kc) + off, TILE, &my_bars[s]);
        bulk_g2s(my_ring + s * C::STAGE_BYTES + TILE, reinterpret_cast<const char *>(a.vc) + off, TILE,
                 &my_bars[s]);
    };
    if (lane == 0)
        for (int it = 0; it < STAGES && it < my_nblk; ++it) issue(it);

    const int hj = head_of_lane<G, LPT>(j);
    const bool writer = (j & (LPT / G - 1)) == 0;  // one of the lanes holding head hj
    float m_run = -INFINITY, l_run = 0.f;
    float o[G][DPV];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPV; ++i) o[h][i] = 0.f;
    float *pw = p_s + warp * kBlockSize * G;

    for (int it = 0; it < my_nblk; ++it) {
        const int s = it % STAGES;
        const uint32_t parity = (it / STAGES) & 1;
        int ok = lane == 0 ? (int)mbar_wait(&my_bars[s], parity, a.wait_ns) : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            // a copy did not land in time: wait (bounded again) for the copies still in
            // flight, so that none lands in shared memory reused below or after exit
            if (lane == 0)
                for (int k = it; k < issued; ++k) mbar_wait(&my_bars[k % STAGES], (k / STAGES) & 1, a.wait_ns);
            __syncwarp();
            break;
        }
        if (lane != 0) mbar_wait(&my_bars[s], parity, a.wait_ns);  // completed: acquires the copied data
        const int jb = warp + it * NW;
        const int pb = my_blk[s];
        const int ntok = (jb == nblk - 1) ? ntok_last : kBlockSize;
        const unsigned char *Ks = my_ring + s * C::STAGE_BYTES;
        const unsigned char *Vs = Ks + TILE;
        if (pb >= 0) {
            float ksc = 1.f, vsc = 1.f;
            if constexpr (sizeof(TKV) == 1) {
                const size_t si = (size_t)pb * (a.Hkv / a.ngroups) + (kvh / a.ngroups);
                ksc = a.ks[si];
                vsc = a.vs[si];
            }
            // ---- scores of the 16 tokens, lane holds (token pass*TPP+grp, head hj)
            float sc[PASSES];
#pragma unroll
            for (int pass = 0; pass < PASSES; ++pass) {
                const int tk = pass * TPP + grp;
                uint32_t w[DPL * C::E / 4];
                lds<DPL * C::E>(Ks + (tk * D + j * DPL) * C::E, w);
                float kf[DPL];
                to_float<TKV, DPL>(w, kf);
                float acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = 0.f;
#pragma unroll
                    for (int i = 0; i < DPL; ++i) x = fmaf(qr[h][i], kf[i], x);
                    acc[h] = x;
                }
                const float r = reduce_heads<G, LPT>(acc, j) * ksc;
                sc[pass] = tk < ntok ? r : -INFINITY;
            }
            // ---- online softmax for head hj
            float bmax = sc[0];
#pragma unroll
            for (int pass = 1; pass < PASSES; ++pass) bmax = fmaxf(bmax, sc[pass]);
#pragma unroll
            for (int mask = LPT; mask < 32; mask <<= 1)
                bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, mask));
            const float m_new = fmaxf(m_run, bmax);
            const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
            float psum = 0.f;
#pragma unroll
            for (int pass = 0; pass < PASSES; ++pass) {
                const float p = fast_exp2(sc[pass] - m_new);
                psum += p;
                if (writer) pw[(pass * TPP + grp) * G + hj] = p * vsc;
            }
            l_run = l_run * alpha + psum;
            m_run = m_new;
            if (writer && grp == 0) alpha_s[warp * G + hj] = alpha;
            __syncwarp();
            // ---- o = alpha o + P V
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float al = alpha_s[warp * G + h];
#pragma unroll
                for (int i = 0; i < DPV; ++i) o[h][i] *= al;
            }
            for (int tk = 0; tk < ntok; ++tk) {
                float pv[G];
#pragma unroll
                for (int h = 0; h < G; ++h) pv[h] = pw[tk * G + h];
                uint32_t w[(DPV * C::E + 3) / 4];
                lds<DPV * C::E>(Vs + (tk * D + lane * DPV) * C::E, w);
                float vf[DPV];
                to_float<TKV, DPV>(w, vf);
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int i = 0; i < DPV; ++i) o[h][i] = fmaf(pv[h], vf[i], o[h][i]);
            }
        }
        __syncwarp();
        if (lane == 0 && it + STAGES < my_nblk) issue(it + STAGES);
    }

    // l for head hj: sum over the token groups (duplicate lanes hold equal values)
#pragma unroll
    for (int mask = LPT; mask < 32; mask <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, mask);

    // ---- merge the 4 warps
    __syncthreads();
    float *cm = reinterpret_cast<float *>(smem);
    float *cl = cm + NW * G;
    float *co = cl + NW * G;
    if (writer && grp == 0) {
        cm[warp * G + hj] = m_run;
        cl[warp * G + hj] = l_run;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPV; ++i) co[(warp * G + h) * D + lane * DPV + i] = o[h][i];
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, dim = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, cm[w * G + h]);
        float Ls = 0.f, Os = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = cm[w * G + h];
            const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
            Ls = fmaf(cl[w * G + h], f, Ls);
            Os = fmaf(co[(w * G + h) * D + dim], f, Os);
        }
        if (nparts == 1) {
            store_out<TQ>(a.out, a.out_f32, out0 + h * D + dim, Os / Ls);
        } else {
            const size_t row = ((size_t)b * a.Hq + (size_t)kvh * G + h) * a.max_parts + part;
            a.ws_o[row * D + dim] = Os / Ls;
            if (dim == 0) a.ws_lse[row] = M + log2f(Ls);
        }
    }
}

// Log-sum-exp merge of the partitions of every (sequence, query head) with more
// than one partition:  M = max lse_p, out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M).
template <typename TQ>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeArgs a) {
    const int qh = blockIdx.x, b = blockIdx.y;
    pdl_wait();  // the partials of the decode kernel before it
    pdl_release_dependents();
    const int L = effective_len(a, b);
    if (L <= a.part) return;  // one partition (or none): written by the decode kernel
    const int np = ceil_div(L, a.part);
    const size_t row = ((size_t)b * a.Hq + qh) * a.max_parts;
    const float *lse = a.ws_lse + row;
    float M = -INFINITY;
    for (int p = 0; p < np; ++p) M = fmaxf(M, lse[p]);
    const size_t out0 = ((size_t)b * a.Hq + qh) * a.D;
    for (int dim = threadIdx.x; dim < a.D; dim += blockDim.x) {
        float S = 0.f, acc = 0.f;
        for (int p = 0; p < np; ++p) {
            const float w = fast_exp2(lse[p] - M);
            S += w;
            acc = fmaf(w, a.ws_o[(row + p) * a.D + dim], acc);
        }
        store_out<TQ>(a.out, a.out_f32, out0 + dim, acc / S);
    }
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int max_len, int part) {
    if (part <= 0 || max_len <= part) return 0;
    const size_t mp = (size_t)((max_len + part - 1) / part);
    const size_t o = (size_t)B * Hq * mp * D * sizeof(float);
    const size_t lse = (size_t)B * Hq * mp * sizeof(float);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up(o) + up(lse);
}

template <typename TQ, typename TKV, int D, int G>
static int launch_one(const DecodeArgs &a, cudaStream_t st) {
    using C = SimtCfg<TKV, D, G>;
    auto kern = decode_simt_kernel<TQ, TKV, D, G>;
    if (!set_smem_attr_once(reinterpret_cast<const void *>(kern), C::SMEM)) return PA_ERR_CUDA;
    const int parts = a.part > 0 ? a.max_parts : 1;
    dim3 grid((unsigned)parts, (unsigned)a.Hkv, (unsigned)a.B);
    if (launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM, st, a) != cudaSuccess) return PA_ERR_CUDA;
    if (a.part > 0 && a.max_parts > 1) {
        if (launch_pdl(merge_kernel<TQ>, dim3((unsigned)a.Hq, (unsigned)a.B), dim3(128), 0, st, a) != cudaSuccess)
            return PA_ERR_CUDA;
    }
    return PA_OK;
}

template <typename TQ, typename TKV, int D>
static int launch_g(const DecodeArgs &a, cudaStream_t st) {
    switch (a.G) {
    case 1: return launch_one<TQ, TKV, D, 1>(a, st);
    case 2: return launch_one<TQ, TKV, D, 2>(a, st);
    case 4: return launch_one<TQ, TKV, D, 4>(a, st);
    case 8: return launch_one<TQ, TKV, D, 8>(a, st);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename TQ, typename TKV>
static int launch_d(const DecodeArgs &a, cudaStream_t st) {
    switch (a.D) {
    case 64: return launch_g<TQ, TKV, 64>(a, st);
    case 128: return launch_g<TQ, TKV, 128>(a, st);
    case 256:
        if constexpr (sizeof(TKV) <= 2) return launch_g<TQ, TKV, 256>(a, st);
        return PA_ERR_UNSUPPORTED;  // a 4-byte 256-dim ring does not fit shared memory
    default: return PA_ERR_UNSUPPORTED;
    }
}

bool decode_simt_supported(int q_dtype, int kv_dtype, int D, int G) {
    const bool pair_ok = (q_dtype == PA_F32 && kv_dtype == PA_F32) ||
                         (q_dtype == PA_F16 && (kv_dtype == PA_F16 || kv_dtype == PA_I8)) ||
                         (q_dtype == PA_BF16 && (kv_dtype == PA_BF16 || kv_dtype == PA_I8));
    const bool d_ok = D == 64 || D == 128 || (D == 256 && kv_dtype != PA_F32);
    return pair_ok && d_ok && (G == 1 || G == 2 || G == 4 || G == 8);
}

int launch_decode_simt(const DecodeArgs &a, cudaStream_t st) {
    if (a.q_dtype == PA_F32 && a.kv_dtype == PA_F32) return launch_d<float, float>(a, st);
    if (a.q_dtype == PA_F16 && a.kv_dtype == PA_F16) return launch_d<__half, __half>(a, st);
    if (a.q_dtype == PA_BF16 && a.kv_dtype == PA_BF16) return launch_d<__nv_bfloat16, __nv_bfloat16>(a, st);
    if (a.q_dtype == PA_F16 && a.kv_dtype == PA_I8) return launch_d<__half, int8_t>(a, st);
    if (a.q_dtype == PA_BF16 && a.kv_dtype == PA_I8) return launch_d<__nv_bfloat16, int8_t>(a, st);
    return PA_ERR_DTYPE;
}

}  // namespace pa
