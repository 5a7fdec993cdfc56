// Cache-side kernels: append scatter, copy-on-write block copy, int8 quantiser.
//
// All three are pure data movement (plus one absmax reduction): HBM-bound,
// written with 16-byte vector accesses where alignment allows, one CTA per
// independent row group so the grid scales with the work.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

PA_ERROR_WORD_ACCESSOR(error_word_cache_ops)

// ---------------------------------------------------------------------------
// reshape_and_cache: token i, KV head h -> slot s = slot_mapping[i]
// (lqnn.cn/news/235768 section 2.2: append at cache_len, then attend).
// Grid: (num_tokens, 2) -- y selects K or V.  Each CTA copies the H_kv rows of
// one token with VEC-byte accesses.
// ---------------------------------------------------------------------------
//
// overlap (PA_APPEND_OVERLAP_PREVIOUS): the caller guarantees that no kernel still
// running before this one reads or writes the slots written here.  The next kernel
// may then launch at once and the copies run while the previous kernel finishes;
// CTA (0, 0) waits for the previous kernel before it exits, so this grid still
// completes after it and a kernel that waits for this one finds every earlier one
// complete.
template <int VEC>
__device__ __forceinline__ void reshape_and_cache_body(
    const char *__restrict__ k, const char *__restrict__ v, char *__restrict__ kc,
    char *__restrict__ vc, const int64_t *__restrict__ slots, int num_kv_heads, int row_bytes,
    int64_t k_stride_bytes, int64_t v_stride_bytes, int64_t num_slots) {
    using V = typename VecT<VEC>::type;
    const int64_t i = blockIdx.x;
    const bool is_v = blockIdx.y != 0;
    const char *src = (is_v ? v : k) + i * (is_v ? v_stride_bytes : k_stride_bytes);
    const int vecs_per_row = row_bytes / VEC;
    const int total = num_kv_heads * vecs_per_row;
    auto src_vec = [&](int idx) {
        const int h = idx / vecs_per_row, c = idx % vecs_per_row;
        return reinterpret_cast<const V *>(src + (int64_t)h * row_bytes)[c];
    };
    // The token's row does not depend on its slot: its first vector is requested
    // together with the slot, so the two loads overlap.
    V first{};
    if ((int)threadIdx.x < total) first = src_vec(threadIdx.x);
    const int64_t s = slots[i];
    if (s < 0) return;
    if (s >= num_slots) {
        if (threadIdx.x == 0 && blockIdx.y == 0) raise_flag(PA_EFLAG_BAD_SLOT);
        return;
    }
    char *dst = is_v ? vc : kc;
    const int64_t blk = s / kBlockSize, off = s % kBlockSize;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int h = idx / vecs_per_row, c = idx % vecs_per_row;
        const int64_t drow = ((blk * num_kv_heads + h) * kBlockSize + off) * (int64_t)row_bytes;
        reinterpret_cast<V *>(dst + drow)[c] = idx == (int)threadIdx.x ? first : src_vec(idx);
    }
}

template <int VEC>
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const char *__restrict__ k, const char *__restrict__ v, char *__restrict__ kc,
    char *__restrict__ vc, const int64_t *__restrict__ slots, int num_kv_heads, int row_bytes,
    int64_t k_stride_bytes, int64_t v_stride_bytes, int64_t num_slots, int overlap) {
    if (!overlap) pdl_wait();  // the previous kernel may still read the slots this one overwrites
    pdl_release_dependents();
    reshape_and_cache_body<VEC>(k, v, kc, vc, slots, num_kv_heads, row_bytes, k_stride_bytes, v_stride_bytes,
                                num_slots);
    if (overlap && blockIdx.x == 0 && blockIdx.y == 0) pdl_wait();
}

int launch_reshape_and_cache(const void *k, const void *v, void *kc, void *vc,
                             const int64_t *slots, int64_t T, int H, int D, int64_t N, int E,
                             int64_t k_stride, int64_t v_stride, int overlap, cudaStream_t st) {
    if (T == 0) return PA_OK;
    const int row = D * E;
    const int64_t ksb = k_stride * E, vsb = v_stride * E;
    // widest access that every address and stride allows
    uint64_t a = (uint64_t)(uintptr_t)k | (uint64_t)(uintptr_t)v | (uint64_t)(uintptr_t)kc |
                 (uint64_t)(uintptr_t)vc | (uint64_t)row | (uint64_t)ksb | (uint64_t)vsb;
    int vec = (a % 16 == 0) ? 16 : (a % 8 == 0) ? 8 : (a % 4 == 0) ? 4 : (a % 2 == 0) ? 2 : 1;
    const int total = H * (row / vec);
    const int threads = total >= 256 ? 256 : ((total + 31) / 32) * 32;
    dim3 grid((unsigned)T, 2);
    const char *kp = (const char *)k, *vp = (const char *)v;
    char *kcp = (char *)kc, *vcp = (char *)vc;
    const int64_t ns = N * kBlockSize;
    cudaError_t e;
    switch (vec) {
    case 16: e = launch_pdl(reshape_and_cache_kernel<16>, grid, dim3(threads), 0, st, kp, vp, kcp, vcp, slots, H, row, ksb, vsb, ns, overlap); break;
    case 8: e = launch_pdl(reshape_and_cache_kernel<8>, grid, dim3(threads), 0, st, kp, vp, kcp, vcp, slots, H, row, ksb, vsb, ns, overlap); break;
    case 4: e = launch_pdl(reshape_and_cache_kernel<4>, grid, dim3(threads), 0, st, kp, vp, kcp, vcp, slots, H, row, ksb, vsb, ns, overlap); break;
    case 2: e = launch_pdl(reshape_and_cache_kernel<2>, grid, dim3(threads), 0, st, kp, vp, kcp, vcp, slots, H, row, ksb, vsb, ns, overlap); break;
    default: e = launch_pdl(reshape_and_cache_kernel<1>, grid, dim3(threads), 0, st, kp, vp, kcp, vcp, slots, H, row, ksb, vsb, ns, overlap); break;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// block_copy (chanyi.net.cn/article/49 section 三: copy-on-write of a shared
// block when a sequence diverges).  Grid: (num_pairs, chunks, 2) -- z selects
// K or V; each CTA copies `chunk` 16-byte vectors of one block.  Scales are
// copied by chunk 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) block_copy_kernel(
    char *__restrict__ kc, char *__restrict__ vc, float *__restrict__ ks, float *__restrict__ vs,
    const int64_t *__restrict__ pairs, int64_t num_blocks, int64_t blk_vecs, int64_t chunk,
    int num_kv_heads) {
    pdl_wait();
    pdl_release_dependents();
    const int64_t src = pairs[2 * (int64_t)blockIdx.x], dst = pairs[2 * (int64_t)blockIdx.x + 1];
    if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) raise_flag(PA_EFLAG_BAD_PAIR);
        return;
    }
    const bool is_v = blockIdx.z != 0;
    uint4 *base = reinterpret_cast<uint4 *>(is_v ? vc : kc);
    const uint4 *s = base + src * blk_vecs;
    uint4 *d = base + dst * blk_vecs;
    const int64_t lo = blockIdx.y * chunk;
    const int64_t hi = min(lo + chunk, blk_vecs);
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) d[i] = s[i];
    float *sc = is_v ? vs : ks;
    if (sc != nullptr && blockIdx.y == 0)
        for (int h = threadIdx.x; h < num_kv_heads; h += blockDim.x)
            sc[dst * num_kv_heads + h] = sc[src * num_kv_heads + h];
}

int launch_block_copy(void *kc, void *vc, float *ks, float *vs, const int64_t *pairs,
                      int64_t n, int H, int D, int64_t N, int E, cudaStream_t st) {
    if (n == 0) return PA_OK;
    const int64_t blk_bytes = (int64_t)H * kBlockSize * D * E;
    if (blk_bytes % 16 || ((uintptr_t)kc | (uintptr_t)vc) % 16) return PA_ERR_ALIGN;
    const int64_t blk_vecs = blk_bytes / 16;
    const int64_t chunk = 2048;  // 32 KB per CTA
    const int64_t chunks = (blk_vecs + chunk - 1) / chunk;
    dim3 grid((unsigned)n, (unsigned)chunks, 2);
    const cudaError_t e = launch_pdl(block_copy_kernel, grid, dim3(256), 0, st, (char *)kc, (char *)vc, ks, vs,
                                     pairs, N, blk_vecs, chunk, H);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// quantize_int8 (lqnn.cn/news/235768 section 4.1: 8-bit KV with a grouped
// scale; the group is one (block, KV head) tile).  One CTA of 128 threads per
// tile; IEEE fp32 divide and round-half-even, as the definition states.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) quantize_int8_kernel(const T *__restrict__ src,
                                                            int8_t *__restrict__ dst,
                                                            float *__restrict__ scales, int tile) {
    __shared__ float red[4];
    pdl_wait();
    pdl_release_dependents();
    const int64_t t = blockIdx.x;
    const T *x = src + t * tile;
    float a = 0.f;
    for (int i = threadIdx.x; i < tile; i += blockDim.x) a = fmaxf(a, fabsf(Cvt<T>::to_f(x[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float s = __fdiv_rn(a, 127.0f);
    if (threadIdx.x == 0) scales[t] = s;
    int8_t *y = dst + t * tile;
    for (int i = threadIdx.x; i < tile; i += blockDim.x) {
        int r = 0;
        if (a != 0.f) {
            r = __float2int_rn(__fdiv_rn(Cvt<T>::to_f(x[i]), s));
            r = max(-127, min(127, r));
        }
        y[i] = (int8_t)r;
    }
}

int launch_quantize_int8(const void *src, int src_dtype, int8_t *dst, float *scales,
                         int64_t N, int H, int D, cudaStream_t st) {
    const int64_t tiles = N * H;
    if (tiles == 0) return PA_OK;
    const int tile = kBlockSize * D;
    cudaError_t e;
    const dim3 grid((unsigned)tiles);
    switch (src_dtype) {
    case PA_F32: e = launch_pdl(quantize_int8_kernel<float>, grid, dim3(128), 0, st, (const float *)src, dst, scales, tile); break;
    case PA_F16: e = launch_pdl(quantize_int8_kernel<__half>, grid, dim3(128), 0, st, (const __half *)src, dst, scales, tile); break;
    case PA_BF16: e = launch_pdl(quantize_int8_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, (const __nv_bfloat16 *)src, dst, scales, tile); break;
    default: return PA_ERR_DTYPE;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// append_int8: single tokens into an int8 cache (the 8-bit grouped-scale KV of
// lqnn.cn/news/235768 section 4.1 once its blocks are quantised).  For token i
// at slot s, block s / 16, slot s % 16, each KV head, K and V separately: the
// token's absmax a gives c = a / 127; when c exceeds the tile's scale the scale
// becomes c and the tile's other codes are re-rounded, q <- rint(q * s_old /
// s_new); the token's codes are rint(x / s_new); all in IEEE fp32 with round
// half to even, clamped to +-127.  Grid (tokens, 2): y selects K or V; warp w
// of the CTA takes KV heads w, w + 4, ...  The tokens of one call must fall in
// distinct blocks (each tile has one writer).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) append_int8_kernel(const T *__restrict__ k, const T *__restrict__ v,
                                                          int8_t *__restrict__ kc, int8_t *__restrict__ vc,
                                                          float *__restrict__ ks, float *__restrict__ vs,
                                                          const int64_t *__restrict__ slots, int H, int D,
                                                          int64_t k_stride, int64_t v_stride, int64_t num_slots) {
    pdl_wait();  // the previous kernel may still read the tiles this one rewrites
    pdl_release_dependents();
    const int64_t i = blockIdx.x;
    const int64_t s = slots[i];
    if (s < 0) return;
    if (s >= num_slots) {
        if (threadIdx.x == 0 && blockIdx.y == 0) raise_flag(PA_EFLAG_BAD_SLOT);
        return;
    }
    const bool is_v = blockIdx.y != 0;
    const T *x = (is_v ? v : k) + i * (is_v ? v_stride : k_stride);
    int8_t *cache = is_v ? vc : kc;
    float *scales = is_v ? vs : ks;
    const int64_t blk = s / kBlockSize;
    const int o = (int)(s % kBlockSize);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < H; h += 4) {
        const T *xh = x + (int64_t)h * D;
        float a = 0.f;
        for (int j = lane; j < D; j += 32) a = fmaxf(a, fabsf(Cvt<T>::to_f(xh[j])));
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
        const float c = __fdiv_rn(a, 127.0f);
        float *sp = scales + blk * H + h;
        const float s_old = *sp;
        const float s_new = c > s_old ? c : s_old;
        int8_t *t = cache + (blk * H + h) * (int64_t)kBlockSize * D;
        if (s_new > s_old) {
            for (int e = lane; e < kBlockSize * D; e += 32) {
                if (e / D == o) continue;
                const float prod = __fmul_rn((float)t[e], s_old);
                int q = __float2int_rn(__fdiv_rn(prod, s_new));
                t[e] = (int8_t)max(-127, min(127, q));
            }
        }
        for (int j = lane; j < D; j += 32) {
            int q = 0;
            if (s_new != 0.f) {
                q = __float2int_rn(__fdiv_rn(Cvt<T>::to_f(xh[j]), s_new));
                q = max(-127, min(127, q));
            }
            t[o * D + j] = (int8_t)q;
        }
        __syncwarp();
        if (lane == 0) *sp = s_new;
    }
}

int launch_append_int8(const void *k, const void *v, int8_t *kc, int8_t *vc, float *ks, float *vs,
                       const int64_t *slots, int64_t T, int H, int D, int64_t N, int src_dtype,
                       int64_t k_stride, int64_t v_stride, cudaStream_t st) {
    if (T == 0) return PA_OK;
    const dim3 grid((unsigned)T, 2);
    const int64_t ns = N * kBlockSize;
    cudaError_t e;
    switch (src_dtype) {
    case PA_F32: e = launch_pdl(append_int8_kernel<float>, grid, dim3(128), 0, st, (const float *)k, (const float *)v, kc, vc, ks, vs, slots, H, D, k_stride, v_stride, ns); break;
    case PA_F16: e = launch_pdl(append_int8_kernel<__half>, grid, dim3(128), 0, st, (const __half *)k, (const __half *)v, kc, vc, ks, vs, slots, H, D, k_stride, v_stride, ns); break;
    case PA_BF16: e = launch_pdl(append_int8_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, kc, vc, ks, vs, slots, H, D, k_stride, v_stride, ns); break;
    default: return PA_ERR_DTYPE;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// quantize_int4 (lqnn.cn/news/235768 section 4.1: 4-bit KV with a grouped
// scale; the group is one (block, KV head) tile).  One CTA of 128 threads per
// tile; IEEE fp32 divide and round-half-even; each thread writes whole bytes
// (two elements).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) quantize_int4_kernel(const T *__restrict__ src,
                                                            uint8_t *__restrict__ dst,
                                                            float *__restrict__ scales, int tile) {
    __shared__ float red[4];
    pdl_wait();
    pdl_release_dependents();
    const int64_t t = blockIdx.x;
    const T *x = src + t * tile;
    float a = 0.f;
    for (int i = threadIdx.x; i < tile; i += blockDim.x) a = fmaxf(a, fabsf(Cvt<T>::to_f(x[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float s = __fdiv_rn(a, 7.0f);
    if (threadIdx.x == 0) scales[t] = s;
    uint8_t *y = dst + t * (tile / 2);
    auto q4 = [&](float v) -> int {
        if (a == 0.f) return 8;
        const int r = __float2int_rn(__fdiv_rn(v, s));
        return max(-7, min(7, r)) + 8;
    };
    for (int k = threadIdx.x; k < tile / 2; k += blockDim.x)
        y[k] = (uint8_t)(q4(Cvt<T>::to_f(x[2 * k])) | (q4(Cvt<T>::to_f(x[2 * k + 1])) << 4));
}

int launch_quantize_int4(const void *src, int src_dtype, uint8_t *dst, float *scales,
                         int64_t N, int H, int D, cudaStream_t st) {
    const int64_t tiles = N * H;
    if (tiles == 0) return PA_OK;
    const int tile = kBlockSize * D;
    cudaError_t e;
    const dim3 grid((unsigned)tiles);
    switch (src_dtype) {
    case PA_F32: e = launch_pdl(quantize_int4_kernel<float>, grid, dim3(128), 0, st, (const float *)src, dst, scales, tile); break;
    case PA_F16: e = launch_pdl(quantize_int4_kernel<__half>, grid, dim3(128), 0, st, (const __half *)src, dst, scales, tile); break;
    case PA_BF16: e = launch_pdl(quantize_int4_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, (const __nv_bfloat16 *)src, dst, scales, tile); break;
    default: return PA_ERR_DTYPE;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
