// Shared device helpers for the paged decode library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

constexpr int kBlockSize = PA_BLOCK_SIZE;
constexpr float kLog2e = 1.4426950408889634f;

// Error word (pa_error_flag bits).  Each translation unit that includes this
// header gets its own copy on every device; PA_ERROR_WORD_ACCESSOR(name) defines
// the host function that reads (and optionally clears) the copy of its unit,
// and pa_get_error_flags ORs them.
static __device__ unsigned int g_error_flags = 0;

__device__ __forceinline__ void raise_flag(unsigned int bit) { atomicOr(&g_error_flags, bit); }

// Programmatic dependent launch.  Every kernel of the library is launched with
// programmatic stream serialisation allowed, so it may become resident while
// the kernel before it on the stream is still finishing.  pdl_wait() returns
// once every grid this one depends on has completed and its writes are
// visible; nothing that a previous kernel may write (or read) is touched
// before it.  pdl_release_dependents() lets the next grid start launching; the
// kernels call it only after pdl_wait(), so a grid that starts early always
// finds the grids before its own predecessor complete.  Both are no-ops for a
// plain launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kern` on `st` with programmatic stream serialisation allowed.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

#define PA_ERROR_WORD_ACCESSOR(name)                                                        \
    int name(unsigned int *flags, bool reset) {                                             \
        if (cudaMemcpyFromSymbol(flags, g_error_flags, sizeof(unsigned int)) != cudaSuccess) \
            return PA_ERR_CUDA;                                                             \
        if (reset) {                                                                        \
            const unsigned int zero = 0;                                                    \
            if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(unsigned int)) != cudaSuccess) \
                return PA_ERR_CUDA;                                                         \
        }                                                                                   \
        return PA_OK;                                                                       \
    }

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T> struct Cvt;
template <> struct Cvt<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Cvt<__half> {
    static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Cvt<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Cvt<int8_t> {
    static __device__ __forceinline__ float to_f(int8_t x) { return (float)x; }
};

// Element idx of a decode output: fp32 when the call asked for an fp32 output
// (PA_DECODE_OUT_F32), else rounded once to T.
template <typename T>
__device__ __forceinline__ void store_out(void *out, int f32, size_t idx, float v) {
    if (f32)
        reinterpret_cast<float *>(out)[idx] = v;
    else
        reinterpret_cast<T *>(out)[idx] = Cvt<T>::from_f(v);
}

// Elements idx, idx + 1 (idx even) of a decode output, as one 4- or 8-byte store
// when the buffer's base allows it.
template <typename T>
__device__ __forceinline__ void store_out2(void *out, int f32, size_t idx, float v0, float v1) {
    if (f32) {
        float *o = reinterpret_cast<float *>(out) + idx;
        if (((uintptr_t)out & 7) == 0) {
            *reinterpret_cast<float2 *>(o) = make_float2(v0, v1);
        } else {
            o[0] = v0;
            o[1] = v1;
        }
    } else {
        T *o = reinterpret_cast<T *>(out) + idx;
        const T h0 = Cvt<T>::from_f(v0), h1 = Cvt<T>::from_f(v1);
        if (((uintptr_t)out & 3) == 0) {
            const uint32_t w = (uint32_t)*reinterpret_cast<const uint16_t *>(&h0) |
                               ((uint32_t)*reinterpret_cast<const uint16_t *>(&h1) << 16);
            *reinterpret_cast<uint32_t *>(o) = w;
        } else {
            o[0] = h0;
            o[1] = h1;
        }
    }
}

// Convert N consecutive elements held in registers (as raw 32-bit words) to float.
template <typename T, int N>
__device__ __forceinline__ void to_float(const uint32_t *w, float *f);

template <int N>
__device__ __forceinline__ void to_float_f32(const uint32_t *w, float *f) {
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = __uint_as_float(w[i]);
}
template <> __device__ __forceinline__ void to_float<float, 4>(const uint32_t *w, float *f) { to_float_f32<4>(w, f); }
template <> __device__ __forceinline__ void to_float<float, 8>(const uint32_t *w, float *f) { to_float_f32<8>(w, f); }
template <> __device__ __forceinline__ void to_float<float, 16>(const uint32_t *w, float *f) { to_float_f32<16>(w, f); }
template <> __device__ __forceinline__ void to_float<float, 2>(const uint32_t *w, float *f) { to_float_f32<2>(w, f); }

template <int N>
__device__ __forceinline__ void to_float_h(const uint32_t *w, float *f) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
        float2 x = __half22float2(h);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
template <> __device__ __forceinline__ void to_float<__half, 2>(const uint32_t *w, float *f) { to_float_h<2>(w, f); }
template <> __device__ __forceinline__ void to_float<__half, 4>(const uint32_t *w, float *f) { to_float_h<4>(w, f); }
template <> __device__ __forceinline__ void to_float<__half, 8>(const uint32_t *w, float *f) { to_float_h<8>(w, f); }
template <> __device__ __forceinline__ void to_float<__half, 16>(const uint32_t *w, float *f) { to_float_h<16>(w, f); }

template <int N>
__device__ __forceinline__ void to_float_b(const uint32_t *w, float *f) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        // bf16 is the top half of an fp32: shift / mask, no rounding involved.
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <> __device__ __forceinline__ void to_float<__nv_bfloat16, 2>(const uint32_t *w, float *f) { to_float_b<2>(w, f); }
template <> __device__ __forceinline__ void to_float<__nv_bfloat16, 4>(const uint32_t *w, float *f) { to_float_b<4>(w, f); }
template <> __device__ __forceinline__ void to_float<__nv_bfloat16, 8>(const uint32_t *w, float *f) { to_float_b<8>(w, f); }
template <> __device__ __forceinline__ void to_float<__nv_bfloat16, 16>(const uint32_t *w, float *f) { to_float_b<16>(w, f); }

template <int N>
__device__ __forceinline__ void to_float_i8(const uint32_t *w, float *f) {
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = (float)(int8_t)((w[i / 4] >> (8 * (i % 4))) & 0xff);
}
template <> __device__ __forceinline__ void to_float<int8_t, 2>(const uint32_t *w, float *f) { to_float_i8<2>(w, f); }
template <> __device__ __forceinline__ void to_float<int8_t, 4>(const uint32_t *w, float *f) { to_float_i8<4>(w, f); }
template <> __device__ __forceinline__ void to_float<int8_t, 8>(const uint32_t *w, float *f) { to_float_i8<8>(w, f); }
template <> __device__ __forceinline__ void to_float<int8_t, 16>(const uint32_t *w, float *f) { to_float_i8<16>(w, f); }

// Load BYTES bytes (2, 4, 8, 16, 32 or 64; naturally aligned) from shared memory into words.
template <int BYTES>
__device__ __forceinline__ void lds(const void *p, uint32_t *w) {
    if constexpr (BYTES == 2) {
        w[0] = *reinterpret_cast<const uint16_t *>(p);
    } else if constexpr (BYTES == 4) {
        w[0] = *reinterpret_cast<const uint32_t *>(p);
    } else if constexpr (BYTES == 8) {
        uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < BYTES / 16; ++i) {
            uint4 v = reinterpret_cast<const uint4 *>(p)[i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    }
}

// ---------------------------------------------------------------------------
// mbarrier + bulk asynchronous copy (TMA, non-tensor form)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Relaxed arrivals: they order none of the thread's earlier memory operations, so
// they do not wait for its outstanding loads.  For use where the data the
// barrier publishes comes only through the transaction count (bulk copies) and
// anything else is ordered by other means.
__device__ __forceinline__ void mbar_arrive_expect_tx_relaxed(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t *bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete.  Gives up after
// limit_ns nanoseconds (one second in every library call; a copy that never
// lands), raises PA_EFLAG_WAIT_TIMEOUT and returns false; the caller then
// abandons its remaining work.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63) == 63 && global_timer_ns() - t0 > limit_ns) {
            raise_flag(PA_EFLAG_WAIT_TIMEOUT);
            return false;
        }
    }
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned), completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Same, with shared-memory addresses given as 32-bit shared-window offsets.
__device__ __forceinline__ void bulk_g2s_u32(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 2^x with the hardware approximation (PTX ex2.approx.ftz: relative error about
// 2^-22; results below 2^-126 flush to 0, 2^-inf = 0).  Every use weights a
// probability against a running maximum that some term reaches at 2^0, so a flushed
// term is below 2^-126 of the sum.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace pa
