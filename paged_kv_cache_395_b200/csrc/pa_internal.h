// Launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

template <int N> struct VecT;
template <> struct VecT<16> { using type = uint4; };
template <> struct VecT<8> { using type = uint2; };
template <> struct VecT<4> { using type = uint32_t; };
template <> struct VecT<2> { using type = uint16_t; };
template <> struct VecT<1> { using type = uint8_t; };

int launch_reshape_and_cache(const void *k, const void *v, void *kc, void *vc,
                             const int64_t *slots, int64_t T, int H, int D, int64_t N, int E,
                             int64_t k_stride, int64_t v_stride, int overlap, cudaStream_t st);
int launch_block_copy(void *kc, void *vc, float *ks, float *vs, const int64_t *pairs, int64_t n,
                      int H, int D, int64_t N, int E, cudaStream_t st);
int launch_append_int8(const void *k, const void *v, int8_t *kc, int8_t *vc, float *ks, float *vs,
                       const int64_t *slots, int64_t T, int H, int D, int64_t N, int src_dtype,
                       int64_t k_stride, int64_t v_stride, cudaStream_t st);
int launch_quantize_int8(const void *src, int src_dtype, int8_t *dst, float *scales, int64_t N,
                         int H, int D, cudaStream_t st);
int launch_quantize_int4(const void *src, int src_dtype, uint8_t *dst, float *scales, int64_t N,
                         int H, int D, cudaStream_t st);

// Everything pa_decode needs after validation.
struct DecodeArgs {
    void *out;
    const void *q;
    const void *kc;
    const void *vc;
    const float *ks;
    const float *vs;
    const int32_t *tables;
    const int32_t *lens;
    float scale_log2;        // scale * log2(e): scores are kept in the log2 domain
    int B, Hq, Hkv, D, G;    // Hkv, G: the kernel's rows per sequence and columns per row.
                             // The gcols = qlen * Greal (query token, head) pairs of one
                             // cache KV head fill the G <= 8 columns of `ngroups` rows
                             // (virtual KV heads; Hkv = cache KV heads * ngroups); column j
                             // of row kvh is pair (kvh % ngroups) * G + j, and pairs past
                             // gcols are padding.
    int ngroups;             // virtual KV heads per cache KV head
    int qlen;                // new tokens per sequence (q, out: [B][qlen][Hq][D])
    int Greal;               // query heads per cache KV head
    int gcols;               // qlen * Greal
    int mbps;                // max_blocks_per_seq
    int64_t N;               // num_blocks
    int max_len;             // effective bound on seq_lens
    int q_dtype, kv_dtype;
    int part;                // partition size in tokens (0 = one pass)
    int max_parts;           // ceil(max_len / part) when part > 0
    float *ws_o;             // [B][Hq][max_parts][D]
    float *ws_lse;           // [B][Hq][max_parts]  (log2 domain)
    int tc_chunk;            // tensor-core schedule: blocks per chunk, 0 = balanced auto,
                             // -1 = whole rows (one pass)
    int tc_W;                // warps of the tensor-core decode grid (its merge kernel redoes the schedule)
    int early;               // PA_DECODE_INPUTS_READY: read lengths, tables and q before
                             // the previous kernel on the stream has finished
    int out_f32;             // PA_DECODE_OUT_F32: out is fp32 of q's shape
    int stall_at;            // -1; else the first worker of the tensor-core family leaves
                             // its stall_at-th copy unissued (pa_decode_stall_selftest)
    unsigned long long wait_ns;  // limit of every bounded wait on a copy
    int umma;                // PA_ALGO_TCGEN05: the tcgen05 kernel (pa_decode_umma.cu)
    // pa_decode_append on the tensor-core family: row b of k_new / v_new ([B][H_kv][D],
    // token strides in elements) is sequence b's new token, written to cache slot
    // slot_new[b] (< 0: none) by the kernel, which also uses it in place of what its
    // copy of that slot's block held
    int append;
    const void *k_new, *v_new;
    const int64_t *slot_new;
    int64_t kn_stride, vn_stride;
};

// Default limit of a bounded wait: one second.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Tensor-core schedule limits: the auto schedule cuts the block stream into at
// most kTcMaxChunks chunks (one per warp of the grid) of at least kTcMinChunk
// blocks; the per-CTA prefix sum holds at most kTcMaxB sequences.
constexpr int kTcMaxChunks = 2048;
#ifndef PA_TC_MIN_CHUNK
#define PA_TC_MIN_CHUNK 4
#endif
constexpr int kTcMinChunk = PA_TC_MIN_CHUNK;
constexpr int kTcMaxB = 4096;

// Per-translation-unit error words (see PA_ERROR_WORD_ACCESSOR).
int error_word_cache_ops(unsigned int *flags, bool reset);
int error_word_decode_simt(unsigned int *flags, bool reset);
int error_word_decode_tc(unsigned int *flags, bool reset);
int error_word_decode_umma(unsigned int *flags, bool reset);

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// (kernel, device).  Thread-safe; returns false if CUDA refuses.
bool set_smem_attr_once(const void *kernel, int bytes);

// Workspace layout for split-K: ws_o | ws_lse, each 256-byte aligned.
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int max_len, int part);
int launch_decode_tc(const DecodeArgs &a, cudaStream_t st);
bool decode_tc_supported(int q_dtype, int kv_dtype, int D, int G, int B);
// groups of 16, 32 or 64 query heads per KV head run one CTA per cache row
bool decode_coop_eligible(int q_dtype, int kv_dtype, int D, int G, int ngroups, int qlen, bool padded, int part);
// groups of 32 or 64 fp16/bf16 query heads per KV head at head_dim 128 on tcgen05
bool decode_umma_eligible(int q_dtype, int kv_dtype, int D, int G, int ngroups, int qlen, bool padded, int part,
                          int B);
int launch_decode_umma(const DecodeArgs &a, cudaStream_t st);
int launch_decode_simt(const DecodeArgs &a, cudaStream_t st);
int launch_merge(const DecodeArgs &a, cudaStream_t st);
bool decode_simt_supported(int q_dtype, int kv_dtype, int D, int G);

}  // namespace pa
