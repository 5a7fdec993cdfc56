/*
 * pa.h -- paged single-token decode attention on NVIDIA B200 (sm_100a), C ABI.
 *
 * The KV cache of one attention layer lives in a pool of fixed-size physical
 * blocks of PA_BLOCK_SIZE tokens.  Each sequence owns a block table that maps
 * its logical block i to a physical block; blocks need not be contiguous and
 * the kernels walk the table in order without gathering the blocks
 * (lqnn.cn/news/235768 section 3.2; chanyi.net.cn/article/49 section 三).
 * Query heads share KV heads under GQA/MQA: query head h reads KV head
 * h / (num_q_heads / num_kv_heads) (lqnn.cn/news/235768 section 4.2).
 *
 * Memory layouts (row-major, innermost last):
 *   key_cache, value_cache  [num_blocks][num_kv_heads][PA_BLOCK_SIZE][head_dim]
 *                           (PA_I4: head_dim / 2 bytes per row, two values per byte)
 *   k_scales, v_scales      [num_blocks][num_kv_heads]  fp32 (int8 and 4-bit caches only)
 *   q, out                  [num_seqs][num_q_heads][head_dim]
 *                           ([num_seqs][Q][num_q_heads][head_dim] for Q = query_len > 1)
 *   block_tables            [num_seqs][max_blocks_per_seq]  int32
 *   seq_lens                [num_seqs]  int32
 *   slot_mapping            [num_tokens]  int64, slot = block * PA_BLOCK_SIZE + offset
 *
 * Ownership: the caller allocates and owns every buffer, including the split-K
 * workspace.  The library allocates no memory and keeps no per-call state
 * (pa_decode_fixed_scratch uses a fixed area compiled into the library).
 * Every pointer argument is a DEVICE pointer except `p` (pa_decode_params) and
 * the host-side out-parameters of pa_get_error_flags.  Every call is
 * asynchronous on `stream` and never synchronises the host, except
 * pa_get_error_flags.
 *
 * Errors: host-checkable problems are reported by the return value before any
 * launch (nothing is launched then).  A failed launch returns PA_ERR_CUDA.
 * Data errors found on the device (a block id outside [0, num_blocks) in a
 * table entry that is read, a slot outside the pool, a copy pair outside the
 * pool, a bounded wait that gave up) never trap: the offending item is
 * skipped and a bit is set in a per-device error word, read with
 * pa_get_error_flags.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *pa_stream_t;

enum pa_status {
    PA_OK = 0,
    PA_ERR_NULL = -1,        /* a required pointer is NULL */
    PA_ERR_SHAPE = -2,       /* a size is negative/zero where it must be positive, or inconsistent */
    PA_ERR_DTYPE = -3,       /* unknown dtype or unsupported q/KV dtype pair */
    PA_ERR_UNSUPPORTED = -4, /* valid but not built: block_size != 16, head_dim, group size */
    PA_ERR_WORKSPACE = -5,   /* split-K workspace missing or smaller than pa_decode_workspace_size */
    PA_ERR_CUDA = -6,        /* a CUDA launch or query failed */
    PA_ERR_ALIGN = -7        /* a buffer is not aligned as documented */
};

/* PA_I4: 4-bit values, two per byte (see pa_quantize_int4); a PA_I4 cache row of
 * head_dim values is head_dim / 2 bytes. */
enum pa_dtype { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_I8 = 3, PA_I4 = 4 };

/* Kernel family for pa_decode.  AUTO picks the fastest built one. */
/* PA_ALGO_TCGEN05: the tcgen05 kernel (5th-generation tensor cores, accumulators in
 * tensor memory) for groups of 32 or 64 fp16/bf16 query heads per KV head at head_dim
 * 128, split-K (partition_size != 0), num_seqs <= 2048; PA_ERR_UNSUPPORTED elsewhere.
 * PA_ALGO_AUTO runs it for the split groups of 64 (faster there); for groups of 16 and 32,
 * and under PA_ALGO_TENSOR, the mma.sync kernel that shares each staged tile across a
 * CTA's warps runs instead (faster for those groups). */
enum pa_algo { PA_ALGO_AUTO = 0, PA_ALGO_SIMT = 1, PA_ALGO_TENSOR = 2, PA_ALGO_TCGEN05 = 3 };

/* Bits of the per-device error word (pa_get_error_flags). */
enum pa_error_flag {
    PA_EFLAG_BAD_BLOCK = 1,   /* a block table entry read by pa_decode was outside the pool */
    PA_EFLAG_BAD_SLOT = 2,    /* a slot_mapping entry was >= num_blocks * PA_BLOCK_SIZE */
    PA_EFLAG_BAD_PAIR = 4,    /* a pa_block_copy pair was outside the pool */
    PA_EFLAG_WAIT_TIMEOUT = 8, /* a bounded wait on an asynchronous copy gave up */
    PA_EFLAG_APPEND_SLOT = 16  /* pa_decode_append: a new token's slot was not the slot of
                                  its sequence's position seq_lens[b] - 1 */
};

#define PA_BLOCK_SIZE 16

/*
 * Append new tokens to the paged cache (lqnn.cn/news/235768 section 2.2:
 * the new token's k, v are written at position cache_len before attention).
 *
 * For every token i with s = slot_mapping[i] >= 0, every KV head h:
 *   key_cache  [s / 16][h][s % 16][:] = k[i * k_token_stride + h * head_dim + :]
 *   value_cache[s / 16][h][s % 16][:] = v[i * v_token_stride + h * head_dim + :]
 * A bit-exact copy.  s < 0 marks padding and is skipped; s >= num_blocks * 16
 * sets PA_EFLAG_BAD_SLOT and is skipped.  Strides are in elements.  Slots
 * must be distinct (two tokens writing one slot race).
 * dtype: PA_F32, PA_F16 or PA_BF16 (PA_I8 caches are written by
 * pa_quantize_int8 and pa_append_int8, so PA_I8 returns PA_ERR_UNSUPPORTED).
 * Any alignment works; 16-byte aligned rows are copied with 16-byte vectors.
 */
int pa_reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, int dtype,
                         int64_t k_token_stride, int64_t v_token_stride, pa_stream_t stream);

/*
 * pa_reshape_and_cache with flags: 0, or PA_APPEND_OVERLAP_PREVIOUS.
 *
 * PA_APPEND_OVERLAP_PREVIOUS: the caller guarantees that no kernel still running
 * before this call on `stream` reads or writes any slot this call writes -- for
 * example a decode engine that puts the blocks of sequences finished after a
 * decode step back on its free list only one step later, so a step's appends
 * never land in a block the previous step's decode reads (slots past a
 * sequence's length are never part of its result).  The copies then run while
 * the previous kernel finishes, and the next kernel may launch at once; the call
 * still completes only after the previous kernel has, so a kernel that waits for
 * this one finds every earlier one complete.  Without the guarantee the result
 * of the previous kernel is undefined.  The inputs (k, v, slot_mapping) must not
 * be produced by the previous kernel either: the flag suits appends of K/V made
 * earlier (the prompt of a newly admitted sequence, written after an earlier
 * prefill), not a decode loop's new token, whose K/V come from the computation
 * just before.  (No counterpart in the pages: it hides an append's latency
 * behind the kernel before it.)
 */
#define PA_APPEND_OVERLAP_PREVIOUS 1
int pa_reshape_and_cache_ex(const void *k, const void *v, void *key_cache, void *value_cache,
                            const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                            int head_dim, int block_size, int64_t num_blocks, int dtype,
                            int64_t k_token_stride, int64_t v_token_stride, int flags, pa_stream_t stream);

typedef struct pa_decode_params {
    int num_seqs;            /* B >= 0 */
    int num_q_heads;         /* H_q, a multiple of num_kv_heads */
    int num_kv_heads;        /* H_kv; group size G = H_q / H_kv with Q * G <= 512 (Q =
                                query_len).  The Q * G (query token, head) pairs of a KV head
                                run as up to 8 columns per kernel row, more as several rows
                                that each read the KV head's tiles (MQA: H_kv = 1).  Counts
                                other than 1, 2, 4, 8 or multiples of 8 are padded, on the
                                tensor-core family only; the CUDA-core family takes
                                single-token decode with G in 1, 2, 4, 8, 16, 32, 64. */
    int head_dim;            /* 64, 128 or 256 (256 not with PA_F32; PA_I4 takes 128
                                only, and the tensor-core int8 path 128 or 256) */
    int block_size;          /* must be PA_BLOCK_SIZE */
    int max_blocks_per_seq;  /* row stride of block_tables */
    int64_t num_blocks;      /* physical blocks in the pool */
    int max_seq_len;         /* >= every seq_lens[b]; sizes the split-K grid and workspace.
                                Tokens beyond max_seq_len or max_blocks_per_seq * 16 are ignored. */
    int q_dtype;             /* dtype of q and out: PA_F32, PA_F16 or PA_BF16 */
    int kv_dtype;            /* PA_F32 (q PA_F32), PA_F16 (q PA_F16), PA_BF16 (q PA_BF16),
                                PA_I8 (q PA_F16 or PA_BF16), or PA_I4 (q PA_F16, head_dim
                                128, tensor-core family) */
    const float *k_scales;   /* PA_I8 / PA_I4 only: [num_blocks][num_kv_heads], else NULL */
    const float *v_scales;
    int partition_size;      /* 0: one pass, one CTA per (sequence, KV head), no workspace.
                                > 0: split-K, partitions of this many tokens (a multiple of
                                16), then a log-sum-exp merge; needs the workspace.
                                -1: the library picks from num_seqs, num_kv_heads and
                                max_seq_len (64..512 tokens, or one pass when max_seq_len
                                fits one partition). */
    int algo;                /* enum pa_algo */
    void *workspace;         /* device scratch, >= pa_decode_workspace_size(p) bytes,
                                16-byte aligned; NULL allowed when that size is 0.  It holds
                                the partial results of one call only: nothing in it needs
                                initialising, and every value a call reads there was written
                                earlier in the same call.  So one workspace serves any
                                sequence of calls, whatever their parameters or kernel
                                family.  Calls that share a workspace must not overlap on
                                the device. */
    size_t workspace_bytes;
    int flags;               /* 0, or PA_DECODE_INPUTS_READY and/or PA_DECODE_OUT_F32 */
    int query_len;           /* new tokens per sequence, Q (0 or 1: single-token decode).
                                q and out are [num_seqs][Q][num_q_heads][head_dim]; seq_lens
                                count all Q new tokens (already appended), and query token i
                                attends causally to tokens 0 .. seq_lens[b] - Q + i.  Q > 1
                                runs on the tensor-core family only. */
} pa_decode_params;

/*
 * Every kernel of the library is launched with programmatic dependent launch
 * allowed: it may become resident while the kernel before it on the stream
 * finishes, and waits for that kernel to complete (with its writes visible)
 * before it touches any memory.  PA_DECODE_INPUTS_READY lets pa_decode start
 * earlier: it reads seq_lens, block_tables and q while the kernel just before
 * it on the stream may still be running, and waits only before its first read
 * of the caches (writes to out and the workspace also come after the wait).
 * Set it only when that kernel does not write q, block_tables or seq_lens --
 * for example when it is a pa_reshape_and_cache, pa_block_copy or pa_decode
 * call of this library (each of which lets its successor start only after the
 * kernels before it have completed).  The tensor-core family uses it; the
 * CUDA-core family ignores it.
 */
#define PA_DECODE_INPUTS_READY 1

/*
 * PA_DECODE_OUT_F32: out is fp32, of q's shape, holding the fp32 result before
 * the one rounding to q_dtype that pa_decode otherwise applies.  With an fp16 or
 * bf16 q the fp16/bf16 output is exactly that fp32 value rounded to nearest
 * even, so the flag shows the arithmetic's accuracy apart from the output
 * format's (bf16 keeps 8 significant bits: its rounding alone moves a value by
 * up to 2^-8 of its size).
 */
#define PA_DECODE_OUT_F32 2

/*
 * Bytes of device workspace pa_decode needs for these parameters (0 when the
 * call runs in one pass; else the partial results).  Depends only on num_seqs,
 * num_q_heads, num_kv_heads, head_dim, query_len, max_seq_len,
 * max_blocks_per_seq, the dtypes, algo and partition_size.  Returns 0 for
 * invalid params.
 */
size_t pa_decode_workspace_size(const pa_decode_params *p);

/*
 * The kernel family pa_decode runs for these parameters and this q:
 * PA_ALGO_TENSOR, PA_ALGO_SIMT or PA_ALGO_TCGEN05, or a negative pa_status for parameters
 * pa_decode would reject.  q (a device pointer, not read) matters only through
 * its alignment: the tensor-core family reads q rows with 16-byte copies, so an
 * unaligned q goes to the CUDA-core family.
 */
int pa_decode_algo(const pa_decode_params *p, const void *q);

/*
 * Kernel launches of one pa_decode call with these parameters and this q (1 or
 * 2), or a negative pa_status for parameters pa_decode would reject: the decode
 * kernel, followed by a merge kernel when the call splits on the family it
 * runs (an unaligned q can move a call to the CUDA-core family, whose own plan
 * decides).
 */
int pa_decode_launches(const pa_decode_params *p, const void *q);

/*
 * Single-token decode attention over the paged cache
 * (lqnn.cn/news/235768 sections 1.2 and 2.2; chanyi.net.cn/article/49 section 四):
 *
 *   out[b][h][:] = sum_t softmax_t(scale * q[b][h] . K[b][t]) V[b][t]
 *
 * over the logical tokens t = 0 .. seq_lens[b]-1 of sequence b, where token t
 * is slot t % 16 of physical block block_tables[b][t / 16], KV head
 * h / (H_q / H_kv).  seq_lens include the token being decoded, which must
 * already be in the cache.  int8 caches are dequantised as x = q8 * scale of
 * its (block, KV head).  The softmax runs online in fp32 and K/V products
 * accumulate in fp32; out is rounded once to q_dtype.  seq_lens[b] <= 0 gives
 * a zero row.  Only the first ceil(seq_lens[b] / 16) entries of a table row
 * are read.  With partition_size > 0 the sequence is cut into partitions whose
 * normalised partial outputs and log-sum-exp go to the workspace and are
 * merged: out = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M).
 * Result does not depend on where the physical blocks sit.
 */
int pa_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *seq_lens, float scale,
              const pa_decode_params *p, pa_stream_t stream);

/*
 * Append, then decode, in one call (lqnn.cn/news/235768 section 2.2: the step's
 * new token goes to the end of its sequence's cache, then the query attends to
 * the whole sequence).  Result, and cache contents afterwards, are those of
 *
 *   pa_reshape_and_cache(k_new, v_new, key_cache, value_cache, slot_mapping,
 *                        p->num_seqs, p->num_kv_heads, p->head_dim, p->block_size,
 *                        p->num_blocks, p->kv_dtype, k_token_stride, v_token_stride, stream);
 *   pa_decode(out, q, key_cache, value_cache, block_tables, seq_lens, scale, p, stream);
 *
 * for one new token per sequence (query_len 0 or 1; kv_dtype == q_dtype): row b
 * of k_new / v_new ([num_seqs][num_kv_heads][head_dim] with token strides in
 * elements) is sequence b's new token and slot_mapping[b] its slot (< 0: none);
 * seq_lens count it.  Quantised caches: pa_append_int8, then pa_decode.
 *
 * Where pa_decode_append_fused says so, the call is one kernel: the decode
 * writes every new token to its slot itself and uses it in place of what its
 * copy of that slot held, so no append kernel runs before it.  That relies on
 * slot_mapping[b] being the slot of position seq_lens[b] - 1 of sequence b
 * under its block table, as in a decode step; a new token whose slot is another
 * one sets PA_EFLAG_APPEND_SLOT, is still written to its slot, and leaves the
 * outputs that read that slot undefined.  A slot >= num_blocks * 16 sets
 * PA_EFLAG_BAD_SLOT and is skipped, as in pa_reshape_and_cache.  Otherwise the
 * two calls above run in order.  With PA_DECODE_INPUTS_READY the fused kernel
 * reads k_new, v_new and slot_mapping early too, so the kernel before it on the
 * stream must not write them either.
 */
int pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                     const int64_t *slot_mapping, int64_t k_token_stride, int64_t v_token_stride,
                     void *key_cache, void *value_cache, const int32_t *block_tables,
                     const int32_t *seq_lens, float scale, const pa_decode_params *p,
                     pa_stream_t stream);

/*
 * 1 when pa_decode_append with these arguments runs as one kernel -- the
 * tensor-core family's per-warp decode of single-token fp16 / bf16 rows (not
 * the cooperative mode of 16-64 query heads per KV head), with q, k_new and
 * v_new 16-byte aligned and token strides a multiple of 8 elements -- 0 when it
 * runs pa_reshape_and_cache then pa_decode, or the negative pa_status it would
 * return.  The pointers are not read.
 */
int pa_decode_append_fused(const pa_decode_params *p, const void *q, const void *k_new,
                           const void *v_new, int64_t k_token_stride, int64_t v_token_stride);

/*
 * pa_decode without a caller workspace.  No counterpart in the paper: it is an
 * addition of this library for callers that cannot allocate device memory
 * where they decode -- an engine that has given all free device memory to its
 * KV block pool up front, or a host integration with no device allocator of
 * its own.  Same arguments, same result and same errors as pa_decode; the
 * split-K workspace fields of `p` are ignored and a scratch area of
 * PA_FIXED_SCRATCH_BYTES compiled into the library (one per device) is used
 * instead.  The library allocates nothing.
 *
 *  - Parameters whose pa_decode_workspace_size exceeds PA_FIXED_SCRATCH_BYTES
 *    return PA_ERR_WORKSPACE and launch nothing.
 *  - The first call on a device looks up the area's address (no stream work:
 *    the area needs no clearing).  Make that first call before any stream
 *    capture.
 *  - All calls on one device share the area: calls that overlap on the device
 *    (different streams, or host threads without ordering) race on it.  Issue
 *    them in one stream order.  Calls in order may use any parameters.
 *  - The area's address is kept for the life of the process: do not use the
 *    library after cudaDeviceReset.
 */
#define PA_FIXED_SCRATCH_BYTES ((size_t)32 << 20)
int pa_decode_fixed_scratch(void *out, const void *q, const void *key_cache, const void *value_cache,
                            const int32_t *block_tables, const int32_t *seq_lens, float scale,
                            const pa_decode_params *p, pa_stream_t stream);

/*
 * Self-test of the failure path of the bounded waits (no counterpart in the
 * pages: it exists so that the library's handling of a copy that never lands
 * can be checked on a working GPU without faulting it).  Runs pa_decode on the
 * tensor-core family (the parameters must select it) with two changes: every
 * bounded wait gives up after limit_ns nanoseconds instead of one second, and
 * the first worker never issues its stall_at-th copy (counted from 0 over its
 * (K tile, V tile) stages), so its wait for that stage runs out: no memory is
 * read or written for it, and nothing hangs.  Expected outcome: PA_OK, the
 * error word gains PA_EFLAG_WAIT_TIMEOUT, the rows that worker had not finished
 * hold no valid result, and the next call may use the same workspace (the
 * worker waits, again bounded, for its copies in flight, then writes empty
 * partial results, weight 0 in the merge, for its remaining segments).
 */
int pa_decode_stall_selftest(void *out, const void *q, const void *key_cache, const void *value_cache,
                             const int32_t *block_tables, const int32_t *seq_lens, float scale,
                             const pa_decode_params *p, int stall_at, uint64_t limit_ns,
                             pa_stream_t stream);

/*
 * Copy-on-write block copy (chanyi.net.cn/article/49 section 三: shared prefix
 * blocks are copied only when a sequence diverges).  For each pair
 * (src = pairs[2i], dst = pairs[2i+1]) the whole physical block -- every KV
 * head and all 16 slots -- of key_cache and of value_cache is copied byte for
 * byte, and k_scales/v_scales[dst][:] = [src][:] when those are non-NULL.
 * A dst must not appear twice or also as a src (the copies run in parallel).
 * Pairs outside [0, num_blocks) set PA_EFLAG_BAD_PAIR and are skipped.
 * dtype: any pa_dtype.
 */
int pa_block_copy(void *key_cache, void *value_cache, float *k_scales, float *v_scales,
                  const int64_t *src_dst_pairs, int64_t num_pairs, int num_kv_heads,
                  int head_dim, int block_size, int64_t num_blocks, int dtype,
                  pa_stream_t stream);

/*
 * 8-bit KV with one scale per group (lqnn.cn/news/235768 section 4.1), the
 * group being one (block, KV head) tile of 16 * head_dim values.  For each of
 * the first num_blocks blocks and each KV head, in IEEE fp32:
 *   a = max |x|,  s = a / 127,  q8 = clamp(round_half_even(x / s), -127, 127)
 * a == 0 gives s = 0 and q8 = 0.  src_cache: [num_blocks][H_kv][16][head_dim]
 * of src_dtype (PA_F32, PA_F16 or PA_BF16); dst_cache int8 of the same shape;
 * scales [num_blocks][H_kv].  Call once for K and once for V.
 */
int pa_quantize_int8(const void *src_cache, int src_dtype, int8_t *dst_cache, float *scales,
                     int64_t num_blocks, int num_kv_heads, int head_dim, int block_size,
                     pa_stream_t stream);

/*
 * Append single tokens into an int8 cache (the 8-bit grouped-scale KV of
 * lqnn.cn/news/235768 section 4.1 after its blocks were quantised; the pages do
 * not spell out the update, this is the library's reading).  For every token i
 * with s = slot_mapping[i] >= 0, block b = s / 16, slot o = s % 16, every KV
 * head h, separately for K (k, key_cache, k_scales) and V:
 *   a = max_j |x_j| over the token's head_dim values, c = a / 127,
 *   s_old = scales[b][h], s_new = max(c, s_old);
 *   if s_new > s_old, every other code of the tile becomes
 *     clamp(rint((q * s_old) / s_new), -127, 127);
 *   the token's codes are clamp(rint(x_j / s_new), -127, 127) (0 when s_new = 0);
 *   scales[b][h] = s_new.
 * IEEE fp32, round half to even: bit-exact with the library's oracle.  The
 * scale never shrinks; a re-rounded value moves by at most s_new / 2.
 * k, v: [num_tokens][num_kv_heads][head_dim] with the given token strides (in
 * elements) of src_dtype PA_F32, PA_F16 or PA_BF16.  Caches int8
 * [num_blocks][num_kv_heads][16][head_dim], scales fp32 [num_blocks][num_kv_heads].
 * The tokens of one call must fall in distinct blocks (one writer per tile).
 * s < 0 is skipped; s >= num_blocks * 16 sets PA_EFLAG_BAD_SLOT and is skipped.
 */
int pa_append_int8(const void *k, const void *v, int src_dtype, int8_t *key_cache, int8_t *value_cache,
                   float *k_scales, float *v_scales, const int64_t *slot_mapping, int64_t num_tokens,
                   int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                   int64_t k_token_stride, int64_t v_token_stride, pa_stream_t stream);


/*
 * 4-bit KV with one scale per group (lqnn.cn/news/235768 section 4.1 names
 * 4-bit storage with grouped scales next to 8-bit), the group being one (block,
 * KV head) tile of 16 * head_dim values.  For each of the first num_blocks
 * blocks and each KV head, in IEEE fp32:
 *   a = max |x|,  s = a / 7,  q = clamp(round_half_even(x / s), -7, 7)
 * stored as n = q + 8: element 2k of a tile in the low four bits of its byte k,
 * element 2k+1 in the high four.  a == 0 gives s = 0 and q = 0 (bytes 0x88).
 * src_cache: [num_blocks][H_kv][16][head_dim] of src_dtype (PA_F32, PA_F16 or
 * PA_BF16); dst_cache: [num_blocks][H_kv][16][head_dim / 2] bytes; scales
 * [num_blocks][H_kv].  head_dim must be even.  Call once for K and once for V.
 */
int pa_quantize_int4(const void *src_cache, int src_dtype, uint8_t *dst_cache, float *scales,
                     int64_t num_blocks, int num_kv_heads, int head_dim, int block_size,
                     pa_stream_t stream);

/*
 * Read the calling thread's current device's error word into *flags
 * (pa_error_flag bits); synchronises `stream` first.  reset != 0 clears it.
 */
int pa_get_error_flags(unsigned int *flags, int reset, pa_stream_t stream);

/* Static description of a status code. */
const char *pa_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
