// C-ABI entry points: argument validation, then dispatch to the kernels.
// Every check that can be made on the host is made here, before any launch.
#include <mutex>
#include <set>
#include <utility>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

bool set_smem_attr_once(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    done.insert({kernel, dev});
    return true;
}

static int elem_size(int dt) {
    switch (dt) {
    case PA_F32: return 4;
    case PA_F16: return 2;
    case PA_BF16: return 2;
    case PA_I8: return 1;
    default: return 0;
    }
}

// Partition size for partition_size == -1.  The persistent kernel runs
// 148 SMs x 2 CTAs x 4 warps = 1184 warp workers on B200; aim for at least
// four (sequence, partition, KV head) items per worker, counting every
// sequence at max_len, with partitions of 64..512 tokens.  Depends only on
// the arguments, so pa_decode_workspace_size agrees with pa_decode.
static int auto_partition(int B, int Hkv, int max_len) {
    const int64_t want = 4 * 1184;
    for (int ps = 512; ps >= 64; ps >>= 1) {
        const int64_t items = (int64_t)B * Hkv * ((max_len + ps - 1) / ps);
        if (items >= want) return ps;
    }
    return 64;
}

// The heads as the kernels see them.  The Q x (query heads per KV head) pairs
// of (query token, head) that share one cache KV head become the columns of
// the kernels' rows: at most 8 per row (the MMA's n), padded up to a power of
// two when fewer, split over ceil(pairs / 8) rows (virtual KV heads) when more.
// The virtual heads of one cache head are adjacent rows, so their repeated
// tile reads meet in L2.
struct KernelHeads {
    int G, Hkv, ngroups, Greal, gcols, qlen;
    bool padded;  // some columns are padding (only the tensor-core family handles that)
};
static bool kernel_heads(const pa_decode_params *p, KernelHeads *kh) {
    const int Greal = p->num_q_heads / p->num_kv_heads;
    const int Q = p->query_len > 1 ? p->query_len : 1;
    const int64_t gcols = (int64_t)Q * Greal;
    if (gcols > 512) return false;  // at most 64 virtual KV heads per cache head
    int G, ng;
    if (gcols <= 8) {
        G = 1;
        while (G < gcols) G <<= 1;
        ng = 1;
    } else {
        G = 8;
        ng = (int)((gcols + 7) / 8);
    }
    *kh = KernelHeads{G, p->num_kv_heads * ng, ng, Greal, (int)gcols, Q, (int64_t)G * ng != gcols};
    return true;
}

// Checks shared by pa_decode and pa_decode_workspace_size.  Fills the partition
// size actually used (auto resolved) and the partition count.
static int check_decode_params(const pa_decode_params *p, int *part, int *max_parts) {
    if (!p) return PA_ERR_NULL;
    if (p->num_seqs < 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->head_dim <= 0 ||
        p->max_blocks_per_seq <= 0 || p->num_blocks <= 0 || p->max_seq_len < 0)
        return PA_ERR_SHAPE;
    if (p->num_q_heads % p->num_kv_heads) return PA_ERR_SHAPE;
    if (p->block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    if (!elem_size(p->q_dtype) || (!elem_size(p->kv_dtype) && p->kv_dtype != PA_I4) || p->q_dtype == PA_I8)
        return PA_ERR_DTYPE;
    if (p->query_len < 0) return PA_ERR_SHAPE;
    KernelHeads kh;
    const bool heads_ok = kernel_heads(p, &kh);
    const bool quant = p->kv_dtype == PA_I8 || p->kv_dtype == PA_I4;
    const bool pair_ok = (p->q_dtype == p->kv_dtype) || quant;
    if (!pair_ok || (quant && p->q_dtype == PA_F32) || (p->kv_dtype == PA_I4 && p->q_dtype != PA_F16))
        return PA_ERR_DTYPE;
    if (!heads_ok) return PA_ERR_UNSUPPORTED;
    const bool simt_ok = kh.qlen == 1 && !kh.padded &&
                         decode_simt_supported(p->q_dtype, p->kv_dtype, p->head_dim, kh.G);
    const bool tc_ok = decode_tc_supported(p->q_dtype, p->kv_dtype, p->head_dim, kh.G, p->num_seqs);
    if (!simt_ok && !tc_ok) return PA_ERR_UNSUPPORTED;
    if (p->algo == PA_ALGO_SIMT && !simt_ok) return PA_ERR_UNSUPPORTED;
    if (p->num_seqs > 65535 || kh.Hkv > 65535) return PA_ERR_UNSUPPORTED;
    if (p->algo < PA_ALGO_AUTO || p->algo > PA_ALGO_TCGEN05) return PA_ERR_UNSUPPORTED;
    if (p->algo == PA_ALGO_TCGEN05 &&
        !decode_umma_eligible(p->q_dtype, p->kv_dtype, p->head_dim, kh.G, kh.ngroups, kh.qlen, kh.padded,
                              p->partition_size, p->num_seqs))
        return PA_ERR_UNSUPPORTED;
    if (p->flags & ~(PA_DECODE_INPUTS_READY | PA_DECODE_OUT_F32)) return PA_ERR_UNSUPPORTED;
    int ps = p->partition_size;
    if (ps < -1 || (ps > 0 && ps % PA_BLOCK_SIZE)) return PA_ERR_SHAPE;
    const int max_len = p->max_seq_len < p->max_blocks_per_seq * PA_BLOCK_SIZE
                            ? p->max_seq_len
                            : p->max_blocks_per_seq * PA_BLOCK_SIZE;
    if (ps == -1) ps = auto_partition(p->num_seqs, kh.Hkv, max_len);
    if (ps > 0 && max_len <= ps) ps = 0;  // one partition: no split needed
    *part = ps;
    *max_parts = ps > 0 ? (max_len + ps - 1) / ps : 1;
    if (*max_parts > 65535) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Which kernel family runs and what workspace it needs.
struct Plan {
    bool tc;
    int part, max_parts;  // CUDA-core family: per-sequence partitions
    int tc_chunk;         // tensor-core family: see DecodeArgs::tc_chunk
    int64_t tc_slots;     // tensor-core family: partial-result slots
    int max_len;
    size_t bytes;
};

static int make_plan(const pa_decode_params *p, Plan *pl) {
    int part = 0, mp = 0;
    const int rc = check_decode_params(p, &part, &mp);
    if (rc != PA_OK) return rc;
    KernelHeads kh;
    kernel_heads(p, &kh);
    const int G = kh.G;
    const int max_len = p->max_seq_len < p->max_blocks_per_seq * PA_BLOCK_SIZE
                            ? p->max_seq_len
                            : p->max_blocks_per_seq * PA_BLOCK_SIZE;
    // the tensor-core family indexes cache rows and the concatenated block stream
    // of all (sequence, KV head) rows with 32-bit integers
    const int64_t stream_blocks =
        (int64_t)p->num_seqs * kh.Hkv * ((max_len + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE);
    const bool tc_ok = decode_tc_supported(p->q_dtype, p->kv_dtype, p->head_dim, G, p->num_seqs) &&
                       p->num_blocks * p->num_kv_heads * PA_BLOCK_SIZE <= 2147483647LL &&
                       stream_blocks <= (1LL << 30);
    if ((p->algo == PA_ALGO_TENSOR || p->algo == PA_ALGO_TCGEN05) && !tc_ok) return PA_ERR_UNSUPPORTED;
    // several new tokens per sequence, or padded columns: the tensor-core family only
    if ((kh.qlen > 1 || kh.padded) && !tc_ok) return PA_ERR_UNSUPPORTED;
    *pl = Plan{};
    pl->max_len = max_len;
    pl->tc = p->algo == PA_ALGO_TENSOR || p->algo == PA_ALGO_TCGEN05 || (p->algo == PA_ALGO_AUTO && tc_ok);
    if (!pl->tc) {
        pl->part = part;
        pl->max_parts = mp;
        pl->bytes = decode_workspace_bytes(p->num_seqs, p->num_q_heads, kh.Hkv, p->head_dim, max_len, part);
        return PA_OK;
    }
    if (p->partition_size == 0 || max_len == 0) {
        pl->tc_chunk = -1;  // one warp per (sequence, KV head) row, no workspace
        return PA_OK;
    }
    const int64_t tmax = (int64_t)p->num_seqs * kh.Hkv * ((max_len + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE);
    int64_t nchunks;
    if (p->partition_size > 0) {
        pl->tc_chunk = p->partition_size / PA_BLOCK_SIZE;
        nchunks = (tmax + pl->tc_chunk - 1) / pl->tc_chunk;
    } else {
        // one chunk per warp of the grid: at most kTcMaxChunks
        pl->tc_chunk = 0;
        nchunks = tmax < kTcMaxChunks ? tmax : kTcMaxChunks;
    }
    if (decode_coop_eligible(p->q_dtype, p->kv_dtype, p->head_dim, G, kh.ngroups, kh.qlen, kh.padded, 1)) {
        // one CTA per chunk of cache rows, 8 * ngroups columns per row
        const int64_t cmax = (int64_t)p->num_seqs * p->num_kv_heads * ((max_len + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE);
        const int64_t cn = p->partition_size > 0 ? (cmax + pl->tc_chunk - 1) / pl->tc_chunk
                                                 : (cmax < kTcMaxChunks ? cmax : kTcMaxChunks);
        pl->tc_slots = 2 * cn;
        pl->bytes = up256((size_t)pl->tc_slots * G * kh.ngroups * p->head_dim * sizeof(float)) +
                    up256((size_t)pl->tc_slots * G * kh.ngroups * sizeof(float));
        return PA_OK;
    }
    pl->tc_slots = 2 * nchunks;
    // partial outputs and lse of two segments per chunk
    pl->bytes = up256((size_t)pl->tc_slots * G * p->head_dim * sizeof(float)) +
                up256((size_t)pl->tc_slots * G * sizeof(float));
    return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" {

int pa_version(void) { return 100; }

const char *pa_status_string(int status) {
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_NULL: return "a required pointer is NULL";
    case PA_ERR_SHAPE: return "invalid or inconsistent size";
    case PA_ERR_DTYPE: return "unknown or unsupported dtype combination";
    case PA_ERR_UNSUPPORTED: return "valid but unsupported configuration";
    case PA_ERR_WORKSPACE: return "split-K workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_ALIGN: return "buffer not aligned as required";
    default: return "unknown status";
    }
}

int pa_reshape_and_cache(const void *k, const void *v, void *key_cache, void *value_cache,
                         const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, int dtype,
                         int64_t k_token_stride, int64_t v_token_stride, pa_stream_t stream) {
    return pa_reshape_and_cache_ex(k, v, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                   block_size, num_blocks, dtype, k_token_stride, v_token_stride, 0, stream);
}

int pa_reshape_and_cache_ex(const void *k, const void *v, void *key_cache, void *value_cache,
                            const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                            int head_dim, int block_size, int64_t num_blocks, int dtype,
                            int64_t k_token_stride, int64_t v_token_stride, int flags, pa_stream_t stream) {
    if (flags & ~PA_APPEND_OVERLAP_PREVIOUS) return PA_ERR_UNSUPPORTED;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0) return PA_ERR_SHAPE;
    if (block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    const int E = elem_size(dtype);
    if (!E) return PA_ERR_DTYPE;
    if (dtype == PA_I8) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
    if (k_token_stride < (int64_t)num_kv_heads * head_dim || v_token_stride < (int64_t)num_kv_heads * head_dim)
        return PA_ERR_SHAPE;
    if (num_tokens > 2147483647LL) return PA_ERR_UNSUPPORTED;
    return launch_reshape_and_cache(k, v, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads,
                                    head_dim, num_blocks, E, k_token_stride, v_token_stride,
                                    (flags & PA_APPEND_OVERLAP_PREVIOUS) ? 1 : 0, (cudaStream_t)stream);
}

int pa_block_copy(void *key_cache, void *value_cache, float *k_scales, float *v_scales,
                  const int64_t *src_dst_pairs, int64_t num_pairs, int num_kv_heads, int head_dim,
                  int block_size, int64_t num_blocks, int dtype, pa_stream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0) return PA_ERR_SHAPE;
    if (block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    // a 4-bit cache row is head_dim / 2 bytes: copy it as bytes
    const int E = dtype == PA_I4 ? 1 : elem_size(dtype);
    if (!E) return PA_ERR_DTYPE;
    if (dtype == PA_I4 && head_dim % 2) return PA_ERR_SHAPE;
    const int row_elems = dtype == PA_I4 ? head_dim / 2 : head_dim;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !src_dst_pairs) return PA_ERR_NULL;
    if ((k_scales == nullptr) != (v_scales == nullptr)) return PA_ERR_NULL;
    if (num_pairs > 2147483647LL) return PA_ERR_UNSUPPORTED;
    return launch_block_copy(key_cache, value_cache, k_scales, v_scales, src_dst_pairs, num_pairs,
                             num_kv_heads, row_elems, num_blocks, E, (cudaStream_t)stream);
}

int pa_quantize_int4(const void *src_cache, int src_dtype, uint8_t *dst_cache, float *scales,
                     int64_t num_blocks, int num_kv_heads, int head_dim, int block_size,
                     pa_stream_t stream) {
    if (num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 2) return PA_ERR_SHAPE;
    if (block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    if (src_dtype != PA_F32 && src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_DTYPE;
    if (num_blocks == 0) return PA_OK;
    if (!src_cache || !dst_cache || !scales) return PA_ERR_NULL;
    if (num_blocks * num_kv_heads > 2147483647LL) return PA_ERR_UNSUPPORTED;
    return launch_quantize_int4(src_cache, src_dtype, dst_cache, scales, num_blocks, num_kv_heads, head_dim,
                                (cudaStream_t)stream);
}

int pa_quantize_int8(const void *src_cache, int src_dtype, int8_t *dst_cache, float *scales,
                     int64_t num_blocks, int num_kv_heads, int head_dim, int block_size,
                     pa_stream_t stream) {
    if (num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0) return PA_ERR_SHAPE;
    if (block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    if (src_dtype != PA_F32 && src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_DTYPE;
    if (num_blocks == 0) return PA_OK;
    if (!src_cache || !dst_cache || !scales) return PA_ERR_NULL;
    if (num_blocks * num_kv_heads > 2147483647LL) return PA_ERR_UNSUPPORTED;
    return launch_quantize_int8(src_cache, src_dtype, dst_cache, scales, num_blocks, num_kv_heads, head_dim,
                                (cudaStream_t)stream);
}

int pa_append_int8(const void *k, const void *v, int src_dtype, int8_t *key_cache, int8_t *value_cache,
                   float *k_scales, float *v_scales, const int64_t *slot_mapping, int64_t num_tokens,
                   int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                   int64_t k_token_stride, int64_t v_token_stride, pa_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0) return PA_ERR_SHAPE;
    if (block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    if (src_dtype != PA_F32 && src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_DTYPE;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !key_cache || !value_cache || !k_scales || !v_scales || !slot_mapping) return PA_ERR_NULL;
    if (k_token_stride < (int64_t)num_kv_heads * head_dim || v_token_stride < (int64_t)num_kv_heads * head_dim)
        return PA_ERR_SHAPE;
    if (num_tokens > 2147483647LL) return PA_ERR_UNSUPPORTED;
    return launch_append_int8(k, v, key_cache, value_cache, k_scales, v_scales, slot_mapping, num_tokens,
                              num_kv_heads, head_dim, num_blocks, src_dtype, k_token_stride, v_token_stride,
                              (cudaStream_t)stream);
}

size_t pa_decode_workspace_size(const pa_decode_params *p) {
    Plan pl;
    if (make_plan(p, &pl) != PA_OK) return 0;
    return pl.bytes;
}

}  // extern "C"

namespace pa {

// The new-token rows of pa_decode_append.
// PA_ALGO_AUTO's kernel for groups of 64 query heads per KV head (eight 8-column rows):
// the tcgen05 kernel, which measured 5-27 % faster there than the cooperative mma.sync
// kernel (fp16 and bf16, batches of 16 to 128 sequences of 4096 tokens); for groups of 16
// and 32 the cooperative kernel stays (faster there).
static bool auto_tcgen05(const pa_decode_params *p, const Plan &pl) {
    if (p->algo != PA_ALGO_AUTO || !pl.tc || pl.tc_chunk < 0) return false;
    KernelHeads kh;
    kernel_heads(p, &kh);
    return kh.ngroups == 8 && decode_umma_eligible(p->q_dtype, p->kv_dtype, p->head_dim, kh.G, kh.ngroups, kh.qlen,
                                                   kh.padded, p->partition_size, p->num_seqs);
}

struct AppendIn {
    const void *k, *v;
    const int64_t *slots;
    int64_t k_stride, v_stride;
};

// pa_decode's checks of its buffers, after make_plan.
static int decode_buffers_ok(const void *out, const void *q, const void *key_cache, const void *value_cache,
                             const int32_t *block_tables, const int32_t *seq_lens, const pa_decode_params *p,
                             const Plan &pl) {
    if (!out || !q || !key_cache || !value_cache || !block_tables || !seq_lens) return PA_ERR_NULL;
    if ((p->kv_dtype == PA_I8 || p->kv_dtype == PA_I4) && (!p->k_scales || !p->v_scales)) return PA_ERR_NULL;
    if (((uintptr_t)key_cache | (uintptr_t)value_cache) % 16) return PA_ERR_ALIGN;
    if (pl.bytes > 0 && (!p->workspace || p->workspace_bytes < pl.bytes)) return PA_ERR_WORKSPACE;
    if (pl.bytes > 0 && (uintptr_t)p->workspace % 16) return PA_ERR_ALIGN;
    return PA_OK;
}

// Whether pa_decode_append runs as one kernel: the per-warp tensor-core decode of
// single-token fp16 / bf16 rows, with the new-token rows 16-byte aligned.
static bool append_fusable(const pa_decode_params *p, const Plan &pl, const void *q, const void *k_new,
                           const void *v_new, int64_t k_stride, int64_t v_stride) {
    KernelHeads kh;
    kernel_heads(p, &kh);
    if (!pl.tc || (uintptr_t)q % 16 || kh.qlen > 1 || kh.padded) return false;
    if (p->kv_dtype != p->q_dtype || (p->kv_dtype != PA_F16 && p->kv_dtype != PA_BF16)) return false;
    if (pl.tc_chunk >= 0 &&
        decode_coop_eligible(p->q_dtype, p->kv_dtype, p->head_dim, kh.G, kh.ngroups, kh.qlen, kh.padded, 1))
        return false;
    return ((uintptr_t)k_new | (uintptr_t)v_new) % 16 == 0 && (k_stride * 2) % 16 == 0 && (v_stride * 2) % 16 == 0;
}

// pa_decode with the two knobs of pa_decode_stall_selftest, and the fused append
// of pa_decode_append (ap != nullptr: the caller has checked append_fusable).
static int decode_impl(void *out, const void *q, const void *key_cache, const void *value_cache,
                       const int32_t *block_tables, const int32_t *seq_lens, float scale,
                       const pa_decode_params *p, pa_stream_t stream, int stall_at,
                       unsigned long long wait_ns, const AppendIn *ap = nullptr) {
    Plan pl;
    int rc = make_plan(p, &pl);
    if (rc != PA_OK) return rc;
    if (p->num_seqs == 0) return PA_OK;
    rc = decode_buffers_ok(out, q, key_cache, value_cache, block_tables, seq_lens, p, pl);
    if (rc != PA_OK) return rc;

    DecodeArgs a{};
    a.out = out;
    a.q = q;
    a.kc = key_cache;
    a.vc = value_cache;
    a.ks = p->k_scales;
    a.vs = p->v_scales;
    a.tables = block_tables;
    a.lens = seq_lens;
    a.scale_log2 = scale * kLog2e;
    a.B = p->num_seqs;
    a.Hq = p->num_q_heads;
    KernelHeads kh;
    kernel_heads(p, &kh);
    a.Hkv = kh.Hkv;
    a.ngroups = kh.ngroups;
    a.qlen = kh.qlen;
    a.Greal = kh.Greal;
    a.gcols = kh.gcols;
    a.D = p->head_dim;
    a.G = kh.G;
    a.mbps = p->max_blocks_per_seq;
    a.N = p->num_blocks;
    a.max_len = pl.max_len;
    a.q_dtype = p->q_dtype;
    a.kv_dtype = p->kv_dtype;
    a.out_f32 = (p->flags & PA_DECODE_OUT_F32) ? 1 : 0;
    a.stall_at = stall_at;
    a.wait_ns = wait_ns;
    a.umma = (p->algo == PA_ALGO_TCGEN05 || auto_tcgen05(p, pl)) ? 1 : 0;
    if (ap) {
        a.append = 1;
        a.k_new = ap->k;
        a.v_new = ap->v;
        a.slot_new = ap->slots;
        a.kn_stride = ap->k_stride;
        a.vn_stride = ap->v_stride;
    }
    char *ws = reinterpret_cast<char *>(p->workspace);
    if (pl.tc && (uintptr_t)q % 16) {
        if (p->algo == PA_ALGO_TENSOR || p->algo == PA_ALGO_TCGEN05 || stall_at >= 0) return PA_ERR_ALIGN;
        // the tensor-core family reads q rows with 16-byte bulk copies; a q that is not
        // 16-byte aligned goes to the CUDA-core family, which needs its own plan
        pa_decode_params p2 = *p;
        p2.algo = PA_ALGO_SIMT;
        return decode_impl(out, q, key_cache, value_cache, block_tables, seq_lens, scale, &p2, stream, -1,
                           wait_ns);
    }
    if (stall_at >= 0 && !pl.tc) return PA_ERR_UNSUPPORTED;
    // workspace: the partial outputs, then their lse
    if (pl.tc) {
        a.part = 0;
        a.max_parts = 1;
        a.tc_chunk = pl.tc_chunk;
        a.early = (p->flags & PA_DECODE_INPUTS_READY) ? 1 : 0;
        if (pl.bytes > 0) {
            // the cooperative mode keeps all 8 * ngroups columns of a cache row per slot
            const bool coop = decode_coop_eligible(a.q_dtype, a.kv_dtype, a.D, a.G, a.ngroups, a.qlen,
                                                   (int64_t)a.G * a.ngroups != a.gcols, 1);
            const size_t o_bytes = up256((size_t)pl.tc_slots * a.G * (coop ? a.ngroups : 1) * a.D * sizeof(float));
            a.ws_o = reinterpret_cast<float *>(ws);
            a.ws_lse = reinterpret_cast<float *>(ws + o_bytes);
        }
        return launch_decode_tc(a, (cudaStream_t)stream);
    }
    a.part = pl.part;
    a.max_parts = pl.max_parts;
    if (pl.bytes > 0) {
        const size_t o_bytes = up256((size_t)a.B * a.Hq * pl.max_parts * a.D * sizeof(float));
        a.ws_o = reinterpret_cast<float *>(ws);
        a.ws_lse = reinterpret_cast<float *>(ws + o_bytes);
    }
    if (pl.max_len == 0) {
        // every row is zero: the one-pass kernel writes zeros for seq_len <= 0
        a.part = 0;
        a.max_parts = 1;
    }
    return launch_decode_simt(a, (cudaStream_t)stream);
}

}  // namespace pa

extern "C" {

int pa_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
              const int32_t *block_tables, const int32_t *seq_lens, float scale,
              const pa_decode_params *p, pa_stream_t stream) {
    return decode_impl(out, q, key_cache, value_cache, block_tables, seq_lens, scale, p, stream, -1,
                       kWaitLimitNs);
}

int pa_decode_stall_selftest(void *out, const void *q, const void *key_cache, const void *value_cache,
                             const int32_t *block_tables, const int32_t *seq_lens, float scale,
                             const pa_decode_params *p, int stall_at, uint64_t limit_ns,
                             pa_stream_t stream) {
    if (stall_at < 0 || limit_ns == 0) return PA_ERR_SHAPE;
    return decode_impl(out, q, key_cache, value_cache, block_tables, seq_lens, scale, p, stream, stall_at,
                       (unsigned long long)limit_ns);
}

int pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slot_mapping,
                     int64_t k_token_stride, int64_t v_token_stride, void *key_cache, void *value_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, float scale, const pa_decode_params *p,
                     pa_stream_t stream) {
    const int fused = pa_decode_append_fused(p, q, k_new, v_new, k_token_stride, v_token_stride);
    if (fused < 0) return fused;
    if (p->num_seqs == 0) return PA_OK;
    if (!slot_mapping) return PA_ERR_NULL;
    Plan pl;
    make_plan(p, &pl);
    const int rc = decode_buffers_ok(out, q, key_cache, value_cache, block_tables, seq_lens, p, pl);
    if (rc != PA_OK) return rc;
    if (fused) {
        const AppendIn ap{k_new, v_new, slot_mapping, k_token_stride, v_token_stride};
        return decode_impl(out, q, key_cache, value_cache, block_tables, seq_lens, scale, p, stream, -1,
                           kWaitLimitNs, &ap);
    }
    const int ra = pa_reshape_and_cache(k_new, v_new, key_cache, value_cache, slot_mapping, p->num_seqs,
                                        p->num_kv_heads, p->head_dim, p->block_size, p->num_blocks, p->kv_dtype,
                                        k_token_stride, v_token_stride, stream);
    if (ra != PA_OK) return ra;
    return decode_impl(out, q, key_cache, value_cache, block_tables, seq_lens, scale, p, stream, -1,
                       kWaitLimitNs);
}

int pa_decode_append_fused(const pa_decode_params *p, const void *q, const void *k_new, const void *v_new,
                           int64_t k_token_stride, int64_t v_token_stride) {
    Plan pl;
    const int rc = make_plan(p, &pl);
    if (rc != PA_OK) return rc;
    if (p->query_len > 1) return PA_ERR_UNSUPPORTED;
    if (p->kv_dtype != p->q_dtype) return PA_ERR_DTYPE;
    if (p->num_seqs > 0 && (!k_new || !v_new)) return PA_ERR_NULL;
    if (k_token_stride < (int64_t)p->num_kv_heads * p->head_dim ||
        v_token_stride < (int64_t)p->num_kv_heads * p->head_dim)
        return PA_ERR_SHAPE;
    return append_fusable(p, pl, q, k_new, v_new, k_token_stride, v_token_stride) ? 1 : 0;
}

int pa_decode_algo(const pa_decode_params *p, const void *q) {
    Plan pl;
    const int rc = make_plan(p, &pl);
    if (rc != PA_OK) return rc;
    if (pl.tc && (uintptr_t)q % 16)
        return p->algo == PA_ALGO_TENSOR || p->algo == PA_ALGO_TCGEN05 ? PA_ERR_ALIGN : PA_ALGO_SIMT;
    if (p->algo == PA_ALGO_TCGEN05 || auto_tcgen05(p, pl)) return PA_ALGO_TCGEN05;
    return pl.tc ? PA_ALGO_TENSOR : PA_ALGO_SIMT;
}

int pa_decode_launches(const pa_decode_params *p, const void *q) {
    const int fam = pa_decode_algo(p, q);
    if (fam < 0) return fam;
    Plan pl;
    if (fam == PA_ALGO_SIMT) {
        pa_decode_params p2 = *p;
        p2.algo = PA_ALGO_SIMT;
        const int rc = make_plan(&p2, &pl);
        if (rc != PA_OK) return rc;
        return pl.bytes > 0 && pl.max_len > 0 ? 2 : 1;  // merge_kernel after a split decode
    }
    const int rc = make_plan(p, &pl);
    if (rc != PA_OK) return rc;
    return pl.bytes > 0 ? 2 : 1;  // merge_tc_kernel after a split decode
}

int pa_get_error_flags(unsigned int *flags, int reset, pa_stream_t stream) {
    if (!flags) return PA_ERR_NULL;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PA_ERR_CUDA;
    int (*const words[])(unsigned int *, bool) = {error_word_cache_ops, error_word_decode_simt,
                                                  error_word_decode_tc, error_word_decode_umma};
    unsigned int all = 0;
    for (auto w : words) {
        unsigned int f = 0;
        if (w(&f, reset != 0) != PA_OK) return PA_ERR_CUDA;
        all |= f;
    }
    *flags = all;
    return PA_OK;
}

}  // extern "C"
