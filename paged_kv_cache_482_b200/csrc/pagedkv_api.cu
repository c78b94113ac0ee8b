// pagedkv_api.cu -- the C ABI of libpagedkv.so (declared in include/pagedkv.h).
//
// Host side only: argument checks, the split-K plan, and the launches. Every
// check that can fail does so before anything is queued on the stream.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "pagedkv.h"
#include "pkv_launch.h"

namespace {

constexpr int kDefaultSms = 148;
constexpr int kMaxPartitions = 1024;        // the reduce kernel's limit
constexpr int kMinAutoPartitionTokens = 1024;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(int d) { return d == PKV_CACHE_BF16 || d == PKV_CACHE_FP8_E4M3 || d == PKV_CACHE_FP8_E4M3_TOKEN; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return kDefaultSms;
    }
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return kDefaultSms;
    }
    return n;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shape checks shared by the plan and the decode call.
int check_shape(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                int max_context_len, int cache_dtype) {
    if (num_seqs < 0 || num_q_heads < 1 || num_kv_heads < 1 || max_context_len < 1) return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(cache_dtype)) return PKV_ERR_INVALID_ARG;
    if (!pow2(block_size) || block_size < 8 || block_size > 1024) return PKV_ERR_INVALID_ARG;
    if (pkv::decode_tile_tokens(head_dim, num_q_heads / num_kv_heads, cache_dtype != PKV_CACHE_BF16) == 0)
        return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}

int make_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_context_len,
              int cache_dtype, int request, pkv_decode_plan *plan) {
    int st = check_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, cache_dtype);
    if (st != PKV_OK) return st;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    const int tile = pkv::decode_tile_tokens(head_dim, num_q_heads / num_kv_heads, fp8);
    // A partition may span at most this many blocks (ids staged on chip); a
    // partition of pt tokens spans at most pt / block_size + 1 blocks.
    const long long max_pt_ids = (long long)(pkv::decode_max_blocks_per_partition() - 1) * block_size;
    const long long max_pt = max_pt_ids / tile * tile;
    long long pt = 0;  // 0: no split
    if (request == -1) {
        // one partition per sequence, of any length (block ids beyond the
        // staged ones are read from the table)
    } else if (request > 0) {
        pt = round_up((size_t)request, (size_t)tile);
        if (pt >= max_context_len) pt = 0;
    } else if (request == 0) {
        const long long units = (long long)num_seqs * num_kv_heads;
        const long long slots = (long long)num_sms() * 3;  // resident blocks
        const bool fits = (long long)max_context_len <= max_pt_ids;
        if (!fits || units < 2 * slots) {
            const long long want = (8 * slots + units - 1) / (units > 0 ? units : 1);
            long long t = (max_context_len + want - 1) / want;
            if (t < kMinAutoPartitionTokens) t = kMinAutoPartitionTokens;
            t = (long long)round_up((size_t)t, (size_t)tile);
            if (t > max_pt) t = max_pt;
            // pkv_decode_workspace_bytes relies on automatic partitions never
            // being shorter than kMinAutoPartitionTokens
            if (t < kMinAutoPartitionTokens) return PKV_ERR_UNSUPPORTED;
            if (t < max_context_len) pt = t;
        }
    } else {
        return PKV_ERR_INVALID_ARG;
    }
    int np = 1;
    if (pt > 0) {
        np = (int)((max_context_len + pt - 1) / pt);
        if (np > kMaxPartitions) return PKV_ERR_UNSUPPORTED;
    }
    plan->partition_tokens = (int)pt;
    plan->max_partitions = np;
    plan->workspace_bytes = 0;
    if (pt > 0) {
        const size_t rows = (size_t)num_seqs * num_q_heads * np;
        plan->workspace_bytes = round_up(rows * head_dim * sizeof(float), 256) + round_up(rows * 2 * sizeof(float), 256);
    }
    return PKV_OK;
}

}  // namespace

extern "C" {

int pkv_version(void) { return 0x000100; }

const char *pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported shape";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_DEVICE_BOUNDS: return "device bounds error (slot, block id or length outside the pool)";
        case PKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

int pkv_store_kvcache(const void *k, const void *v, void *k_cache, void *v_cache, const int32_t *slot_mapping,
                      int num_tokens, int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                      int cache_dtype, float *k_scale, float *v_scale, int *dev_err, void *stream) {
    if (num_tokens < 0 || num_kv_heads < 1 || head_dim < 8 || head_dim % 8 != 0 || block_size < 1 ||
        num_blocks < 1)
        return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(cache_dtype)) return PKV_ERR_INVALID_ARG;
    // per-token scales: the lanes of one row reduce its amax together
    if (cache_dtype == PKV_CACHE_FP8_E4M3_TOKEN && (!pow2(head_dim / 8) || head_dim > 256))
        return PKV_ERR_UNSUPPORTED;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    if (num_tokens == 0) return PKV_OK;  // no rows to read: k, v, slot_mapping may be NULL
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_store_kvcache(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads,
                                              head_dim, block_size, num_blocks, cache_dtype, k_scale, v_scale,
                                              dev_err, num_sms(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_store_kvcache_rope(const void *q, void *q_out, const void *k, const void *v, void *k_cache, void *v_cache,
                           const int32_t *slot_mapping, const int32_t *positions, const float *cos_sin,
                           int max_position, int rope_style, int num_tokens, int num_q_heads, int num_kv_heads,
                           int head_dim, int block_size, int64_t num_blocks, int cache_dtype, float *k_scale,
                           float *v_scale, int *dev_err, void *stream) {
    if (num_tokens < 0 || num_kv_heads < 1 || head_dim < 16 || head_dim % 16 != 0 || block_size < 1 ||
        num_blocks < 1 || max_position < 1 || (rope_style != 0 && rope_style != 1))
        return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(cache_dtype)) return PKV_ERR_INVALID_ARG;
    // a row spans head_dim / 16 adjacent lanes (a power of two up to 32)
    if (!pow2(head_dim / 16) || head_dim > 512) return PKV_ERR_UNSUPPORTED;
    if ((q == nullptr) != (q_out == nullptr)) return PKV_ERR_INVALID_ARG;
    if (q && num_q_heads < 1) return PKV_ERR_INVALID_ARG;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping || !positions || !cos_sin) return PKV_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(cos_sin) ||
        (q && (!aligned16(q) || !aligned16(q_out))))
        return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_store_kvcache_rope(q, q_out, k, v, k_cache, v_cache, slot_mapping, positions,
                                                   cos_sin, max_position, rope_style, num_tokens, num_q_heads,
                                                   num_kv_heads, head_dim, block_size, num_blocks, cache_dtype,
                                                   k_scale, v_scale, dev_err, num_sms(),
                                                   static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_plan_decode(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_context_len, int cache_dtype, int partition_request, pkv_decode_plan *plan) {
    if (!plan) return PKV_ERR_INVALID_ARG;
    return make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, cache_dtype,
                     partition_request, plan);
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len) {
    if (num_seqs < 1 || num_q_heads < 1 || head_dim < 1 || max_context_len < 1) return 0;
    // An automatic plan never cuts partitions shorter than
    // kMinAutoPartitionTokens (and the longest partition cap is above it for
    // every supported block size), so it has at most this many partitions.
    const long long np = ((long long)max_context_len + kMinAutoPartitionTokens - 1) / kMinAutoPartitionTokens;
    if (np <= 1) return 0;
    const size_t rows = (size_t)num_seqs * num_q_heads * (size_t)np;
    return round_up(rows * head_dim * sizeof(float), 256) + round_up(rows * 2 * sizeof(float), 256);
}

namespace {

// Plan of the shared-prefix decode: the suffix partitions of the ordinary
// plan (one, of max_context_len tokens, when it does not split) plus slot 0.
int make_shared_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_context_len, int cache_dtype, int request, pkv_decode_plan *plan) {
    int st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, cache_dtype,
                       request, plan);
    if (st != PKV_OK) return st;
    if (head_dim != 128) return PKV_OK;  // served by the ordinary decode (same result)
    const int np_suffix = plan->partition_tokens > 0 ? plan->max_partitions : 1;
    if (np_suffix + 1 > kMaxPartitions) return PKV_ERR_UNSUPPORTED;
    if (plan->partition_tokens == 0) plan->partition_tokens = max_context_len;
    plan->max_partitions = np_suffix + 1;
    const size_t rows = (size_t)num_seqs * num_q_heads * plan->max_partitions;
    plan->workspace_bytes = round_up(rows * head_dim * sizeof(float), 256) + round_up(rows * 2 * sizeof(float), 256);
    return PKV_OK;
}

}  // namespace

int pkv_plan_decode_shared_prefix(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int max_context_len, int cache_dtype, int partition_request,
                                  pkv_decode_plan *plan) {
    if (!plan) return PKV_ERR_INVALID_ARG;
    return make_shared_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, cache_dtype,
                            partition_request, plan);
}

int pkv_paged_attention_decode_shared_prefix(const void *q, const void *k_cache, const void *v_cache,
                                             const int32_t *block_tables, int max_blocks_per_seq,
                                             const int32_t *context_lens, const int32_t *seq_order, int num_seqs,
                                             int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                             int64_t num_blocks,
                                             float scale, int cache_dtype, const float *k_scale,
                                             const float *v_scale, int max_context_len,
                                             const int32_t *cu_group_seqs, const int32_t *group_prefix_tokens,
                                             int num_groups, int max_group_seqs, int partition_request,
                                             void *workspace, size_t workspace_bytes, void *out, int *dev_err,
                                             void *stream) {
    if (num_groups < 0 || (num_groups > 0 && (!cu_group_seqs || !group_prefix_tokens || max_group_seqs < 1)))
        return PKV_ERR_INVALID_ARG;
    if (num_groups == 0 || head_dim != 128)  // nothing declared shared, or no prefix kernel for this head size
        return pkv_paged_attention_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                          seq_order, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                          num_blocks, scale, cache_dtype, k_scale, v_scale, max_context_len,
                                          partition_request, workspace, workspace_bytes, out, dev_err, stream);
    pkv_decode_plan plan;
    int st = make_shared_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                              cache_dtype, partition_request, &plan);
    if (st != PKV_OK) return st;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    if (max_blocks_per_seq < 1 || num_blocks < 1 || num_blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size) return PKV_ERR_INVALID_ARG;
    if (!(scale == scale)) return PKV_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < plan.workspace_bytes) return PKV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;

    pkv::DecodeArgs a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.context_lens = context_lens;
    a.seq_order = seq_order;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.scale = scale;
    a.fp8 = fp8;
    a.token_scales = cache_dtype == PKV_CACHE_FP8_E4M3_TOKEN;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.max_context_len = max_context_len;
    a.partition_tokens = plan.partition_tokens;
    a.num_partitions = plan.max_partitions;
    const size_t rows = (size_t)num_seqs * num_q_heads * plan.max_partitions;
    a.part_o = static_cast<float *>(workspace);
    a.part_ml =
        reinterpret_cast<float *>(static_cast<char *>(workspace) + round_up(rows * head_dim * sizeof(float), 256));
    a.out = out;
    a.dev_err = dev_err;
    a.cu_group_seqs = cu_group_seqs;
    a.group_prefix = group_prefix_tokens;
    a.num_groups = num_groups;
    a.max_group_seqs = max_group_seqs;
    cudaError_t e = pkv::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidConfiguration) return PKV_ERR_UNSUPPORTED;
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_paged_attention_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                               int max_blocks_per_seq, const int32_t *context_lens, const int32_t *seq_order,
                               int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                               int cache_dtype, const float *k_scale, const float *v_scale, int max_context_len,
                               int partition_request, void *workspace, size_t workspace_bytes, void *out,
                               int *dev_err, void *stream) {
    pkv_decode_plan plan;
    int st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, cache_dtype,
                       partition_request, &plan);
    if (st != PKV_OK) return st;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PKV_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    if (max_blocks_per_seq < 1 || num_blocks < 1 || num_blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size) return PKV_ERR_INVALID_ARG;
    if (!(scale == scale)) return PKV_ERR_INVALID_ARG;  // NaN
    if (plan.workspace_bytes > 0) {
        if (!workspace || workspace_bytes < plan.workspace_bytes) return PKV_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_INVALID_ARG;
    }
    if (num_seqs == 0) return PKV_OK;

    pkv::DecodeArgs a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.context_lens = context_lens;
    a.seq_order = seq_order;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.scale = scale;
    a.fp8 = fp8;
    a.token_scales = cache_dtype == PKV_CACHE_FP8_E4M3_TOKEN;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.max_context_len = max_context_len;
    a.partition_tokens = plan.partition_tokens;
    a.num_partitions = plan.max_partitions;
    a.part_o = nullptr;
    a.part_ml = nullptr;
    if (plan.workspace_bytes > 0) {
        const size_t rows = (size_t)num_seqs * num_q_heads * plan.max_partitions;
        a.part_o = static_cast<float *>(workspace);
        a.part_ml = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                              round_up(rows * head_dim * sizeof(float), 256));
    }
    a.out = out;
    a.dev_err = dev_err;
    cudaError_t e = pkv::launch_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

size_t pkv_prefill_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                                   int block_size, int cache_dtype) {
    if (!valid_dtype(cache_dtype)) return 0;
    return pkv::prefill_workspace_bytes(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
                                        cache_dtype != PKV_CACHE_BF16, cache_dtype == PKV_CACHE_FP8_E4M3_TOKEN);
}

int pkv_paged_attention_prefill(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq, const int32_t *cu_q_lens,
                                const int32_t *context_lens, int num_seqs, int total_q, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                                int cache_dtype, const float *k_scale, const float *v_scale, int max_q_len,
                                void *workspace, size_t workspace_bytes, void *out, int *dev_err, void *stream) {
    if (num_seqs < 0 || total_q < 0 || num_q_heads < 1 || num_kv_heads < 1) return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(cache_dtype)) return PKV_ERR_INVALID_ARG;
    if (!pow2(block_size) || block_size < 8 || block_size > 1024) return PKV_ERR_INVALID_ARG;
    if (!pkv::prefill_supported(head_dim, num_q_heads / num_kv_heads)) return PKV_ERR_UNSUPPORTED;
    const bool fp8 = cache_dtype != PKV_CACHE_BF16;
    if (!q || !k_cache || !v_cache || !block_tables || !cu_q_lens || !context_lens || !out)
        return PKV_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    if (max_blocks_per_seq < 1 || num_blocks < 1 || num_blocks > INT32_MAX) return PKV_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale > 3.0e38f) return PKV_ERR_INVALID_ARG;  // positive and finite
    if (workspace && !aligned16(workspace)) return PKV_ERR_INVALID_ARG;
    // the widening workspace: used by an E4M3 cache when its bound is nonzero
    size_t staging_need = 0;
    if (workspace && fp8) {
        staging_need = pkv_prefill_workspace_bytes(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
                                                   cache_dtype);
        if (staging_need && workspace_bytes < staging_need) return PKV_ERR_WORKSPACE;
    }
    if (num_seqs == 0 || total_q == 0) return PKV_OK;
    if (max_q_len < 1) return PKV_ERR_INVALID_ARG;

    pkv::PrefillArgs a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.cu_q_lens = cu_q_lens;
    a.context_lens = context_lens;
    a.num_seqs = num_seqs;
    a.total_q = total_q;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.scale = scale;
    a.fp8 = fp8;
    a.token_scales = cache_dtype == PKV_CACHE_FP8_E4M3_TOKEN;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.max_q_len = max_q_len;
    a.out = out;
    a.dev_err = dev_err;
    a.small_cut = 0;
    if (staging_need) {
        a.staging = workspace;
        a.staging_stride = pkv::prefill_staging_stride(max_blocks_per_seq, block_size);
    }
    cudaError_t e = pkv::launch_prefill(a, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidConfiguration) return PKV_ERR_UNSUPPORTED;
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_fused_add_rmsnorm(const void *x, void *residual, const void *weight, void *out, int num_tokens, int hidden,
                          float eps, void *stream) {
    if (!x || !weight || !out || num_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (hidden < 8 || hidden % 8 != 0) return PKV_ERR_INVALID_ARG;
    if (hidden > pkv::norm_max_hidden()) return PKV_ERR_UNSUPPORTED;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return PKV_ERR_INVALID_ARG;  // negative, NaN or infinite
    if (!aligned16(x) || !aligned16(weight) || !aligned16(out) || (residual && !aligned16(residual)))
        return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    pkv::NormArgs a{x, residual, weight, out, num_tokens, hidden, eps};
    cudaError_t e = pkv::launch_fused_add_rmsnorm(a, num_sms(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_read_device_error(const int *dev_err, void *stream) {
    if (!dev_err) return PKV_ERR_INVALID_ARG;
    int h = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&h, dev_err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PKV_ERR_CUDA;
    if (h & PKV_DEVERR_TIMEOUT) return PKV_ERR_DEVICE_TIMEOUT;
    if (h & PKV_DEVERR_BOUNDS) return PKV_ERR_DEVICE_BOUNDS;
    return PKV_OK;
}

}  // extern "C"
