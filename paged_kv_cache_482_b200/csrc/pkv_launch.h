// pkv_launch.h -- internal launchers behind the C ABI (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pkv {

cudaError_t launch_store_kvcache(const void *k, const void *v, void *k_cache, void *v_cache,
                                 const int32_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                 int block_size, int64_t num_blocks, int mode, float *k_scale, float *v_scale,
                                 int *dev_err, int num_sms, cudaStream_t stream);

cudaError_t launch_store_kvcache_rope(const void *q, void *q_out, const void *k, const void *v, void *k_cache,
                                      void *v_cache, const int32_t *slot_mapping, const int32_t *positions,
                                      const float *cos_sin, int max_position, int style, int num_tokens,
                                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                      int64_t num_blocks, int mode, float *k_scale, float *v_scale, int *dev_err,
                                      int num_sms, cudaStream_t stream);

// Everything the decode kernels need, resolved by the host layer.
struct DecodeArgs {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens;
    const int32_t *seq_order;  // may be null
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int head_dim;
    int block_size;
    int64_t num_blocks;
    float scale;
    bool fp8;
    bool token_scales;  // E4M3 with scale pools [num_blocks][num_kv_heads][block_size]
    const float *k_scale;
    const float *v_scale;
    int max_context_len;
    int partition_tokens;  // 0: one partition per sequence
    int num_partitions;    // grid partitions per (sequence, KV head)
    float *part_o;         // [num_seqs][num_q_heads][num_partitions][head_dim]
    float *part_ml;        // [num_seqs][num_q_heads][num_partitions][2]
    void *out;
    int *dev_err;
    // one-token chunks of a chunked-prefill call (null for a decode call):
    // sequence i is served only if cu_q_lens[i + 1] - cu_q_lens[i] == 1, and
    // its q / out row is cu_q_lens[i]
    const int32_t *cu_q_lens = nullptr;
    int total_q = 0;
    // shared-prefix (cascade) mode (null: off): groups of sequences
    // cu_group_seqs[j] .. cu_group_seqs[j + 1] - 1 share their first
    // group_prefix[j] tokens; num_partitions then counts the prefix slot too
    const int32_t *cu_group_seqs = nullptr;
    const int32_t *group_prefix = nullptr;
    int num_groups = 0;
    int max_group_seqs = 0;
};

// Tile (tokens per pipeline stage) of the decode kernel chosen for a shape;
// split-K partitions are whole multiples of it. 0 when unsupported.
int decode_tile_tokens(int head_dim, int group, bool fp8);
// Largest number of physical blocks one partition may span.
int decode_max_blocks_per_partition();

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Everything the chunked-prefill kernel needs, resolved by the host layer.
struct PrefillArgs {
    const void *q;  // [total_q][num_q_heads][head_dim] bf16
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *cu_q_lens;     // [num_seqs + 1]
    const int32_t *context_lens;  // [num_seqs]
    int num_seqs;
    int total_q;
    int num_q_heads;
    int num_kv_heads;
    int head_dim;
    int block_size;
    int64_t num_blocks;
    float scale;
    bool fp8;
    bool token_scales;  // E4M3 with scale pools [num_blocks][num_kv_heads][block_size]
    const float *k_scale;
    const float *v_scale;
    int max_q_len;
    void *out;
    int *dev_err;
    // routing between the one-tile and warp-specialised kernels (set by
    // launch_prefill): 0 = none;
    // > 0: the one-tile kernel takes the sequences with chunks of at most
    // small_cut tokens, the warp-specialised kernel the others
    int small_cut;
    // the one-tile kernel skips chunks shorter than this (one-token chunks
    // go to the decode kernel when it is 2)
    int small_min = 0;
    // E4M3 only, may be null: the widening workspace (prefill_ws.cu, Staging)
    // and its rows per (sequence, KV head), a multiple of 128
    void *staging = nullptr;
    int staging_stride = 0;
    // shared-prefix mode of the warp-specialised kernel (launch_prefix_tc;
    // null: off): the rows of group j are its members' queries (sequences
    // cu_group_seqs[j] ..), the keys its group_prefix[j] shared tokens, and
    // each row's result its split-K slot-0 partial in part_o / part_ml
    const int32_t *cu_group_seqs = nullptr;
    const int32_t *group_prefix = nullptr;
    int num_groups = 0;
    int max_context_len = 0;
    float *part_o = nullptr;
    float *part_ml = nullptr;
    int num_partitions = 0;
};

// The shared prefixes of a cascade decode (DecodeArgs with cu_group_seqs)
// on the tensor cores: every member's slot-0 partial. bf16 cache, head_dim
// 128 (prefix_tc_supported); the decode kernel then attends the suffixes.
bool prefix_tc_supported(int head_dim, int group, bool fp8);
cudaError_t launch_prefix_tc(const DecodeArgs &d, cudaStream_t stream);

// The library's low-priority stream of the current device (created on first
// use, kept for the process; null if it cannot be made). Work put on it is
// forked from and joined back into the caller's stream with events.
cudaStream_t library_side_stream();

// Staging rows per (sequence, KV head) of the E4M3 prefill workspace (the
// table capacity rounded up to 128) and the workspace's bytes; 0 when there
// is no staging (bf16 cache, or more rows than int32 tensor-map coordinates).
int prefill_staging_stride(int max_blocks_per_seq, int block_size);
size_t prefill_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq, int block_size,
                               bool fp8, bool token_scales);

struct NormArgs {
    const void *x;   // [num_tokens][hidden] bf16
    void *residual;  // [num_tokens][hidden] bf16, in / out; may be null
    const void *weight;
    void *out;
    int num_tokens;
    int hidden;
    float eps;
};

int norm_max_hidden();
cudaError_t launch_fused_add_rmsnorm(const NormArgs &a, int num_sms, cudaStream_t stream);

bool prefill_supported(int head_dim, int group);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_ws(const PrefillArgs &a, cudaStream_t stream);  // warp-specialised, every cache type

}  // namespace pkv
