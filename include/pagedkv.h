/*
 * pagedkv.h -- C ABI of libpagedkv.so: one decode step of attention over a
 * paged KV cache, on B200 (sm_100a).
 *
 * The operation. The KV cache is cut into fixed-size blocks that live
 * anywhere in a physical pool; a per-sequence block table maps the logical
 * block j of a sequence to a physical block, and several sequences may map
 * to the same physical blocks (a shared prefix). Pages: "DeepSeek复刻vLLM反超
 * 原版：AI推理新标杆", section "vLLM：大模型推理的加速引擎与挑战" (block table
 * from logical to physical blocks, KV sharing within and across requests);
 * "nano-vllm：轻量级大模型推理引擎的技术探索与实践", section "PagedAttention 原理
 * 回顾" (fixed-size blocks, non-contiguous allocation); "Nano-vLLM：轻量高效的
 * 大模型推理框架", section 三.1 (the block manager hands each request its
 * blocks). The decode attends one new query token per sequence over its
 * cached tokens in logical order, out = softmax(scale * q K^T) V, which the
 * pages describe as bound by KV-cache read bandwidth ("nano-vllm-lite：深入
 * 理解LLM推理机制的教育级开源项目", section 核心技术改进 2); the optional FP8
 * cache is from the same page, section 核心技术改进 3 "FP8 KV Cache量化".
 *
 * Conventions (readings where the pages are silent):
 *  - Pool layout: k_cache and v_cache are [num_blocks][num_kv_heads]
 *    [block_size][head_dim], row-major, element type bf16 or E4M3 (1 byte).
 *    Slot s is block s / block_size, offset s % block_size.
 *  - Grouped-query attention: query head h reads KV head
 *    h / (num_q_heads / num_kv_heads).
 *  - context_lens[i] counts the step's own token, which store_kvcache
 *    writes before the decode on the same stream.
 *  - FP8: code = E4M3(x / scale[h]) with one IEEE fp32 division, round to
 *    nearest even, saturating at +-448; value = code * scale[h].
 *  - FP8 with per-token scales (PKV_CACHE_FP8_E4M3_TOKEN; the page leaves
 *    the scale granularity open): k_scale / v_scale are scale pools
 *    [num_blocks][num_kv_heads][block_size] fp32, one scale per cached
 *    (token, KV head) row. store_kvcache computes s = max(amax / 448, the
 *    smallest normal fp32) for each row it writes (amax: the row's largest
 *    |x|; one IEEE division), writes s at the row's slot and the codes
 *    E4M3(x / s); a read is code * s of its own row. The scale pools need no
 *    initialisation: only written rows are read.
 *
 * Ownership and execution. The caller owns every buffer (device memory unless
 * stated) and keeps it alive until the stream work finishes. The library
 * allocates no device memory. Its only state across calls is looked up or
 * created once per device and kept for the process: the static scratch's
 * device address (pkv_paged_attention_decode_static_scratch) and one
 * low-priority stream for the one-token chunks of a mixed prefill batch
 * (pkv_paged_attention_prefill). Calls are re-entrant. Every call is
 * asynchronous on the given stream (a cudaStream_t passed as void*; NULL is
 * the legacy default stream) and returns once the work is queued; work the
 * library puts on its own stream is joined back into the given stream with
 * events before the call returns, so the call stays stream-ordered.
 *
 * Errors. Arguments the host can check are checked before anything is
 * launched; a failed check returns the status and launches nothing. Faults
 * only the device can see (a slot, block id or length outside the pool or
 * the table) set bits in *dev_err (device memory, one int, OR-ed atomically;
 * the caller zeroes it) and the affected rows are skipped or written as
 * zeros; the kernels never trap. A bounded wait inside a kernel that gives
 * up sets PKV_DEVERR_TIMEOUT. dev_err may be NULL, in which case those
 * faults are still skipped but not reported.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size */
    PKV_ERR_UNSUPPORTED = 2,   /* shape the kernels are not built for */
    PKV_ERR_WORKSPACE = 3,     /* workspace missing or too small */
    PKV_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
    PKV_ERR_DEVICE_BOUNDS = 5, /* pkv_read_device_error: bounds bit set */
    PKV_ERR_DEVICE_TIMEOUT = 6 /* pkv_read_device_error: timeout bit set */
} pkv_status;

typedef enum {
    PKV_CACHE_BF16 = 0,
    PKV_CACHE_FP8_E4M3 = 1,      /* one fp32 scale per KV head: [num_kv_heads] */
    PKV_CACHE_FP8_E4M3_TOKEN = 2 /* one fp32 scale per (token, KV head): scale pools */
} pkv_cache_dtype;

/* Bits of the device error word. */
#define PKV_DEVERR_BOUNDS 0x1
#define PKV_DEVERR_TIMEOUT 0x2

/*
 * store_kvcache: for each token t < num_tokens with slot_mapping[t] >= 0,
 * write k[t] and v[t] (all KV heads) into that slot of k_cache / v_cache.
 * slot_mapping[t] == -1 skips token t (e.g. a token already held by a shared
 * prefix block).
 *
 *  k, v          [num_tokens][num_kv_heads][head_dim] bf16, contiguous
 *  k_cache, ...  pools as above; bf16 (copy) or E4M3 (quantised)
 *  slot_mapping  [num_tokens] int32
 *  k_scale, ...  FP8 only (NULL for bf16): [num_kv_heads] fp32, read; or, for
 *                PKV_CACHE_FP8_E4M3_TOKEN, the scale pools, written at each
 *                stored row's slot (head_dim / 8 must then be a power of two
 *                up to 32, i.e. head_dim 8 .. 256)
 *
 * Host checks: non-null pointers, 16-byte aligned k/v/caches, head_dim a
 * multiple of 8, sizes >= 1 (num_tokens may be 0: nothing is launched and no
 * pointer is looked at).
 * Device check: slot >= num_blocks * block_size sets PKV_DEVERR_BOUNDS and
 * the token is not written.
 */
PKV_API int pkv_store_kvcache(const void *k, const void *v, void *k_cache, void *v_cache,
                      const int32_t *slot_mapping, int num_tokens, int num_kv_heads,
                      int head_dim, int block_size, int64_t num_blocks, int cache_dtype,
                      float *k_scale, float *v_scale, int *dev_err, void *stream);

/*
 * store_kvcache_rope: the rotary position embedding of q and k fused with
 * store_kvcache. The FP8 cache of "nano-vllm-lite：深入理解LLM推理机制的教育级开
 * 源项目" (section 核心技术改进 3) holds rotated keys, so the rotation that
 * precedes the write is done in the same pass. The rotation is the RoFormer
 * paper's (Su et al., 2021): pair i of a row at position m = positions[t]
 * turns by the angle whose cosine and sine are cos_sin[m][i] and
 * cos_sin[m][head_dim/2 + i]; the caller builds the table once
 * (theta_i = base^(-2i/head_dim) in the paper). For every element pair, in
 * binary32 with one rounding per step and then bf16 round-to-nearest-even:
 *   x' = fma(-y, sin, x * cos),  y' = fma(x, sin, y * cos)
 * Pairs are (i, i + head_dim/2) for rope_style 0 and (2i, 2i + 1) for
 * rope_style 1. The result is exactly store_kvcache of the rotated k (bf16)
 * and of v, and q_out = the rotated q.
 *
 *  q, q_out      [num_tokens][num_q_heads][head_dim] bf16, or both NULL (keys
 *                only); q_out may be q (in place)
 *  k, v          [num_tokens][num_kv_heads][head_dim] bf16
 *  positions     [num_tokens] int32, each in [0, max_position)
 *  cos_sin       [max_position][head_dim] fp32 (cos of the head_dim/2 angles,
 *                then their sin), 16-byte aligned
 *  other arguments as pkv_store_kvcache
 *
 * Host checks: as pkv_store_kvcache, plus head_dim a multiple of 16 with
 * head_dim / 16 a power of two (16 .. 512), rope_style 0 or 1, q and q_out
 * both given or both NULL, max_position >= 1. Device checks: a position
 * outside [0, max_position) sets PKV_DEVERR_BOUNDS and nothing of that token
 * is written (neither q_out nor the cache); slots as in pkv_store_kvcache
 * (slot -1 skips the cache write but q is still rotated).
 */
PKV_API int pkv_store_kvcache_rope(const void *q, void *q_out, const void *k, const void *v, void *k_cache,
                                   void *v_cache, const int32_t *slot_mapping, const int32_t *positions,
                                   const float *cos_sin, int max_position, int rope_style, int num_tokens,
                                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                   int64_t num_blocks, int cache_dtype, float *k_scale, float *v_scale,
                                   int *dev_err, void *stream);

/*
 * Split-K plan of a decode call. A sequence's tokens are cut into partitions
 * of partition_tokens logical tokens; each partition is one thread block per
 * KV head, and a reduce kernel merges the partials (flash-decoding). When
 * partition_tokens == 0 the whole context is one partition, no workspace is
 * used and no reduce kernel runs.
 */
typedef struct {
    int partition_tokens;   /* 0: no split */
    int max_partitions;     /* partitions of the longest allowed context */
    size_t workspace_bytes; /* device scratch the decode needs (0: none) */
} pkv_decode_plan;

/*
 * pkv_plan_decode: the plan pkv_paged_attention_decode will use for these
 * sizes. partition_request: 0 = choose automatically, -1 = never split,
 * > 0 = split into partitions of that many tokens (rounded up to the tile
 * size of the kernel). Returns PKV_ERR_UNSUPPORTED for shapes without a
 * kernel (head_dim not 64 or 128; group size not 1, 2, 4 or 8).
 */
PKV_API int pkv_plan_decode(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int max_context_len, int cache_dtype,
                    int partition_request, pkv_decode_plan *plan);

/*
 * pkv_decode_workspace_bytes: device scratch that is always enough for
 * pkv_paged_attention_decode with partition_request = 0 (automatic split-K)
 * on num_seqs sequences of num_q_heads query heads of head_dim, with
 * contexts of at most max_context_len tokens -- whatever the KV head count,
 * block size and cache type. The problem statement gives only these four
 * sizes ("DeepSeek复刻vLLM反超原版：AI推理新标杆", section "vLLM：大模型推理的加速
 * 引擎与挑战": one query token per sequence against its block table), so the
 * value is a bound over the plans the other arguments can select: an
 * automatic plan never cuts partitions shorter than 1024 tokens, so it uses
 * at most ceil(max_context_len / 1024) partitions of (head_dim + 2) floats per
 * (sequence, query head). Returns 0 when no automatic plan can split
 * (max_context_len <= 1024) and for sizes below 1. pkv_plan_decode gives the
 * exact figure for one shape (and for explicit partition requests).
 */
PKV_API size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len);

/*
 * paged_attention_decode: for each sequence i < num_seqs and query head h,
 *   out[i][h][:] = sum_t softmax_t(scale * q[i][h] . K_t) V_t
 * over the context_lens[i] tokens t of sequence i, where the K/V row of
 * logical token t is slot block_tables[i][t / block_size] * block_size +
 * t % block_size of the pools (KV head h / group). Scores, softmax and the
 * weighted sum accumulate in fp32; out is rounded to bf16.
 *
 *  q                  [num_seqs][num_q_heads][head_dim] bf16, contiguous
 *  block_tables       [num_seqs][max_blocks_per_seq] int32
 *  context_lens       [num_seqs] int32, each in [1, min(max_context_len,
 *                     max_blocks_per_seq * block_size)]
 *  seq_order          optional [num_seqs] int32, a permutation of
 *                     0..num_seqs-1: the order in which sequences are
 *                     scheduled (NULL: 0, 1, 2, ...). Longest first shortens
 *                     the tail of the grid; the result does not depend on
 *                     it. An entry outside [0, num_seqs) sets
 *                     PKV_DEVERR_BOUNDS and is skipped; the out rows of a
 *                     sequence that no valid entry names are then left
 *                     unwritten (the split-K merge follows the same
 *                     order, so it never reads partials of another call).
 *  max_context_len    host-known bound on context_lens (sizes split-K)
 *  partition_request  as in pkv_plan_decode
 *  workspace          device scratch of at least plan.workspace_bytes,
 *                     256-byte aligned (may be NULL when that is 0);
 *                     contents need not be initialised and are clobbered
 *  out                [num_seqs][num_q_heads][head_dim] bf16
 *
 * Host checks: pointers non-null and 16-byte aligned (q, caches, out,
 * workspace), block_size a power of two in [8, 1024], head_dim and group
 * supported, max_context_len >= 1 and <= max_blocks_per_seq * block_size,
 * workspace large enough (PKV_ERR_WORKSPACE otherwise). Device checks: a
 * length outside [1, max_context_len] or a block id outside
 * [0, num_blocks) sets PKV_DEVERR_BOUNDS and that sequence's KV-head rows of
 * out are written as zeros.
 */
PKV_API int pkv_paged_attention_decode(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, const int32_t *seq_order,
                               int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int64_t num_blocks, float scale, int cache_dtype,
                               const float *k_scale, const float *v_scale,
                               int max_context_len, int partition_request, void *workspace,
                               size_t workspace_bytes, void *out, int *dev_err, void *stream);

/*
 * pkv_paged_attention_decode_shared_prefix: the same decode for a batch
 * whose sequences share cached prefixes, computed as a cascade. Blocks that
 * several requests share (prefix caching: "Nano-vLLM：轻量高效的大模型推理框架",
 * section 三.2(1) 前缀缓存; sharing within and across requests:
 * "DeepSeek复刻vLLM反超原版：AI推理新标杆", section "vLLM：大模型推理的加速引擎
 * 与挑战") are then read and multiplied once per group of members instead of
 * once per sequence: a prefix kernel attends each group's shared tokens for
 * many query rows at a time (bf16: the tcgen05 kernel, 256 rows of (member,
 * query head) per CTA, run beside the suffix decode on the library's side
 * stream; E4M3: up to 32 rows per block on the warp-level MMA), the decode
 * kernel attends each sequence's own tokens, and the split-K merge combines
 * the two (out is the same attention as pkv_paged_attention_decode, to
 * rounding).
 *
 *  cu_group_seqs        [num_groups + 1] int32, device: group j is
 *                       sequences cu_group_seqs[j] .. cu_group_seqs[j+1] - 1
 *                       (consecutive in the batch; the groups cover it in
 *                       order, single sequences are groups of one)
 *  group_prefix_tokens  [num_groups] int32, device: P_j, the number of
 *                       leading tokens every member of group j shares: a
 *                       multiple of block_size, at most each member's
 *                       context length, and the members' block-table
 *                       entries 0 .. P_j / block_size - 1 are the same
 *                       physical blocks (0: nothing shared)
 *  max_group_seqs       host-known bound on the group sizes (sizes the grid)
 *  workspace            at least pkv_plan_decode_shared_prefix's
 *                       workspace_bytes (the prefix partial is one more
 *                       split-K slot per (sequence, query head)), 256-byte
 *                       aligned
 *  seq_order            optional (NULL: natural order), as for
 *                       pkv_paged_attention_decode: the order in which the
 *                       suffix decode and the merge visit the sequences
 *                       (the groups keep their batch positions)
 *  other arguments as pkv_paged_attention_decode
 *
 * Device checks: a P_j that is not a multiple of block_size or exceeds a
 * member's context, a member whose shared block ids differ from the first
 * member's, a group larger than max_group_seqs, or groups that do not lie
 * inside the batch set
 * PKV_DEVERR_BOUNDS and the affected sequences' out rows are written as
 * zeros (where they can be located). head_dim 64, or num_groups == 0,
 * run the ordinary decode (same result).
 */
PKV_API int pkv_plan_decode_shared_prefix(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_context_len, int cache_dtype,
                                          int partition_request, pkv_decode_plan *plan);
PKV_API int pkv_paged_attention_decode_shared_prefix(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, const int32_t *seq_order, int num_seqs, int num_q_heads, int num_kv_heads,
    int head_dim, int block_size,
    int64_t num_blocks, float scale, int cache_dtype, const float *k_scale, const float *v_scale,
    int max_context_len, const int32_t *cu_group_seqs, const int32_t *group_prefix_tokens, int num_groups,
    int max_group_seqs, int partition_request, void *workspace, size_t workspace_bytes, void *out, int *dev_err,
    void *stream);

/*
 * pkv_paged_attention_decode_static_scratch: pkv_paged_attention_decode for
 * callers that cannot allocate device memory -- for example an engine that
 * reserves all device memory for its KV pool at start-up and forbids later
 * allocations, or a plugin that cannot reach its host framework's device
 * allocator through a C ABI. (The pages have no counterpart: it only changes
 * where the split-K scratch lives.)
 *
 * Same arguments and result as pkv_paged_attention_decode, without
 * workspace / workspace_bytes: the split-K partials go to a library-owned
 * device array of PKV_STATIC_SCRATCH_BYTES (32 MiB), which every GPU that
 * loads the library holds until the process exits. Nothing is allocated:
 * no cudaMalloc, cudaFree or allocating library routine is called.
 *
 * The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. A plan that needs more scratch than the array
 * holds returns PKV_ERR_WORKSPACE and launches nothing. All calls share the
 * one array and it keeps the last call's contents (the kernels need no
 * zeroed scratch): calls that overlap on the GPU -- on different streams, or
 * from different threads -- race on it and must be serialised by the caller.
 */
#define PKV_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
PKV_API int pkv_paged_attention_decode_static_scratch(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
    int max_blocks_per_seq, const int32_t *context_lens, const int32_t *seq_order,
    int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
    int cache_dtype, const float *k_scale, const float *v_scale, int max_context_len,
    int partition_request, void *out, int *dev_err, void *stream);

/*
 * pkv_paged_attention_prefill: chunked prefill over the paged cache
 * ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section 核心技术改进 2
 * "Chunked Prefill": a long prompt's prefill runs in chunks scheduled
 * together with decode requests). Sequence i brings a chunk of
 * c_i = cu_q_lens[i + 1] - cu_q_lens[i] query tokens (rows cu_q_lens[i] ..
 * cu_q_lens[i + 1] - 1 of q) whose K/V pkv_store_kvcache has already written
 * as the last c_i of its context_lens[i] positions. Token j of the chunk sits
 * at position p = context_lens[i] - c_i + j and attends causally:
 *   out[row][h][:] = sum_{t <= p} softmax_t(scale * q[row][h] . K_t) V_t
 * (KV head h / group). A chunk of one token is a decode step, so one call
 * can serve a batch mixing prefill chunks and decode requests; c_i = 0 is
 * allowed (no rows). QK^T and PV run on the tensor cores with fp32
 * accumulation. Operands: bf16 for a bf16 cache. For an E4M3 cache the codes
 * are widened exactly: chunks of more than 128 / group tokens use f16 for QK^T
 * (q scaled per row by a power of two into f16 range, exact for bf16 q) and,
 * with one scale per KV head, f16 for PV too; with per-token scales PV runs in
 * bf16; shorter chunks use bf16. With per-token scales, scores are scaled
 * by their token's K scale, and V is dequantised to bf16 before P V (each
 * code times its token's V scale in fp32, rounded to bf16). The softmax
 * weights are rounded to the PV operand type and the normaliser sums those
 * rounded weights. out is rounded to bf16.
 *
 *  q             [total_q][num_q_heads][head_dim] bf16, contiguous
 *  block_tables  [num_seqs][max_blocks_per_seq] int32
 *  cu_q_lens     [num_seqs + 1] int32: 0, then running sums of the c_i
 *  context_lens  [num_seqs] int32, c_i <= context_lens[i] <=
 *                max_blocks_per_seq * block_size
 *  max_q_len     host-known bound on every c_i (sizes the grid)
 *  workspace     optional, E4M3 cache only (ignored for bf16; may be NULL):
 *                at least pkv_prefill_workspace_bytes(...) bytes, 16-byte
 *                aligned, owned by the caller, contents not kept between
 *                calls (calls that may run at the same time, on different
 *                streams, need separate workspaces). With it, the codes of
 *                the sequences whose chunks are
 *                longer than 128 / G tokens are widened once per call into
 *                dense 16-bit rows there (K f16; V f16, or with per-token
 *                scales V dequantised to bf16 and the K scales as fp32 rows;
 *                zeros past the context), and the warp-specialised kernel copies
 *                its tiles from there instead of widening the codes in every
 *                CTA: the same operand values, so the same result for finite
 *                cache contents. NULL: the CTAs widen the codes themselves.
 *                A non-NULL workspace smaller than a nonzero bound returns
 *                PKV_ERR_WORKSPACE and launches nothing.
 *  out           [total_q][num_q_heads][head_dim] bf16
 *
 * Host checks: pointers non-null, q / caches / out 16-byte aligned,
 * head_dim 64 or 128, group 1, 2, 4 or 8, block_size a power of two in
 * [8, 1024], scale positive and finite, max_q_len >= 1 (when total_q > 0). Device checks: cu_q_lens not
 * starting at or above 0, decreasing or past total_q, a chunk longer than
 * its context or than max_q_len, a context beyond the table row, or a block
 * id outside [0, num_blocks) set PKV_DEVERR_BOUNDS; the sequence's rows are
 * written as zeros where they can be located. The library allocates nothing.
 *
 * Routing: one-token chunks run in the decode kernel, chunks of up to 128 / G
 * tokens in a one-tile kernel, longer ones in a warp-specialised kernel.
 * When the batch has chunks longer than one token (max_q_len > 1), the
 * one-token chunks run on the library's low-priority stream of this device,
 * beside the chunk kernels on the given stream (forked from and joined back
 * into it with events), so that their many small blocks use the SMs the long
 * chunks' few blocks leave idle.
 */
PKV_API int pkv_paged_attention_prefill(const void *q, const void *k_cache, const void *v_cache,
                                        const int32_t *block_tables, int max_blocks_per_seq,
                                        const int32_t *cu_q_lens, const int32_t *context_lens, int num_seqs,
                                        int total_q, int num_q_heads, int num_kv_heads, int head_dim,
                                        int block_size, int64_t num_blocks, float scale, int cache_dtype,
                                        const float *k_scale, const float *v_scale, int max_q_len,
                                        void *workspace, size_t workspace_bytes, void *out, int *dev_err,
                                        void *stream);

/*
 * pkv_prefill_workspace_bytes: size of the optional widening workspace of
 * pkv_paged_attention_prefill for an E4M3 cache:
 *   num_seqs * num_kv_heads * R * (4 * head_dim + (per-token scales ? 4 : 0))
 * with R = max_blocks_per_seq * block_size rounded up to a multiple of 128
 * (the table's capacity: one run of R staging rows per sequence and KV
 * head). 0 for a bf16 cache, for arguments below 1, and when the staging
 * would have 2^31 rows or more (the call then widens in its CTAs).
 */
PKV_API size_t pkv_prefill_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                                           int block_size, int cache_dtype);

/*
 * pkv_fused_add_rmsnorm: the residual add and RMSNorm around attention in
 * one kernel ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section
 * 核心技术改进 1 "CUDA融合内核：Add+RMSNorm"). For each row t < num_tokens:
 *   h = x[t] + residual[t]            (fp32; residual[t] <- bf16(h), RNE)
 *   out[t] = weight * h / sqrt(mean(h^2) + eps)   (fp32, rounded to bf16)
 * With residual == NULL, h = x[t] and nothing else is written.
 *
 *  x, out     [num_tokens][hidden] bf16; out may be x (in place)
 *  residual   [num_tokens][hidden] bf16, read and overwritten (or NULL)
 *  weight     [hidden] bf16
 *
 * The sum of squares is accumulated in fp32, so rows with elements beyond
 * about 1e19 in magnitude (far outside any activation range) overflow it.
 *
 * Host checks: non-null x / weight / out, 16-byte aligned pointers, hidden a
 * multiple of 8 in [8, 16384] (above: PKV_ERR_UNSUPPORTED), num_tokens >= 0,
 * eps >= 0 and finite. No
 * device-side checks are needed (every index is derived from the sizes).
 */
PKV_API int pkv_fused_add_rmsnorm(const void *x, void *residual, const void *weight, void *out, int num_tokens,
                                  int hidden, float eps, void *stream);

/* Human-readable name of a pkv_status value (static storage). */
PKV_API const char *pkv_status_string(int status);

/*
 * pkv_read_device_error: synchronise the stream, read *dev_err and map it to
 * a status (PKV_OK, PKV_ERR_DEVICE_BOUNDS, PKV_ERR_DEVICE_TIMEOUT; the
 * timeout bit wins). Does not clear the word.
 */
PKV_API int pkv_read_device_error(const int *dev_err, void *stream);

/* Library version, e.g. 0x000100 for 0.1.0. */
PKV_API int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
