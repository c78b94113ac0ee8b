// decode.cuh -- paged decode attention on the CUDA cores (sm_100a): the
// kernel for head_dim 64 (head_dim 128 runs on the warp-level MMA,
// decode_mma.cuh), the split-K merge both use, and the parameters they share.
//
// One thread block per (sequence, KV head, partition). It serves all G query
// heads that share the KV head, so every K/V byte of the partition is read
// from HBM exactly once. The pages give the problem (a block table maps each
// sequence's logical blocks to physical blocks of a shared pool: "DeepSeek复刻
// vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战") and state that decode
// is bound by KV-cache read bandwidth ("nano-vllm-lite", section 核心技术改进 2);
// attention is computed flash-style, without materialising the score row
// ("Nano-vLLM：轻量高效的大模型推理框架", section 三.3 注意力层).
//
// Block structure: 4 warps, each running its own pipeline over its own rows.
//  * Tiles: a partition is walked in tiles of kTile logical tokens; warp w
//    owns rows [w*kRows, (w+1)*kRows) of every tile. Lane 0 of the warp cuts
//    its rows at block boundaries into runs that are contiguous in the HND
//    pool and bulk-copies each run of K and of V (non-tensor TMA,
//    cp.async.bulk, no multicast) into the warp's slice of a kStages-deep K
//    ring and V ring in shared memory, completing on the warp's own "full"
//    mbarriers. Only valid tokens are copied; the rings are zeroed once so
//    that rows past the end of a partial tile are finite and can take part
//    in the arithmetic with weight 0. When the warp is done with a stage it
//    refills it itself: no producer warp, no cross-warp counters.
//  * Lanes: a row is spread over kLPT = head_dim/8 lanes (8 elements each:
//    16-byte loads for bf16, 8-byte for E4M3); a warp covers kTPS rows per
//    step and kSteps steps per tile.
//  * QK: each lane forms its chunk's partial dot for every (step, head) with
//    mixed-precision FMAs (exact 16-bit products, fp32 sums): bf16 x bf16 on
//    the packed cache, or f16 x f16 after the exact E4M3 -> f16x2 conversion
//    with q in f16 (block-scaled by a power of two). A reduce-scatter butterfly
//    over the kLPT lanes of a row then leaves each lane with the full score
//    of one (step, head); each lane holds its values in a lane-permuted order
//    so that no round needs a select.
//  * Softmax: base 2 (the reduced score is multiplied by scale*log2(e), and
//    for E4M3 by the K scale and q's power of two); per head, the tile max over the warp's rows,
//    rescale factor alpha and p = 2^(s - m); p goes through a few bytes of
//    shared memory to the lanes that own the V chunks. The accumulators are
//    rescaled only when some head's max moved.
//  * Software pipeline: iteration j runs QK of tile j, then the shuffle /
//    exponential chain of tile j interleaved with P * V of tile j - 1 in one
//    branch-free block, so the chain's latency hides behind FMAs.
//  * P * V: fp32 accumulators; packed f32x2 FMAs with (p, p) pairs.
//  * Epilogue: merge the warps' (max, sum, accumulators) in shared memory
//    (reusing the rings) and write bf16 output, or, for split-K, the
//    normalised fp32 partial with its (max, sum) for the reduce kernel.
//
// Every wait is bounded (PKV_DEVERR_TIMEOUT), every block id and length is
// checked before a byte is copied (PKV_DEVERR_BOUNDS), and each warp waits
// for its own copies in flight before the block exits.
#pragma once

#include <math_constants.h>

#include "pkv_common.cuh"
#include "pkv_launch.h"

namespace pkv {

struct DecodeParams {
    const __nv_bfloat16 *q;
    const uint8_t *k_cache;
    const uint8_t *v_cache;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens;
    const int32_t *seq_order;  // may be null: natural order
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int log2_block_size;
    long long num_blocks;
    float qk_scale_log2;  // scale * log2(e)
    const float *k_scale;
    const float *v_scale;
    int max_context_len;
    int partition_tokens;  // > 0; >= max_context_len when not split
    int num_partitions;
    float *part_o;
    float *part_ml;
    __nv_bfloat16 *out;
    int *dev_err;
    // Rows of a chunked-prefill call routed here: when set, sequence i is
    // served only if its chunk is one token (cu_q_lens[i + 1] - cu_q_lens[i]
    // == 1), and its q and out row is cu_q_lens[i] (of total_q rows).
    const int32_t *cu_q_lens;
    int total_q;
    // Shared-prefix (cascade) mode, when cu_group_seqs is set: sequences
    // cu_group_seqs[j] .. cu_group_seqs[j + 1] - 1 form group j, whose first
    // group_prefix[j] tokens are the same cached blocks for every member. The
    // prefix kernel writes each member's prefix partial to slot 0; the decode
    // kernel attends the rest of each sequence, partition p to slot p + 1.
    const int32_t *cu_group_seqs;
    const int32_t *group_prefix;
    int num_groups;
    int max_group_seqs;  // host bound: sizes the prefix kernel's grid
    int grid_partitions;  // partitions per (sequence, KV head) in the decode grid
};

// Group of sequence seq in shared-prefix mode (largest j with
// cu_group_seqs[j] <= seq; -1 when seq precedes group 0).
__device__ __forceinline__ int group_of(const DecodeParams &p, int seq) {
    int lo = 0, hi = p.num_groups - 1, ans = -1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.cu_group_seqs + mid) <= seq) {
            ans = mid;
            lo = mid + 1;
        } else {
            hi = mid - 1;
        }
    }
    return ans;
}

// Prefix length of sequence seq in shared-prefix mode, or -1 when it is not
// usable (negative, not a whole number of blocks, past the context, the
// sequence in no group, or a group larger than the host's bound
// max_group_seqs, whose members past the bound no prefix kernel covers).
__device__ __forceinline__ int prefix_of(const DecodeParams &p, int seq, int ctx) {
    const int j = group_of(p, seq);
    if (j < 0) return -1;
    const int g1 = __ldg(p.cu_group_seqs + j + 1);
    if (seq >= g1 || g1 - __ldg(p.cu_group_seqs + j) > p.max_group_seqs) return -1;
    const int P = __ldg(p.group_prefix + j);
    if (P < 0 || P > ctx || (P & (p.block_size - 1)) != 0) return -1;
    return P;
}

// Block ids of a partition staged in shared memory; ids beyond are read
// from the table row in global memory (every id is checked up front).
constexpr int kMaxIdsPerPartition = 256;

// Tuning constants (compile-time; the defaults are the measured choice).
#ifndef PKV_DECODE_CONSUMER_WARPS
#define PKV_DECODE_CONSUMER_WARPS 4
#endif
#ifndef PKV_DECODE_MAX_STEPS
#define PKV_DECODE_MAX_STEPS 4
#endif
#ifndef PKV_DECODE_RING_BYTES
#define PKV_DECODE_RING_BYTES 49152
#endif

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cclamp(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

template <int D, int G, bool FP8>
struct DecodeTraits {
    static constexpr int kNCW = PKV_DECODE_CONSUMER_WARPS;
    static constexpr int kESize = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kESize;
    static constexpr int kLPT = D / 8;                    // lanes per row
    static constexpr int kTPS = 32 / kLPT;                // rows per warp step
    static constexpr int kSteps = cmin(PKV_DECODE_MAX_STEPS, kLPT / G);  // steps per tile
    static constexpr int kNV = kSteps * G;                // scores per lane group (<= kLPT)
    static constexpr int kShiftV = ilog2(kLPT) - ilog2(kNV);
    static constexpr int kRows = kSteps * kTPS;           // rows per warp per tile
    static constexpr int kTile = kRows * kNCW;            // tokens per tile
    static constexpr int kTileBytes = kTile * kRowBytes;  // one tile of K (or of V)
    static constexpr int kStages = cclamp(PKV_DECODE_RING_BYTES / (2 * kTileBytes), 2, 8);
    static constexpr int kThreads = kNCW * 32;
    // per warp, two tiles of p[row][head], stored as (p, p) pairs so that
    // P * V runs on packed f32x2 FMAs without rearranging registers
    static constexpr int kPBufFloats = 2 * kRows * G * 2;
    // shared memory layout (bytes); the merge area reuses the rings
    static constexpr int kRingBytes = kStages * kTileBytes;  // one ring (K or V)
    static constexpr int kOffV = kRingBytes;
    static constexpr int kOffBars = 2 * kRingBytes;          // full_k[NCW][S], full_v[NCW][S]
    static constexpr int kOffCnt = kOffBars + 2 * kNCW * kStages * 8;  // issued K, V tiles per warp
    static constexpr int kOffIds = kOffCnt + 2 * kNCW * 4;
    static constexpr int kOffPBuf = (kOffIds + kMaxIdsPerPartition * 4 + 15) / 16 * 16;
    static constexpr int kSmemBytes = kOffPBuf + kNCW * kPBufFloats * 4;
    static constexpr int kMergeFloats = kNCW * G * D + 3 * kNCW * G;
    static_assert((32 % kLPT) == 0 && kLPT >= 2, "row mapping");
    static_assert(kSteps >= 1 && kNV <= kLPT, "one score per lane after the reduction");
    static_assert(kTileBytes % 128 == 0, "stage alignment");
    static_assert(kMergeFloats * 4 <= 2 * kRingBytes, "merge area must fit in the rings");
};

// 8 cached elements (bf16: 16 bytes, E4M3: 8 bytes) -> 8 floats (exact).
template <bool FP8>
__device__ __forceinline__ void load8(const uint8_t *p, float (&x)[8]) {
    if constexpr (FP8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        const float2 a = e4m3x2_to_float2((uint16_t)(w.x & 0xffffu));
        const float2 b = e4m3x2_to_float2((uint16_t)(w.x >> 16));
        const float2 c = e4m3x2_to_float2((uint16_t)(w.y & 0xffffu));
        const float2 d = e4m3x2_to_float2((uint16_t)(w.y >> 16));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
        x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
    } else {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
        x[4] = bf16lo(w.z); x[5] = bf16hi(w.z); x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
    }
}

// Reduce-scatter of N partial sums over the lanes that differ in bits
// O, O/2, ..., 1 of the lane index. Each lane holds its N values in a
// lane-specific order -- position i holds logical value i ^ v_lane, where
// v_lane is the lane's own bits O.. taken as a number -- so that in every
// round the half a lane keeps is its lower half and the half it sends is its
// upper half: no selects. After the scatter rounds x[0] is the full sum of
// value v_lane; rounds past one value are plain butterflies.
template <int N, int O>
struct ReduceScatter {
    static __device__ __forceinline__ void run(float *x) {
        if constexpr (O >= 1) {
            if constexpr (N > 1) {
#pragma unroll
                for (int i = 0; i < N / 2; ++i) x[i] += __shfl_xor_sync(0xffffffffu, x[i + N / 2], O);
                ReduceScatter<N / 2, O / 2>::run(x);
            } else {
                x[0] += __shfl_xor_sync(0xffffffffu, x[0], O);
                ReduceScatter<1, O / 2>::run(x);
            }
        }
    }
};

// TS: E4M3 cache with one scale per (token, KV head) in scale pools shaped
// like the cache without head_dim (p.k_scale / p.v_scale); each lane loads
// the scales of the row its score belongs to, one tile ahead of use.
template <int D, int G, bool FP8, int MIN_BLOCKS, bool TS = false>
__global__ void __launch_bounds__(DecodeTraits<D, G, FP8>::kThreads, MIN_BLOCKS)
    paged_decode_kernel(const DecodeParams p) {
    using T = DecodeTraits<D, G, FP8>;
    constexpr int NCW = T::kNCW;
    constexpr int TILE = T::kTile;
    constexpr int STAGES = T::kStages;
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t *ids = reinterpret_cast<int32_t *>(smem + T::kOffIds);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // which (sequence, KV head, partition)
    const int part = blockIdx.x % p.num_partitions;
    const int rest = blockIdx.x / p.num_partitions;
    const int kvh = rest % p.num_kv_heads;
    const int seq_slot = rest / p.num_kv_heads;
    const int seq = p.seq_order ? __ldg(p.seq_order + seq_slot) : seq_slot;
    if (seq < 0 || seq >= p.num_seqs) {  // not a permutation entry: nothing to write to
        if (threadIdx.x == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
        return;
    }

    long long row = seq;  // q / out row
    if (p.cu_q_lens) {
        const int q0 = __ldg(p.cu_q_lens + seq), q1 = __ldg(p.cu_q_lens + seq + 1);
        if (q0 < 0 || q1 < q0 || q1 > p.total_q || q1 - q0 != 1) return;  // the prefill kernels' sequence
        row = q0;
    }
    const int ctx = __ldg(p.context_lens + seq);
    const int table_cap = p.max_blocks_per_seq << p.log2_block_size;
    const bool bad_len = ctx < 1 || ctx > p.max_context_len || ctx > table_cap;
    const int start = part * p.partition_tokens;
    const int end = bad_len ? start : min(start + p.partition_tokens, ctx);
    const int n_parts_seq = bad_len ? 1 : (ctx + p.partition_tokens - 1) / p.partition_tokens;
    const bool single = n_parts_seq == 1;  // this block writes the final output
    if (!bad_len && start >= end) return;  // partition past this sequence's end
    if (bad_len && part != 0) return;

    // Check every block id of this partition and stage the first ones, zero
    // the rings (rows past the end of a partial tile are then finite, so they
    // can take part in the arithmetic with weight 0), set up the barriers.
    const int first_blk = start >> p.log2_block_size;
    const int n_blk = bad_len ? 0 : ((end - 1) >> p.log2_block_size) - first_blk + 1;
    int bad = bad_len;
    const int32_t *table = p.block_tables + (long long)seq * p.max_blocks_per_seq + first_blk;
    for (int i = tid; i < n_blk; i += T::kThreads) {
        const int32_t id = __ldg(table + i);
        if (i < kMaxIdsPerPartition) ids[i] = id;
        bad |= (id < 0 || (long long)id >= p.num_blocks);
    }
    auto blk_id = [&](int i) -> long long { return i < kMaxIdsPerPartition ? ids[i] : __ldg(table + i); };
    for (int i = tid; i < 2 * T::kRingBytes / 16; i += T::kThreads)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();  // the zeros, before bulk copies overwrite them
    // Each warp runs its own pipeline over its own rows of every tile: its
    // barriers, its slice of each stage, its own refills.
    uint64_t *full_k = reinterpret_cast<uint64_t *>(smem + T::kOffBars) + warp * STAGES;
    uint64_t *full_v = full_k + NCW * STAGES;
    int *issued = reinterpret_cast<int *>(smem + T::kOffCnt) + 2 * warp;  // K, V tiles this warp issued
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
        }
        fence_barrier_init();
    }
    bad = __syncthreads_or(bad);

    const int qh0 = kvh * G;  // first query head of this KV head
    if (bad) {
        if (tid == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
        if (single || bad_len) {
            for (int i = tid; i < G * D; i += T::kThreads)
                p.out[(row * p.num_q_heads + qh0) * D + i] = __float2bfloat16_rn(0.f);
        } else if (tid < G) {
            float *ml = p.part_ml + (((long long)seq * p.num_q_heads + qh0 + tid) * p.num_partitions + part) * 2;
            ml[0] = -CUDART_INF_F;
            ml[1] = 0.f;
        }
        return;
    }

    const int n_tiles = (end - start + TILE - 1) / TILE;
    const long long head_stride = (long long)p.block_size * T::kRowBytes;  // bytes of one (block, head) run
    const long long blk_stride = head_stride * p.num_kv_heads;

    // Issue this warp's rows of the K (or V) half of tile j into stage s:
    // logical tokens [start + j*TILE + warp*ROWS, ...), split at block
    // boundaries into contiguous runs of the HND pool, one bulk copy each.
    // The warp's rows start on a multiple of ROWS, so when a block holds at
    // least ROWS tokens they are always one run.
    constexpr int ROWS_W = T::kRows;
    const long long head_off = (long long)kvh * head_stride;
    auto issue = [&](int j, int s, bool is_v) {
        const int a0 = start + j * TILE + warp * ROWS_W;
        const int a1 = min(a0 + ROWS_W, end);
        uint8_t *dst0 = smem + (is_v ? T::kOffV : 0) + s * T::kTileBytes + warp * ROWS_W * T::kRowBytes;
        const uint8_t *src0 = (is_v ? p.v_cache : p.k_cache) + head_off;
        uint64_t *bar = (is_v ? full_v : full_k) + s;
        mbar_arrive_expect_tx(bar, (uint32_t)(max(a1 - a0, 0) * T::kRowBytes));
        if (p.block_size >= ROWS_W) {
            if (a1 > a0) {
                const long long phys = blk_id((a0 >> p.log2_block_size) - first_blk);
                const int off = a0 & (p.block_size - 1);
                bulk_g2s(dst0, src0 + phys * blk_stride + (long long)off * T::kRowBytes,
                         (uint32_t)((a1 - a0) * T::kRowBytes), bar);
            }
        } else {
            for (int a = a0; a < a1;) {
                const int lb = a >> p.log2_block_size;
                const int off = a & (p.block_size - 1);
                const int n = min(p.block_size - off, a1 - a);
                const long long phys = blk_id(lb - first_blk);
                bulk_g2s(dst0 + (a - a0) * T::kRowBytes, src0 + phys * blk_stride + (long long)off * T::kRowBytes,
                         (uint32_t)(n * T::kRowBytes), bar);
                a += n;
            }
        }
    };
    // This warp is done with the K half of tile jk (stage sk) and the V half
    // of tile jv (stage sv): refill those stages with tiles jk + STAGES and
    // jv + STAGES -- lane 0 the K stage, lane 1 the V stage, through one
    // code path. A negative tile index means "nothing to release". Callers
    // __syncwarp() first, so every lane's reads of the stages are done.
    auto release = [&](int jk, int sk, int jv, int sv) {
        if (lane < 2) {
            const bool is_v = lane == 1;
            const int j = is_v ? jv : jk;
            if (j >= 0 && j + STAGES < n_tiles) {
                fence_proxy_async_smem();
                issue(j + STAGES, is_v ? sv : sk, is_v);
                issued[lane] = j + STAGES + 1;
            }
        }
    };
    if (lane < 2) {  // lane 0 primes the K ring, lane 1 the V ring
        const int first = min(STAGES, n_tiles);
        for (int j = 0; j < first; ++j) issue(j, j, lane == 1);
        issued[lane] = first;
    }

    // ------------------------------------------------------------ per lane
    constexpr int LPT = T::kLPT;
    constexpr int TPS = T::kTPS;
    constexpr int STEPS = T::kSteps;
    constexpr int ROWS = T::kRows;
    constexpr int LOG2G = ilog2(G);
    constexpr int HEAD_BITS_END = T::kShiftV + LOG2G;  // lane bits below this: duplicate or head
    const int sub = lane / LPT;    // row within a step
    const int chunk = lane % LPT;  // 8-element chunk of the row
    // The score this lane holds after the reduction: (my_st, my_h), row my_row.
    const int my_v = chunk >> T::kShiftV;
    const int my_h = my_v & (G - 1);
    const int my_st = my_v >> LOG2G;
    const int my_row = my_st * TPS + sub;
    const bool canon = (chunk & ((1 << T::kShiftV) - 1)) == 0;  // first of its duplicates
    float *pbuf = reinterpret_cast<float *>(smem + T::kOffPBuf) + warp * T::kPBufFloats;  // [2][ROWS][G]

    // q in this lane's slot order: slot hs holds head hs ^ my_h (see
    // ReduceScatter). bf16 cache: q stays packed bf16 and QK uses the
    // bf16 x bf16 -> fp32 FMA (exact products, fp32 sums); the scale is applied
    // to the reduced score. E4M3 cache: q in fp32, pre-multiplied by the scale
    // and the K scale.
    uint32_t qw[G][4];
#pragma unroll
    for (int hs = 0; hs < G; ++hs) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(
            p.q + (row * p.num_q_heads + qh0 + (hs ^ my_h)) * D + chunk * 8));
        qw[hs][0] = w.x; qw[hs][1] = w.y; qw[hs][2] = w.z; qw[hs][3] = w.w;
    }
    // Multiplier of the reduced score: scale*log2(e) (and, for E4M3, the K
    // scale and the power of two below).
    float score_scale = p.qk_scale_log2;
    if constexpr (FP8) {
        // QK runs as f32 += f16 x f16 FMAs on the f16 pairs the E4M3 codes
        // convert to exactly. q becomes f16 after a power-of-two rescale that
        // puts this block's largest |q| just under 2^15, so every element keeps
        // its bf16 value exactly (elements below 2^-29 of the largest one are
        // rounded to f16's subnormal grid); the power of two is undone on the
        // score.
        float mx = 0.f;
#pragma unroll
        for (int hs = 0; hs < G; ++hs)
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fmaxf(fabsf(bf16lo(qw[hs][i])), fabsf(bf16hi(qw[hs][i]))));
#pragma unroll
        for (int o = 1; o < LPT; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        frexpf(mx, &e);  // mx < 2^e (e = 0 for mx = 0)
        const int k = 15 - e;
#pragma unroll
        for (int hs = 0; hs < G; ++hs)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __half2 h = __floats2half2_rn(ldexpf(bf16lo(qw[hs][i]), k), ldexpf(bf16hi(qw[hs][i]), k));
                qw[hs][i] = *reinterpret_cast<const uint32_t *>(&h);
            }
        score_scale = ldexpf(TS ? p.qk_scale_log2 : p.qk_scale_log2 * __ldg(p.k_scale + kvh), -k);
    }

    float acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = 0.f;
    float m = -CUDART_INF_F;  // running max of head my_h
    float l = 0.f;            // running sum of this lane's rows of head my_h

    const int row0 = warp * ROWS;
    const int lane_off = row0 * T::kRowBytes + chunk * 8 * T::kESize;

    // QK of the tile in K stage sk: this lane's partial dots in its (step, head) order.
    auto qk = [&](int sk, float (&sc)[T::kNV]) {
        const uint8_t *ks = smem + sk * T::kTileBytes + lane_off;
#pragma unroll
        for (int ps = 0; ps < STEPS; ++ps) {
            const uint8_t *row = ks + ((ps ^ my_st) * TPS + sub) * T::kRowBytes;
            if constexpr (FP8) {
                const uint2 w = *reinterpret_cast<const uint2 *>(row);
                const uint32_t kw[4] = {e4m3x2_to_f16x2((uint16_t)(w.x & 0xffffu)),
                                        e4m3x2_to_f16x2((uint16_t)(w.x >> 16)),
                                        e4m3x2_to_f16x2((uint16_t)(w.y & 0xffffu)),
                                        e4m3x2_to_f16x2((uint16_t)(w.y >> 16))};
#pragma unroll
                for (int hs = 0; hs < G; ++hs) {
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) a = fma_f16x2_acc(qw[hs][i], kw[i], a);
                    sc[ps * G + hs] = a;
                }
            } else {
                const uint4 kw4 = *reinterpret_cast<const uint4 *>(row);
                const uint32_t kw[4] = {kw4.x, kw4.y, kw4.z, kw4.w};
#pragma unroll
                for (int hs = 0; hs < G; ++hs) {
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) a = fma_bf16x2_acc(qw[hs][i], kw[i], a);
                    sc[ps * G + hs] = a;
                }
            }
        }
    };
    // Per-token scales of this lane's row of tile j (TS only): K scale
    // multiplies the score, V scale the weight that P * V uses (l sums the
    // unscaled weights). Rows past the end get 0 (their weight is 0 anyway).
    // The loop loads tile j + 1's scales while it works on tile j.
    auto tok_scales = [&](int j, float &ks, float &vs) {
        ks = 0.f;
        vs = 0.f;
        if constexpr (TS) {
            const int a = start + j * TILE + row0 + my_row;
            if (a < end) {
                const long long phys = blk_id((a >> p.log2_block_size) - first_blk);
                const long long idx = (phys * p.num_kv_heads + kvh) * p.block_size + (a & (p.block_size - 1));
                ks = __ldg(p.k_scale + idx);
                vs = __ldg(p.v_scale + idx);
            }
        }
    };
    // Scores of tile j -> p (to this warp's p buffer) and the rescale factor
    // of head my_h; returns whether any head of the warp changed its max.
    auto softmax = [&](int j, float (&sc)[T::kNV], float &alpha, float ks, float vs) {
        ReduceScatter<T::kNV, LPT / 2>::run(sc);
        sc[0] *= TS ? score_scale * ks : score_scale;
        const int n_valid = min(TILE, end - (start + j * TILE));
        const float sv = my_row < n_valid - row0 ? sc[0] : -CUDART_INF_F;
        float tmax = sv;
#pragma unroll
        for (int o = 1 << HEAD_BITS_END; o < 32; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float m_new = fmaxf(m, tmax);
        const float mref = m_new == -CUDART_INF_F ? 0.f : m_new;  // no row seen yet: keep everything at 0
        alpha = fast_exp2(m - mref);
        const float pr = fast_exp2(sv - mref);
        l = fmaf(l, alpha, pr);
        m = m_new;
        const float pw = TS ? pr * vs : pr;
        if (canon) reinterpret_cast<float2 *>(pbuf)[(j & 1) * ROWS * G + my_row * G + my_h] = make_float2(pw, pw);
    };
    // P * V of the tile in V stage sv (p buffer half pj) into the
    // accumulators; rows past the end have p = 0.
    auto pv = [&](int sv, int pj) {
        const uint8_t *vs = smem + T::kOffV + sv * T::kTileBytes + lane_off;
#pragma unroll
        for (int st = 0; st < STEPS; ++st) {
            const int r = st * TPS + sub;
            float vf[8];
            load8<FP8>(vs + r * T::kRowBytes, vf);
            // packed f32x2 FMAs: (p, p) x (v_2i, v_2i+1) + (acc_2i, acc_2i+1)
            const float2 *pb = reinterpret_cast<const float2 *>(pbuf) + pj * ROWS * G;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float2 pp = pb[r * G + h];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 a = __ffma2_rn(pp, make_float2(vf[2 * i], vf[2 * i + 1]),
                                                make_float2(acc[h][2 * i], acc[h][2 * i + 1]));
                    acc[h][2 * i] = a.x;
                    acc[h][2 * i + 1] = a.y;
                }
            }
        }
    };
    // acc[h] *= alpha of head h (held by the lanes with my_h == h), only when
    // some head's max moved.
    auto rescale = [&](float alpha) {
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float a = __shfl_sync(0xffffffffu, alpha, h << T::kShiftV);  // lane: chunk = h, step 0, row 0
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[h][i] *= a;
            }
        }
    };

    // Software pipeline: iteration j runs QK of tile j, then the shuffle /
    // exponential chain of tile j interleaved with P * V of tile j - 1.
    // (sk, rk) and (sv, rv): stage and round of K tile j and V tile j - 1.
    bool ok = true;
    {
        float sc[T::kNV];
        float alpha;
        float ks, vs;      // this lane's row scales (TS) for the tile being scored
        float ks_n, vs_n;  // ... and for the next tile, loaded one tile ahead
        int sk = 0, rk = 0, sv = 0, rv = 0;
        if (!mbar_wait(&full_k[0], 0)) ok = false;
        if (ok) {
            tok_scales(0, ks, vs);
            tok_scales(1, ks_n, vs_n);
            qk(0, sc);
            __syncwarp();
            release(0, 0, -1, 0);
            softmax(0, sc, alpha, ks, vs);  // acc is still zero: nothing to rescale
            __syncwarp();
            if (++sk == STAGES) { sk = 0; ++rk; }
        }
        for (int j = 1; ok && j < n_tiles; ++j) {
            if (!mbar_wait(&full_k[sk], rk & 1) || !mbar_wait(&full_v[sv], rv & 1)) {
                ok = false;
                break;
            }
            ks = ks_n;
            vs = vs_n;
            tok_scales(j + 1, ks_n, vs_n);
            qk(sk, sc);
            softmax(j, sc, alpha, ks, vs);
            pv(sv, (j - 1) & 1);
            __syncwarp();
            release(j, sk, j - 1, sv);
            rescale(alpha);
            if (++sk == STAGES) { sk = 0; ++rk; }
            if (++sv == STAGES) { sv = 0; ++rv; }
        }
        if (ok && mbar_wait(&full_v[sv], rv & 1)) {
            pv(sv, (n_tiles - 1) & 1);
            __syncwarp();
            release(-1, 0, n_tiles - 1, sv);
        } else {
            ok = false;
        }
    }
    if (!ok) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);

    // ------------------------------------------------------------- epilogue
    // l: sum over the lanes holding the same head (step and row bits).
#pragma unroll
    for (int o = 1 << HEAD_BITS_END; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    // accumulators: sum over the rows of a step (lanes with the same chunk).
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[h][i] += __shfl_xor_sync(0xffffffffu, acc[h][i], o);
    }
    // Every warp is past the loop: no stage is read any more. Wait for any
    // copy still in flight (only after a timeout), then reuse the rings.
    if (lane == 0) {  // copies of this warp still in flight (only after a timeout)
        for (int h = 0; h < 2; ++h) {
            uint64_t *bars = h ? full_v : full_k;
            for (int j = max(0, issued[h] - STAGES); j < issued[h]; ++j)
                if (!mbar_wait(&bars[j % STAGES], (j / STAGES) & 1)) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
        }
    }
    __syncthreads();
    float *merge_acc = reinterpret_cast<float *>(smem);  // [NCW][G][D]
    float *merge_m = merge_acc + NCW * G * D;            // [NCW][G]
    float *merge_l = merge_m + NCW * G;                  // [NCW][G]
    float *merge_w = merge_l + NCW * G;                  // [NCW][G]
    if (sub == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < 8; i += 4)
                *reinterpret_cast<float4 *>(merge_acc + (warp * G + h) * D + chunk * 8 + i) =
                    make_float4(acc[h][i], acc[h][i + 1], acc[h][i + 2], acc[h][i + 3]);
        if (canon && my_st == 0) {
            merge_m[warp * G + my_h] = m;
            merge_l[warp * G + my_h] = l;
        }
    }
    __syncthreads();
    if (tid < G) {
        const int h = tid;
        float M = -CUDART_INF_F;
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, merge_m[w * G + h]);
        float L = 0.f;
        for (int w = 0; w < NCW; ++w) {
            // 0 for a warp that saw no token (its m is -inf, its l and acc 0)
            const float e = merge_m[w * G + h] == -CUDART_INF_F ? 0.f : exp2f(merge_m[w * G + h] - M);
            merge_w[w * G + h] = e;
            L += merge_l[w * G + h] * e;
        }
        float post = 1.f / L;
        if constexpr (FP8 && !TS) post *= __ldg(p.v_scale + kvh);
        for (int w = 0; w < NCW; ++w) merge_w[w * G + h] *= post;
        if (!single) {
            float *ml = p.part_ml + (((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + part) * 2;
            ml[0] = M;
            ml[1] = L;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += T::kThreads) {
        const int h = idx / D;
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) o = fmaf(merge_acc[(w * G + h) * D + (idx % D)], merge_w[w * G + h], o);
        if (single) {
            p.out[(row * p.num_q_heads + qh0) * D + idx] = __float2bfloat16_rn(o);
        } else {
            p.part_o[(((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + part) * D + (idx % D)] = o;
        }
    }
}

// Merge the split-K partials of one (sequence, query head): weights
// l_p * 2^(m_p - M) over the sequence's partitions, in partition order. One
// warp per (sequence, query head), four per block: the lanes load the
// partitions' (max, sum) pairs together and reduce them with shuffles, then
// each lane accumulates D / 32 dims over the partitions. The grid visits
// sequences through seq_order like the decode grid, so it merges only
// partials this call's decode blocks wrote; a sequence that no valid entry
// names is left alone by both.
constexpr int kReduceWarps = 4;

template <int D>
__global__ void __launch_bounds__(32 * kReduceWarps) paged_decode_reduce_kernel(const DecodeParams p) {
    constexpr int DPL = D / 32;  // dims per lane
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kReduceWarps + (threadIdx.x >> 5);
    if (row >= (long long)p.num_seqs * p.num_q_heads) return;
    const int qh = (int)(row % p.num_q_heads);
    const int seq_slot = (int)(row / p.num_q_heads);
    const int seq = p.seq_order ? __ldg(p.seq_order + seq_slot) : seq_slot;
    if (seq < 0 || seq >= p.num_seqs) return;  // the decode grid reported it
    // the partials of slots 0 and 1 (every merged row has at least two slots),
    // loaded before the length and the group are known
    const long long base0 = ((long long)seq * p.num_q_heads + qh) * p.num_partitions;
    float2 spec_ml[2];
    float spec_o[2][DPL];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        spec_ml[i] = *reinterpret_cast<const float2 *>(p.part_ml + (base0 + i) * 2);
        const float *po = p.part_o + (base0 + i) * D + lane * DPL;
        if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(po);
            spec_o[i][0] = v.x;
            spec_o[i][1] = v.y;
            spec_o[i][2] = v.z;
            spec_o[i][3] = v.w;
        } else {
#pragma unroll
            for (int k = 0; k < DPL; ++k) spec_o[i][k] = po[k];
        }
    }
    const int ctx = __ldg(p.context_lens + seq);
    const int table_cap = p.max_blocks_per_seq << p.log2_block_size;
    const bool bad_len = ctx < 1 || ctx > p.max_context_len || ctx > table_cap;
    // partial slots first .. first + n - 1 of this sequence
    int first = 0, n = 0;
    bool bad = false;
    if (p.cu_group_seqs) {  // slot 0: the shared prefix (when there is one), then the suffix partitions
        const int P = bad_len ? -1 : prefix_of(p, seq, ctx);
        bad = P < 0;
        const int n_suf = P >= 0 ? (ctx - P + p.partition_tokens - 1) / p.partition_tokens : 0;
        first = P == 0 ? 1 : 0;
        n = (P != 0) + n_suf;
    } else {
        if (bad_len) return;  // decode wrote zeros
        n = (ctx + p.partition_tokens - 1) / p.partition_tokens;
        if (n <= 1) return;  // decode wrote the output itself
    }
    const long long base = ((long long)seq * p.num_q_heads + qh) * p.num_partitions + first;
    float acc[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
    // Rows of at most two partials in slots 0 and 1 (a shared prefix and a
    // short suffix, or a split in two) use the loads issued above, before the
    // length and the group were known; the arithmetic is the general path's,
    // operation for operation.
    if (first + n <= 2 && !bad) {
        // slot `first` (0, or 1 when there is no prefix), then slot 1 when n == 2;
        // selects with constant indices keep the loaded values in registers
        const float2 ml0 = first ? spec_ml[1] : spec_ml[0];
        const float2 mla = lane == 0 ? ml0 : (lane == 1 && n == 2 ? spec_ml[1] : make_float2(-CUDART_INF_F, 1.f));
        float M = lane < n ? mla.x : -CUDART_INF_F;
        bool empty = lane < n && !(mla.y > 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        if (!__any_sync(0xffffffffu, empty)) {
            float L = lane < n ? mla.y * exp2f(mla.x - M) : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            const float inv = 1.f / L;
            const float w0 = ml0.y * exp2f(ml0.x - M) * inv;
#pragma unroll
            for (int k = 0; k < DPL; ++k) acc[k] = fmaf(first ? spec_o[1][k] : spec_o[0][k], w0, acc[k]);
            if (n == 2) {
                const float w1 = spec_ml[1].y * exp2f(spec_ml[1].x - M) * inv;
#pragma unroll
                for (int k = 0; k < DPL; ++k) acc[k] = fmaf(spec_o[1][k], w1, acc[k]);
            }
        }
        __nv_bfloat16 *dst = p.out + ((long long)seq * p.num_q_heads + qh) * D + lane * DPL;
#pragma unroll
        for (int k = 0; k < DPL; ++k) dst[k] = __float2bfloat16_rn(acc[k]);
        return;
    }
    // maximum over the partitions, and whether any is empty (sum 0: a bad block)
    float M = -CUDART_INF_F;
    bool empty = false;
    for (int i = lane; i < n && !bad; i += 32) {
        const float2 ml = *reinterpret_cast<const float2 *>(p.part_ml + (base + i) * 2);
        M = fmaxf(M, ml.x);
        empty |= !(ml.y > 0.f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    bad = __any_sync(0xffffffffu, bad || empty);
    if (!bad) {
        float L = 0.f;
        for (int i = lane; i < n; i += 32) {
            const float2 ml = *reinterpret_cast<const float2 *>(p.part_ml + (base + i) * 2);
            L += ml.y * exp2f(ml.x - M);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        const float inv = 1.f / L;
        for (int i = 0; i < n; ++i) {
            const float2 ml = *reinterpret_cast<const float2 *>(p.part_ml + (base + i) * 2);
            const float w = ml.y * exp2f(ml.x - M) * inv;
            const float *po = p.part_o + (base + i) * D + lane * DPL;
            if constexpr (DPL == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(po);
                acc[0] = fmaf(v.x, w, acc[0]);
                acc[1] = fmaf(v.y, w, acc[1]);
                acc[2] = fmaf(v.z, w, acc[2]);
                acc[3] = fmaf(v.w, w, acc[3]);
            } else {
#pragma unroll
                for (int k = 0; k < DPL; ++k) acc[k] = fmaf(po[k], w, acc[k]);
            }
        }
    }
    __nv_bfloat16 *dst = p.out + ((long long)seq * p.num_q_heads + qh) * D + lane * DPL;
#pragma unroll
    for (int k = 0; k < DPL; ++k) dst[k] = __float2bfloat16_rn(acc[k]);
}

}  // namespace pkv
