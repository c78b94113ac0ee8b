// decode.cuh -- paged decode attention kernels (sm_100a, CUDA cores).
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
// Block structure: NCW consumer warps + 1 producer warp.
//  * Producer (one lane): walks the partition in tiles of TILE logical
//    tokens. A tile is cut at block boundaries into runs that are contiguous
//    in the HND pool; each run of K and of V is one bulk copy (non-tensor TMA,
//    cp.async.bulk) into a STAGES-deep ring in shared memory, completing on
//    the stage's "full" mbarrier. Only valid tokens are copied.
//  * Consumers: warp w owns rows [w*R, (w+1)*R) of every tile. A token row is
//    spread over LPT = head_dim/8 lanes, 8 elements each (16-byte loads for
//    bf16, 8-byte for E4M3), so a warp handles 32/LPT tokens per step. Per
//    tile: all scores of the warp's rows (8 fp32 FMAs per head per lane, then
//    a butterfly shuffle sum over the LPT lanes), the warp's running max per
//    head, rescale, then P*V into fp32 accumulators. Scores are kept in base
//    2: q is pre-multiplied by scale*log2(e) (and by the K scale for E4M3).
//  * Epilogue: merge the warps' (max, sum, accumulators) in shared memory and
//    write bf16 output, or, for split-K, the normalised fp32 partial with its
//    (max, sum) for the reduce kernel.
//
// Every wait is bounded (PKV_DEVERR_TIMEOUT), every block id and length is
// checked before a byte is copied (PKV_DEVERR_BOUNDS), and the producer
// waits for its own copies in flight before the block exits.
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
};

constexpr int kMaxIdsPerPartition = 256;

template <int D, int G, bool FP8, int TILE, int STAGES, int NCW>
struct DecodeTraits {
    static constexpr int kESize = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kESize;
    static constexpr int kEPL = 8;               // elements per lane of a row
    static constexpr int kLPT = D / kEPL;        // lanes per token row
    static constexpr int kTPS = 32 / kLPT;       // tokens per warp step
    static constexpr int kRows = TILE / NCW;     // rows per warp per tile
    static constexpr int kSteps = kRows / kTPS;  // steps per warp per tile
    static constexpr int kTileBytes = TILE * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kThreads = (NCW + 1) * 32;
    // shared memory layout (bytes)
    static constexpr int kOffBars = STAGES * kStageBytes;
    static constexpr int kOffIds = kOffBars + 2 * STAGES * 8;
    static constexpr int kOffMerge = kOffIds + kMaxIdsPerPartition * 4;
    static constexpr int kMergeFloats = NCW * G * D + 2 * NCW * G + NCW * G;
    static constexpr int kSmemBytes = kOffMerge + kMergeFloats * 4;
    static_assert(D % (kEPL * 1) == 0 && (32 % kLPT) == 0, "row mapping");
    static_assert(kRows % kTPS == 0 && kSteps >= 1, "tile must split evenly over warps and steps");
    static_assert(kStageBytes % 128 == 0, "stage alignment");
};

// 8 elements of a cached row (bf16: 16 bytes, E4M3: 8 bytes) -> fp32.
template <bool FP8>
__device__ __forceinline__ void load_row8(const uint8_t *p, float (&x)[8]) {
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

template <int D, int G, bool FP8, int TILE, int STAGES, int NCW, int MIN_BLOCKS>
__global__ void __launch_bounds__((NCW + 1) * 32, MIN_BLOCKS) paged_decode_kernel(const DecodeParams p) {
    using T = DecodeTraits<D, G, FP8, TILE, STAGES, NCW>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + T::kOffBars);
    uint64_t *empty_bar = full_bar + STAGES;
    int32_t *ids = reinterpret_cast<int32_t *>(smem + T::kOffIds);
    float *merge_acc = reinterpret_cast<float *>(smem + T::kOffMerge);  // [NCW][G][D]
    float *merge_m = merge_acc + NCW * G * D;                             // [NCW][G]
    float *merge_l = merge_m + NCW * G;                                   // [NCW][G]
    float *merge_w = merge_l + NCW * G;                                   // [NCW][G]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // which (sequence, KV head, partition)
    const int part = blockIdx.x % p.num_partitions;
    const int rest = blockIdx.x / p.num_partitions;
    const int kvh = rest % p.num_kv_heads;
    const int seq = rest / p.num_kv_heads;

    const int ctx = __ldg(p.context_lens + seq);
    const int table_cap = p.max_blocks_per_seq << p.log2_block_size;
    const bool bad_len = ctx < 1 || ctx > p.max_context_len || ctx > table_cap;
    const int start = part * p.partition_tokens;
    const int end = bad_len ? start : min(start + p.partition_tokens, ctx);
    const int n_parts_seq = bad_len ? 1 : (ctx + p.partition_tokens - 1) / p.partition_tokens;
    const bool single = n_parts_seq == 1;  // this block writes the final output
    if (!bad_len && start >= end) return;  // partition past this sequence's end
    if (bad_len && part != 0) return;

    // Stage this partition's block ids (checked) and set up the barriers.
    const int first_blk = start >> p.log2_block_size;
    const int n_blk = bad_len ? 0 : ((end - 1) >> p.log2_block_size) - first_blk + 1;
    int bad = bad_len || n_blk > kMaxIdsPerPartition;
    const int32_t *table = p.block_tables + (long long)seq * p.max_blocks_per_seq + first_blk;
    for (int i = tid; i < n_blk && i < kMaxIdsPerPartition; i += T::kThreads) {
        const int32_t id = __ldg(table + i);
        ids[i] = id;
        bad |= (id < 0 || (long long)id >= p.num_blocks);
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NCW);
        }
        fence_barrier_init();
    }
    bad = __syncthreads_or(bad);

    const int qh0 = kvh * G;  // first query head of this KV head
    if (bad) {
        if (tid == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
        if (single || bad_len) {
            for (int i = tid; i < G * D; i += T::kThreads)
                p.out[((long long)seq * p.num_q_heads + qh0) * D + i] = __float2bfloat16_rn(0.f);
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

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&empty_bar[s], ((j / STAGES) - 1) & 1)) {
                    set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
                    break;
                }
                const int a0 = start + j * TILE;
                const int a1 = min(a0 + TILE, end);
                uint8_t *ks = smem + s * T::kStageBytes;
                uint8_t *vs = ks + T::kTileBytes;
                mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(2 * (a1 - a0) * T::kRowBytes));
                for (int a = a0; a < a1;) {
                    const int lb = a >> p.log2_block_size;
                    const int off = a & (p.block_size - 1);
                    const int n = min(p.block_size - off, a1 - a);
                    const long long phys = ids[lb - first_blk];
                    const long long src = phys * blk_stride + kvh * head_stride + (long long)off * T::kRowBytes;
                    const int dst = (a - a0) * T::kRowBytes;
                    bulk_g2s(ks + dst, p.k_cache + src, (uint32_t)(n * T::kRowBytes), &full_bar[s]);
                    bulk_g2s(vs + dst, p.v_cache + src, (uint32_t)(n * T::kRowBytes), &full_bar[s]);
                    a += n;
                }
                issued = j + 1;
            }
            // Wait for every copy still in flight before this block may exit.
            for (int j = max(0, issued - STAGES); j < issued; ++j)
                if (!mbar_wait(&full_bar[j % STAGES], (j / STAGES) & 1)) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int sub = lane / T::kLPT;   // token within a step
    const int chunk = lane % T::kLPT;  // 8-element chunk of the row

    float qf[G][8];
    {
        float qs = p.qk_scale_log2;
        if constexpr (FP8) qs *= __ldg(p.k_scale + kvh);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p.q + ((long long)seq * p.num_q_heads + qh0 + h) * D +
                                                                  chunk * 8));
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                qf[h][2 * i] = bf16lo(ww[i]) * qs;
                qf[h][2 * i + 1] = bf16hi(ww[i]) * qs;
            }
        }
    }

    float acc[G][8];
    float m[G], l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -CUDART_INF_F;
        l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = 0.f;
    }

    const int row0 = warp * T::kRows;
    for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (!mbar_wait(&full_bar[s], (j / STAGES) & 1)) {
            set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
            break;
        }
        const int n_valid = min(TILE, end - (start + j * TILE));
        const int cnt = min(T::kRows, n_valid - row0);  // this warp's valid rows (warp-uniform)
        if (cnt > 0) {
            const uint8_t *ks = smem + s * T::kStageBytes + row0 * T::kRowBytes + chunk * 8 * T::kESize;
            const uint8_t *vs = ks + T::kTileBytes;
            float sc[T::kSteps][G];
            float tmax[G];
#pragma unroll
            for (int h = 0; h < G; ++h) tmax[h] = -CUDART_INF_F;
#pragma unroll
            for (int st = 0; st < T::kSteps; ++st) {
                const int r = st * T::kTPS + sub;
                if (st * T::kTPS < cnt) {
                    const bool valid = r < cnt;
                    float kf[8];
                    if (valid) {
                        load_row8<FP8>(ks + r * T::kRowBytes, kf);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) kf[i] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float d = 0.f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) d = fmaf(qf[h][i], kf[i], d);
#pragma unroll
                        for (int o = T::kLPT / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                        sc[st][h] = valid ? d : -CUDART_INF_F;
                        tmax[h] = fmaxf(tmax[h], sc[st][h]);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) sc[st][h] = -CUDART_INF_F;
                }
            }
            // warp-wide max per head, then rescale the running state
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int o = T::kLPT; o < 32; o <<= 1) tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], o));
                const float m_new = fmaxf(m[h], tmax[h]);
                const float alpha = exp2f(m[h] - m_new);
                m[h] = m_new;
                l[h] *= alpha;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[h][i] *= alpha;
            }
            // P * V
#pragma unroll
            for (int st = 0; st < T::kSteps; ++st) {
                const int r = st * T::kTPS + sub;
                if (st * T::kTPS < cnt) {
                    if (r < cnt) {
                        float vf[8];
                        load_row8<FP8>(vs + r * T::kRowBytes, vf);
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float pr = exp2f(sc[st][h] - m[h]);
                            l[h] += pr;
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[h][i] = fmaf(pr, vf[i], acc[h][i]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
    }

    // ------------------------------------------------------------- epilogue
    // Sum over the token groups of the warp (lanes with the same chunk).
#pragma unroll
    for (int o = T::kLPT; o < 32; o <<= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[h][i] += __shfl_xor_sync(0xffffffffu, acc[h][i], o);
        }
    }
    if (sub == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int i = 0; i < 8; ++i) merge_acc[(warp * G + h) * D + chunk * 8 + i] = acc[h][i];
            if (chunk == 0) {
                merge_m[warp * G + h] = m[h];
                merge_l[warp * G + h] = l[h];
            }
        }
    }
    named_sync(1, NCW * 32);
    if (tid < G) {
        const int h = tid;
        float M = -CUDART_INF_F;
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, merge_m[w * G + h]);
        float L = 0.f;
        for (int w = 0; w < NCW; ++w) {
            const float e = exp2f(merge_m[w * G + h] - M);  // 0 for a warp that saw no token
            merge_w[w * G + h] = e;
            L += merge_l[w * G + h] * e;
        }
        float post = 1.f / L;
        if constexpr (FP8) post *= __ldg(p.v_scale + kvh);
        for (int w = 0; w < NCW; ++w) merge_w[w * G + h] *= post;
        if (!single) {
            float *ml = p.part_ml + (((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + part) * 2;
            ml[0] = M;
            ml[1] = L;
        }
    }
    named_sync(1, NCW * 32);
    for (int idx = tid; idx < G * D; idx += NCW * 32) {
        const int h = idx / D;
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) o = fmaf(merge_acc[(w * G + h) * D + (idx % D)], merge_w[w * G + h], o);
        if (single) {
            p.out[((long long)seq * p.num_q_heads + qh0) * D + idx] = __float2bfloat16_rn(o);
        } else {
            p.part_o[(((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + part) * D + (idx % D)] = o;
        }
    }
}

// Merge the split-K partials of one (sequence, query head): weights
// l_p * 2^(m_p - M) over the sequence's partitions, fixed order.
template <int D>
__global__ void __launch_bounds__(D) paged_decode_reduce_kernel(const DecodeParams p) {
    const int qh = blockIdx.x % p.num_q_heads;
    const int seq = blockIdx.x / p.num_q_heads;
    const int ctx = __ldg(p.context_lens + seq);
    const int table_cap = p.max_blocks_per_seq << p.log2_block_size;
    if (ctx < 1 || ctx > p.max_context_len || ctx > table_cap) return;  // decode wrote zeros
    const int n = (ctx + p.partition_tokens - 1) / p.partition_tokens;
    if (n <= 1) return;  // decode wrote the output itself
    const long long base = ((long long)seq * p.num_q_heads + qh) * p.num_partitions;
    __shared__ float w_s[1024];
    __shared__ int bad_s;
    if (threadIdx.x == 0) {
        float M = -CUDART_INF_F;
        int bad = 0;
        for (int i = 0; i < n; ++i) {
            const float li = p.part_ml[(base + i) * 2 + 1];
            bad |= !(li > 0.f);
            M = fmaxf(M, p.part_ml[(base + i) * 2]);
        }
        float L = 0.f;
        for (int i = 0; i < n && !bad; ++i) {
            const float e = p.part_ml[(base + i) * 2 + 1] * exp2f(p.part_ml[(base + i) * 2] - M);
            w_s[i] = e;
            L += e;
        }
        const float inv = bad ? 0.f : 1.f / L;
        for (int i = 0; i < n && !bad; ++i) w_s[i] *= inv;
        bad_s = bad;
    }
    __syncthreads();
    float o = 0.f;
    if (!bad_s)
        for (int i = 0; i < n; ++i) o = fmaf(p.part_o[(base + i) * D + threadIdx.x], w_s[i], o);
    p.out[((long long)seq * p.num_q_heads + qh) * D + threadIdx.x] = __float2bfloat16_rn(o);
}

}  // namespace pkv
