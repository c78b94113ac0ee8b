/*
 * pkv_oracle.c -- plain, slow, fp64 CPU oracle for paged attention (one
 * decode step, and a chunk of prefill tokens attending causally) and for the
 * residual add + RMSNorm of the layer around it.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
 * CPU-baseline leg are the only callers. It shares no code, header, table or
 * constant with the CUDA library; the two meet only through the seeded inputs
 * that both consume.
 *
 * What it computes, and where the pages fix it:
 *
 *  - The KV cache is split into fixed-size blocks that need not be contiguous;
 *    a per-sequence block table maps logical block j to a physical block, and
 *    several requests may share physical blocks ("DeepSeek复刻vLLM反超原版",
 *    section "vLLM：大模型推理的加速引擎与挑战"; "nano-vllm：轻量级大模型推理引擎的
 *    技术探索与实践", section "PagedAttention 原理回顾"). The result is therefore
 *    ordinary attention over each sequence's tokens in logical order:
 *    out = softmax(scale * q K^T) V, evaluated here directly, in fp64, with no
 *    blocking, splitting or online rescaling.
 *  - The FP8 cache stores E4M3 codes ("nano-vllm-lite：深入理解LLM推理机制的教育级
 *    开源项目", section 核心技术改进 3 "FP8 KV Cache量化"). The code set is the
 *    OCP 8-bit floating point format, E4M3 variant: exponent bias 7, three
 *    mantissa bits, subnormals at exponent field 0, S.1111.111 the only NaN,
 *    no infinities, largest finite magnitude 448.
 *
 * Readings where the pages are silent (the same ones the CUDA library takes):
 *  - pool layout [num_blocks][num_kv_heads][block_size][head_dim]; slot s is
 *    block s / block_size, offset s % block_size;
 *  - query head h reads KV head h / (num_q_heads / num_kv_heads);
 *  - slot -1 means "do not write";
 *  - FP8 store: y = x / scale[h] as one IEEE binary32 division, then the
 *    nearest E4M3 value, ties to the even code, magnitudes beyond 448 clamped
 *    to 448 (NaN stays NaN);
 *  - FP8 read: code value times the head's scale, both exact in fp64.
 *  - FP8 with one scale per (token, KV head) (the same page, section 3, does
 *    not fix the scale granularity; this is the finer of its two readings):
 *    the store takes the row's largest |x| (over head_dim), s = that / 448
 *    as one binary32 division, raised to the smallest normal binary32 if it
 *    falls below it (so an all-zero row has a positive scale), writes s to
 *    the scale pool [num_blocks][num_kv_heads][block_size] at the token's
 *    slot and encodes x / s as above; a read multiplies the code by the
 *    token's own scale. fp8 == 2 selects this mode (fp8 == 1: one scale per
 *    KV head).
 *  - Add + RMSNorm (same page, section 核心技术改进 1 "CUDA融合内核：Add+RMSNorm":
 *    the residual add and the RMSNorm that follows it, fused): h = x + r,
 *    the residual stream continues as h, and the normalised output is
 *    w * h / sqrt(mean(h^2) + eps) over the hidden dimension.
 *  - Rotary position embedding of q and k before the store (orc_rope,
 *    orc_store_kvcache_rope; readings next to them): the rotation of the
 *    RoFormer paper, from a caller-built cos/sin table, in binary32 with a
 *    fixed operation order because its result is rounded to bf16.
 *  - Chunked prefill ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目",
 *    section 核心技术改进 2 "Chunked Prefill": a long prompt's prefill is cut
 *    into chunks that run interleaved with decode work): a chunk of c new
 *    tokens of a sequence whose K/V are already stored occupies the last c of
 *    its context_len positions, and each of them attends causally -- to
 *    itself and every earlier token of its sequence. A decode step is the
 *    case c = 1.
 *
 * Every function here is pinned by a CPU test (brute force against a
 * library softmax, invariants, closed forms, the OCP format points and a
 * library FP8 cast); none is "parity unpinned".
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_BOUNDS 5

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
double orc_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Value of one E4M3 code, from the format definition. */
double orc_e4m3_to_double(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6); /* subnormal: 0.mmm * 2^(1-7) */
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7); /* normal: 1.mmm * 2^(e-7) */
    return sign ? -mag : mag;
}

/*
 * Nearest E4M3 code to y: codes 0x00..0x7E have increasing magnitude, so a
 * binary search finds the code just below |y|; the nearer neighbour wins and
 * an exact midpoint goes to the even code. Saturating: |y| >= 448 gives 448.
 */
uint8_t orc_e4m3_from_float(float y)
{
    uint8_t sign;
    double a;
    int lo, hi;
    if (isnan(y))
        return 0x7F;
    sign = signbit(y) ? 0x80 : 0x00;
    a = fabs((double)y);
    if (a >= 448.0)
        return sign | 0x7E;
    lo = 0;
    hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_e4m3_to_double((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    if (lo < 0x7E) {
        double below = orc_e4m3_to_double((uint8_t)lo);
        double above = orc_e4m3_to_double((uint8_t)(lo + 1));
        double d_lo = a - below, d_hi = above - a;
        if (d_hi < d_lo || (d_hi == d_lo && (lo & 1)))
            lo += 1;
    }
    return sign | (uint8_t)lo;
}

/* Pool element index of (block, kv head, offset, dim) in the HND layout. */
static int64_t pool_index(int64_t blk, int h, int off, int i, int nkv, int bs, int d)
{
    return ((blk * nkv + h) * bs + off) * (int64_t)d + i;
}

/*
 * store_kvcache: write token t's K and V rows (all KV heads) into the pool
 * slot slot_mapping[t]; slot -1 is skipped. Pools hold bf16 bit patterns
 * (fp8 == 0) or E4M3 codes (fp8 == 1: scales per KV head, read; fp8 == 2:
 * scale pools per token and KV head, written). A slot beyond the pool is not
 * written and the call reports ORC_ERR_BOUNDS.
 */
int orc_store_kvcache(const uint16_t *k, const uint16_t *v, void *k_cache, void *v_cache,
                      const int32_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                      int head_dim, int block_size, int64_t num_blocks, int fp8,
                      float *k_scale, float *v_scale)
{
    int status = ORC_OK;
    int64_t t;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping || num_tokens < 0 || num_kv_heads < 1 ||
        head_dim < 1 || block_size < 1 || num_blocks < 1 || (fp8 && (!k_scale || !v_scale)))
        return ORC_ERR_ARG;
    for (t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        int64_t blk;
        int off, h, i;
        if (slot < 0)
            continue;
        if (slot >= num_blocks * (int64_t)block_size) {
            status = ORC_ERR_BOUNDS;
            continue;
        }
        blk = slot / block_size;
        off = (int)(slot % block_size);
        for (h = 0; h < num_kv_heads; ++h) {
            float ks = 0.0f, vs = 0.0f;
            if (fp8 == 1) {
                ks = k_scale[h];
                vs = v_scale[h];
            } else if (fp8 == 2) {
                /* this row's own scales: largest magnitude / 448 */
                int64_t sidx = ((int64_t)blk * num_kv_heads + h) * block_size + off;
                float ka = 0.0f, va = 0.0f;
                for (i = 0; i < head_dim; ++i) {
                    int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim + i;
                    ka = fmaxf(ka, fabsf((float)orc_bf16_to_double(k[src])));
                    va = fmaxf(va, fabsf((float)orc_bf16_to_double(v[src])));
                }
                ks = ka / 448.0f;
                vs = va / 448.0f;
                if (ks < FLT_MIN)
                    ks = FLT_MIN;
                if (vs < FLT_MIN)
                    vs = FLT_MIN;
                k_scale[sidx] = ks;
                v_scale[sidx] = vs;
            }
            for (i = 0; i < head_dim; ++i) {
                int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim + i;
                int64_t dst = pool_index(blk, h, off, i, num_kv_heads, block_size, head_dim);
                if (fp8) {
                    float kx = (float)orc_bf16_to_double(k[src]);
                    float vx = (float)orc_bf16_to_double(v[src]);
                    float ky = kx / ks;
                    float vy = vx / vs;
                    ((uint8_t *)k_cache)[dst] = orc_e4m3_from_float(ky);
                    ((uint8_t *)v_cache)[dst] = orc_e4m3_from_float(vy);
                } else {
                    ((uint16_t *)k_cache)[dst] = k[src];
                    ((uint16_t *)v_cache)[dst] = v[src];
                }
            }
        }
    }
    return status;
}

/* One cached element as an exact fp64 value (bf16 bits, or code * scale):
 * element idx of the pool, KV head h, and sidx its token's index in the
 * per-token scale pools (fp8 == 2). */
static double cache_value(const void *cache, int64_t idx, int fp8, const float *scale, int h, int64_t sidx)
{
    if (fp8 == 1)
        return orc_e4m3_to_double(((const uint8_t *)cache)[idx]) * (double)scale[h];
    if (fp8 == 2)
        return orc_e4m3_to_double(((const uint8_t *)cache)[idx]) * (double)scale[sidx];
    return orc_bf16_to_double(((const uint16_t *)cache)[idx]);
}

/* Index of (block, kv head, offset) in a per-token scale pool. */
static int64_t scale_index(int64_t blk, int h, int off, int nkv, int bs)
{
    return (blk * nkv + h) * bs + off;
}

/*
 * paged_attention_decode: for each of the S sequences (row s of q,
 * block_tables and context_lens) and each query head h, attend over the
 * context_lens[s] tokens whose K/V the block table locates, and write the
 * fp64 result to out[s][h][:]. A sequence whose length or block ids fall
 * outside the pool gets zeros and the call reports ORC_ERR_BOUNDS.
 * num_threads > 1 spreads sequences over OpenMP threads (no change in the
 * arithmetic of any one output).
 */
int orc_paged_attention_decode(const uint16_t *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                               float scale, int fp8, const float *k_scale, const float *v_scale,
                               double *out, int num_threads)
{
    int status = ORC_OK;
    int group, s;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || num_seqs < 0 ||
        num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads || head_dim < 1 ||
        block_size < 1 || num_blocks < 1 || max_blocks_per_seq < 1 ||
        (fp8 && (!k_scale || !v_scale)))
        return ORC_ERR_ARG;
    group = num_q_heads / num_kv_heads;
    if (num_threads < 1)
        num_threads = 1;

#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : status)
    for (s = 0; s < num_seqs; ++s) {
        const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;
        double *out_s = out + (int64_t)s * num_q_heads * head_dim;
        int ctx = context_lens[s];
        int bad = (ctx < 1 || ctx > max_blocks_per_seq * block_size);
        double *score, *w, *acc;
        int h, t, i;
        for (t = 0; !bad && t < ctx; t += block_size)
            bad = (table[t / block_size] < 0 || table[t / block_size] >= num_blocks);
        if (bad) {
            memset(out_s, 0, sizeof(double) * (size_t)num_q_heads * head_dim);
            status |= ORC_ERR_BOUNDS;
            continue;
        }
        score = (double *)malloc(sizeof(double) * (size_t)ctx);
        w = (double *)malloc(sizeof(double) * (size_t)ctx);
        acc = (double *)malloc(sizeof(double) * (size_t)head_dim);
        for (h = 0; h < num_q_heads; ++h) {
            int g = h / group;
            const uint16_t *q_h = q + ((int64_t)s * num_q_heads + h) * head_dim;
            double m = -INFINITY, z = 0.0;
            for (t = 0; t < ctx; ++t) {
                int64_t blk = table[t / block_size];
                int off = t % block_size;
                double dot = 0.0;
                for (i = 0; i < head_dim; ++i) {
                    int64_t idx = pool_index(blk, g, off, i, num_kv_heads, block_size, head_dim);
                    dot += orc_bf16_to_double(q_h[i]) * cache_value(k_cache, idx, fp8, k_scale, g, scale_index(blk, g, off, num_kv_heads, block_size));
                }
                score[t] = (double)scale * dot;
                if (score[t] > m)
                    m = score[t];
            }
            for (t = 0; t < ctx; ++t) {
                w[t] = exp(score[t] - m);
                z += w[t];
            }
            /* out_i = sum_t w_t V[t][i] / z, summed in increasing t. */
            for (i = 0; i < head_dim; ++i)
                acc[i] = 0.0;
            for (t = 0; t < ctx; ++t) {
                int64_t blk = table[t / block_size];
                int off = t % block_size;
                for (i = 0; i < head_dim; ++i) {
                    int64_t idx = pool_index(blk, g, off, i, num_kv_heads, block_size, head_dim);
                    acc[i] += w[t] * cache_value(v_cache, idx, fp8, v_scale, g, scale_index(blk, g, off, num_kv_heads, block_size));
                }
            }
            for (i = 0; i < head_dim; ++i)
                out_s[(int64_t)h * head_dim + i] = acc[i] / z;
        }
        free(score);
        free(w);
        free(acc);
    }
    return status;
}

/*
 * paged_attention_prefill: sequence s has c_s = cu_q_lens[s + 1] -
 * cu_q_lens[s] query tokens, rows cu_q_lens[s] .. cu_q_lens[s + 1] - 1 of q
 * ([total_q][num_q_heads][head_dim] bf16), and context_lens[s] tokens in the
 * cache including those c_s. Query token i of the chunk sits at position
 * p = context_lens[s] - c_s + i and attends over positions 0 .. p:
 * out = softmax(scale * q K[0..p]^T) V[0..p], in fp64, written to the same
 * row of out. A sequence with c_s = 0 has no rows. A sequence whose chunk is
 * longer than its context, whose context does not fit its table row, or
 * whose table names a block outside the pool gets zero rows and the call
 * reports ORC_ERR_BOUNDS. cu_q_lens must start at 0, never decrease, and end
 * at total_q (else ORC_ERR_ARG).
 */
int orc_paged_attention_prefill(const uint16_t *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *cu_q_lens, const int32_t *context_lens, int num_seqs,
                                int total_q, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int64_t num_blocks, float scale, int fp8,
                                const float *k_scale, const float *v_scale, double *out,
                                int num_threads)
{
    int status = ORC_OK;
    int group, s;
    if (!q || !k_cache || !v_cache || !block_tables || !cu_q_lens || !context_lens || !out ||
        num_seqs < 0 || total_q < 0 || num_q_heads < 1 || num_kv_heads < 1 ||
        num_q_heads % num_kv_heads || head_dim < 1 || block_size < 1 || num_blocks < 1 ||
        max_blocks_per_seq < 1 || (fp8 && (!k_scale || !v_scale)))
        return ORC_ERR_ARG;
    if (cu_q_lens[0] != 0 || cu_q_lens[num_seqs] != total_q)
        return ORC_ERR_ARG;
    for (s = 0; s < num_seqs; ++s)
        if (cu_q_lens[s + 1] < cu_q_lens[s])
            return ORC_ERR_ARG;
    group = num_q_heads / num_kv_heads;
    if (num_threads < 1)
        num_threads = 1;

#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : status)
    for (s = 0; s < num_seqs; ++s) {
        const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;
        int c = cu_q_lens[s + 1] - cu_q_lens[s];
        int ctx = context_lens[s];
        int bad, h, t, i, r;
        double *score, *w, *acc;
        if (c == 0)
            continue;
        bad = (ctx < c || ctx > max_blocks_per_seq * block_size);
        for (t = 0; !bad && t < ctx; t += block_size)
            bad = (table[t / block_size] < 0 || table[t / block_size] >= num_blocks);
        if (bad) {
            memset(out + (int64_t)cu_q_lens[s] * num_q_heads * head_dim, 0,
                   sizeof(double) * (size_t)c * num_q_heads * head_dim);
            status |= ORC_ERR_BOUNDS;
            continue;
        }
        score = (double *)malloc(sizeof(double) * (size_t)ctx);
        w = (double *)malloc(sizeof(double) * (size_t)ctx);
        acc = (double *)malloc(sizeof(double) * (size_t)head_dim);
        for (r = 0; r < c; ++r) {
            int64_t row = cu_q_lens[s] + r;
            int p = ctx - c + r; /* this query token's position */
            for (h = 0; h < num_q_heads; ++h) {
                int g = h / group;
                const uint16_t *q_h = q + (row * num_q_heads + h) * head_dim;
                double *out_h = out + (row * num_q_heads + h) * head_dim;
                double m = -INFINITY, z = 0.0;
                for (t = 0; t <= p; ++t) {
                    int64_t blk = table[t / block_size];
                    int off = t % block_size;
                    double dot = 0.0;
                    for (i = 0; i < head_dim; ++i) {
                        int64_t idx = pool_index(blk, g, off, i, num_kv_heads, block_size, head_dim);
                        dot += orc_bf16_to_double(q_h[i]) * cache_value(k_cache, idx, fp8, k_scale, g, scale_index(blk, g, off, num_kv_heads, block_size));
                    }
                    score[t] = (double)scale * dot;
                    if (score[t] > m)
                        m = score[t];
                }
                for (t = 0; t <= p; ++t) {
                    w[t] = exp(score[t] - m);
                    z += w[t];
                }
                for (i = 0; i < head_dim; ++i)
                    acc[i] = 0.0;
                for (t = 0; t <= p; ++t) {
                    int64_t blk = table[t / block_size];
                    int off = t % block_size;
                    for (i = 0; i < head_dim; ++i) {
                        int64_t idx = pool_index(blk, g, off, i, num_kv_heads, block_size, head_dim);
                        acc[i] += w[t] * cache_value(v_cache, idx, fp8, v_scale, g, scale_index(blk, g, off, num_kv_heads, block_size));
                    }
                }
                for (i = 0; i < head_dim; ++i)
                    out_h[i] = acc[i] / z;
            }
        }
        free(score);
        free(w);
        free(acc);
    }
    return status;
}

/*
 * Nearest bf16 value of an fp64 number, ties to the even significand,
 * overflow to infinity (IEEE round-to-nearest-even with 8 significant bits,
 * exponent range of binary32); returns the bf16 bit pattern. NaN gives the
 * quiet NaN 0x7FC0.
 */
uint16_t orc_bf16_from_double(double v)
{
    double a = fabs(v), quantum, q, fl, r;
    int e;
    uint16_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x8000 : 0;
    union { float f; uint32_t u; } cv;
    if (v != v)
        return 0x7FC0;
    if (a == 0.0)
        return sign;
    frexp(a, &e); /* a = m * 2^e, 0.5 <= m < 1 */
    if (e - 1 < -126)
        quantum = ldexp(1.0, -133); /* subnormal spacing */
    else
        quantum = ldexp(1.0, e - 8); /* 8 significant bits */
    q = a / quantum;                 /* exact: a power-of-two scaling */
    fl = floor(q);
    r = q - fl;
    if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) == 1.0))
        fl += 1.0;
    a = fl * quantum;
    if (a > 3.3895313892515355e38) /* beyond the largest finite bf16 */
        return sign | 0x7F80;
    cv.f = (float)a; /* exact: a has at most 8 significant bits */
    return sign | (uint16_t)(cv.u >> 16);
}

/*
 * fused_add_rmsnorm: for each of the num_tokens rows of hidden elements,
 * h = x + residual (x alone when residual is NULL), computed exactly in
 * fp64; residual_out (if not NULL) receives h rounded to bf16; out receives
 * weight * h / sqrt(mean(h^2) + eps) in fp64.
 */
int orc_fused_add_rmsnorm(const uint16_t *x, const uint16_t *residual, const uint16_t *weight, int num_tokens,
                          int hidden, double eps, double *out, uint16_t *residual_out, int num_threads)
{
    int t;
    if (!x || !weight || !out || num_tokens < 0 || hidden < 1 || !(eps >= 0))
        return ORC_ERR_ARG;
    if (num_threads < 1)
        num_threads = 1;
#pragma omp parallel for schedule(static) num_threads(num_threads)
    for (t = 0; t < num_tokens; ++t) {
        const int64_t row = (int64_t)t * hidden;
        double ss = 0.0, inv;
        int i;
        for (i = 0; i < hidden; ++i) {
            double h = orc_bf16_to_double(x[row + i]);
            if (residual)
                h += orc_bf16_to_double(residual[row + i]);
            out[row + i] = h;
            ss += h * h;
        }
        inv = 1.0 / sqrt(ss / hidden + eps);
        for (i = 0; i < hidden; ++i) {
            if (residual_out)
                residual_out[row + i] = orc_bf16_from_double(out[row + i]);
            out[row + i] = orc_bf16_to_double(weight[i]) * (out[row + i] * inv);
        }
    }
    return ORC_OK;
}

/*
 * Rotary position embedding (Su, Lu, Pan, Murtadha, Wen, Liu, "RoFormer:
 * Enhanced Transformer with Rotary Position Embedding", 2021): a head vector
 * of head_dim elements is cut into head_dim / 2 coordinate pairs, and pair i
 * of a token at position m is rotated by the angle m * theta_i,
 *     (x, y) -> (x cos - y sin, x sin + y cos).
 * The pages name the FP8 cache that the rotated keys are stored into
 * ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section 核心技术改进 3)
 * but give no formula for the rotation; these readings are taken:
 *  - the angles come from a table the caller builds once, cos_sin[m] =
 *    cos(m theta_0 .. m theta_{d/2-1}) then sin(...), binary32, for
 *    positions 0 .. max_position - 1 (theta_i = base^(-2i/d) in the paper);
 *  - pair i is (i, i + d/2) for style 0 (the halves of the vector) and
 *    (2i, 2i + 1) for style 1 (neighbours, as the paper writes it);
 *  - the rotated value is rounded to bf16 (the cache and q are bf16), so the
 *    arithmetic that decides the bf16 bits is fixed, in binary32, one
 *    rounding per step: x' = fma(-y, sin, x * cos), y' = fma(x, sin, y * cos)
 *    (fmaf is correctly rounded), then round to nearest even.
 * A position outside [0, max_position) leaves the row unwritten and the call
 * reports ORC_ERR_BOUNDS.
 */
static void pair_index(int i, int head_dim, int style, int *a, int *b)
{
    if (style == 1) {
        *a = 2 * i;
        *b = 2 * i + 1;
    } else {
        *a = i;
        *b = i + head_dim / 2;
    }
}

int orc_rope(const uint16_t *x, uint16_t *out, const int32_t *positions, int64_t num_tokens, int num_heads,
             int head_dim, const float *cos_sin, int64_t max_position, int style)
{
    int status = ORC_OK;
    int64_t t;
    if (!x || !out || !positions || !cos_sin || num_tokens < 0 || num_heads < 1 || head_dim < 2 ||
        head_dim % 2 != 0 || max_position < 1 || (style != 0 && style != 1))
        return ORC_ERR_ARG;
    for (t = 0; t < num_tokens; ++t) {
        int64_t m = positions[t];
        int h, i;
        if (m < 0 || m >= max_position) {
            status = ORC_ERR_BOUNDS;
            continue;
        }
        for (h = 0; h < num_heads; ++h) {
            const uint16_t *row = x + (t * num_heads + h) * (int64_t)head_dim;
            uint16_t *dst = out + (t * num_heads + h) * (int64_t)head_dim;
            for (i = 0; i < head_dim / 2; ++i) {
                int a, b;
                float xa, xb, c, s, ya, yb;
                pair_index(i, head_dim, style, &a, &b);
                xa = (float)orc_bf16_to_double(row[a]);
                xb = (float)orc_bf16_to_double(row[b]);
                c = cos_sin[m * head_dim + i];
                s = cos_sin[m * head_dim + head_dim / 2 + i];
                ya = fmaf(-xb, s, xa * c);
                yb = fmaf(xa, s, xb * c);
                dst[a] = orc_bf16_from_double((double)ya);
                dst[b] = orc_bf16_from_double((double)yb);
            }
        }
    }
    return status;
}

/*
 * store_kvcache_rope: q (if given) and k rotated at each token's position,
 * then k (rotated) and v (as is) stored exactly as orc_store_kvcache does --
 * the composition of the two steps, fused on the GPU. A token whose position
 * is out of range is neither rotated nor stored (ORC_ERR_BOUNDS).
 */
int orc_store_kvcache_rope(const uint16_t *q, uint16_t *q_out, const uint16_t *k, const uint16_t *v,
                           void *k_cache, void *v_cache, const int32_t *slot_mapping, const int32_t *positions,
                           int64_t num_tokens, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int64_t num_blocks, int fp8, float *k_scale, float *v_scale, const float *cos_sin,
                           int64_t max_position, int style)
{
    int status = ORC_OK, st;
    int64_t t;
    uint16_t *k_rot;
    int32_t *slots;
    if (!k || !v || !slot_mapping || !positions || num_tokens < 0 || (q && !q_out) || (q && num_q_heads < 1))
        return ORC_ERR_ARG;
    if (num_tokens == 0)
        return ORC_OK;
    k_rot = (uint16_t *)calloc((size_t)num_tokens * num_kv_heads * head_dim, sizeof(uint16_t));
    slots = (int32_t *)malloc((size_t)num_tokens * sizeof(int32_t));
    if (!k_rot || !slots) {
        free(k_rot);
        free(slots);
        return ORC_ERR_ARG;
    }
    if (q) {
        st = orc_rope(q, q_out, positions, num_tokens, num_q_heads, head_dim, cos_sin, max_position, style);
        if (st == ORC_ERR_ARG) {
            free(k_rot);
            free(slots);
            return st;
        }
    }
    st = orc_rope(k, k_rot, positions, num_tokens, num_kv_heads, head_dim, cos_sin, max_position, style);
    if (st == ORC_ERR_ARG) {
        free(k_rot);
        free(slots);
        return st;
    }
    for (t = 0; t < num_tokens; ++t) {
        int bad = positions[t] < 0 || positions[t] >= max_position;
        if (bad)
            status = ORC_ERR_BOUNDS;
        slots[t] = bad ? -1 : slot_mapping[t];
    }
    st = orc_store_kvcache(k_rot, v, k_cache, v_cache, slots, num_tokens, num_kv_heads, head_dim, block_size,
                           num_blocks, fp8, k_scale, v_scale);
    free(k_rot);
    free(slots);
    return st != ORC_OK ? st : status;
}
