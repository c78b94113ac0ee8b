// decode_mma.cuh -- paged decode attention over an E4M3 cache (head_dim 128)
// with the products on the warp-level tensor-core MMA (sm_100a).
//
// Two cache types share the kernel (template flag BF): E4M3 (one byte per
// element) and bf16.
//
// Why: with one byte per cached element, the CUDA-core decode is bound by
// instruction issue, not by HBM -- every (token, KV head) costs 2 * G * 128
// multiply-adds plus the E4M3 widening against only 256 bytes of K and V.
// The G query heads of a KV head against a tile of tokens are small matrix
// products, [tokens x d] x [d x G] for the scores and [d x tokens] x [tokens
// x G] for P V, so this kernel hands them to mma.sync m16n8k16 (f16 operands,
// fp32 accumulation): every E4M3 code widens exactly to f16 (one conversion
// per pair, straight into an operand register), q is scaled by a power of
// two into f16 (exact for bf16 q), and the MMA forms the exact products and
// accumulates them in fp32. What remains on the CUDA cores is the widening,
// the softmax and the bookkeeping. A bf16 cache feeds the MMA directly (bf16
// operands, no widening); its weights go in as a bf16 pair hi + lo (two MMAs)
// so that they keep about 16 significant bits. With bf16 the CUDA-core kernel
// already streams HBM near its peak, but its instruction stream is what
// limits it when the K/V come from L2 (blocks shared by many sequences), and
// it draws the power that caps the clock. The problem is the pages' decode
// ("DeepSeek复刻vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战":
// block tables into a shared pool; "nano-vllm-lite", section 核心技术改进 3:
// the FP8 KV cache and its 2x smaller reads).
//
// Block structure: one thread block of kNW warps per (sequence, KV head,
// partition); every K/V byte of the partition is read from HBM once. Each
// warp owns kWT consecutive tokens of every kTile-token tile and runs its own
// pipeline: lane 0 copies its rows of K and V with tensor-map copies
// (cp.async.bulk.tensor, 16-row boxes of 128 bytes -- one per row for E4M3,
// the two 64-element halves of a row for bf16 -- 128-byte swizzle, no
// multicast) into a kStages-deep ring, completing on the warp's own
// mbarriers, and refills a stage once the warp is done with it.
//
// Per 16-token group (fragment layouts of m16n8k16; g = lane / 4, t = lane % 4):
//  * Scores, S^T[16 tokens x 8 heads] = K[16 x 128] . Q^T[128 x 8]: A = K rows
//    g and g + 8, B = q of head g (zero for g >= G). The contraction order of
//    the 128 dims is free, so a lane's k-steps cover 32 dims of its two rows
//    that sit in two adjacent 16-byte chunks of each 128-byte half row:
//    E4M3, dims 32t .. 32t + 31 (one conversion per code pair gives an
//    operand register); bf16, dims 16t .. 16t + 15 and 64 + 16t .. + 15 (the
//    words are the operand registers). The swizzle makes these reads free of
//    bank conflicts.
//  * Softmax in base 2 over the warp's tile (scores times scale * log2 e,
//    the K scale and q's power of two), with a lazy reference maximum: it
//    moves only when the tile maximum exceeds it by more than 8, so weights
//    stay <= 2^8 (f16 range) and the accumulators are rescaled rarely.
//  * The weights, packed to f16, are transposed in registers
//    (movmatrix.trans) into the B operand of P V.
//  * P V, O^T[128 dims x 8 heads] += V^T[128 x 16 tokens] . P^T[16 x 8]: an
//    m-tile covers dims e (row g) and e + 1 (row g + 8), with e = 16g + 2j
//    (E4M3) or 64h + 8g + 2q (bf16, m-tile 4h + q), so a lane reads the
//    16-byte chunk g of 4 rows (of each half, bf16); byte permutes pair two
//    tokens' elements at one dim (before the conversion, for E4M3).
//  * Rows past the end of the context (inside the last copied box) are
//    excluded: their scores become -inf and their V codes zero.
//  * Per-token scales (TS): the K and V scale runs are bulk-copied with the
//    boxes; a score is multiplied by its token's K scale; a weight by its V
//    scale times 2^-E before it is rounded to f16, where E tracks the largest
//    V scale seen so far (a rise of E rescales the accumulators exactly, like
//    a rise of the maximum), and l sums the unscaled weights.
//  * Epilogue as in the CUDA-core kernel: the warps' (max, sum, accumulators)
//    merge in shared memory, then bf16 output or a normalised split-K partial.
//
// Every wait is bounded (PKV_DEVERR_TIMEOUT), every block id and length is
// checked before a byte is copied (PKV_DEVERR_BOUNDS), and each warp waits
// for its own copies in flight before the block exits.
#pragma once

#include <cuda.h>

#include "decode.cuh"
#include "tc_common.cuh"

namespace pkv {

#ifndef PKV_MMA_WARPS
#define PKV_MMA_WARPS 4
#endif
#ifndef PKV_MMA_WARP_TOKENS
#define PKV_MMA_WARP_TOKENS 32
#endif
#ifndef PKV_MMA_STAGES
#define PKV_MMA_STAGES 2
#endif

#ifndef PKV_MMA_WARP_TOKENS_BF16
#define PKV_MMA_WARP_TOKENS_BF16 16
#endif
#ifndef PKV_MMA_STAGES_BF16
#define PKV_MMA_STAGES_BF16 2
#endif

template <int G, bool BF = false>
struct MmaTraits {
    static constexpr int kD = 128;
    static constexpr int kNW = PKV_MMA_WARPS;
    static constexpr int kWT = BF ? PKV_MMA_WARP_TOKENS_BF16 : PKV_MMA_WARP_TOKENS;  // tokens per warp per tile
    static constexpr int kNGW = kWT / 16;            // 16-token groups per warp per tile
    static constexpr int kTile = kNW * kWT;
    static constexpr int kStages = BF ? PKV_MMA_STAGES_BF16 : PKV_MMA_STAGES;
    static constexpr int kRowBytes = BF ? 256 : 128;
    static constexpr int kHalves = BF ? 2 : 1;  // 128-byte boxes per row
    // a 16-row group: [half][16 rows][128 bytes]
    static constexpr int kGroupBytes = 16 * kRowBytes;
    static constexpr int kSliceBytes = kWT * kRowBytes;  // a warp's K (or V) rows of one tile
    // [stage][warp][K slice | V slice], 1024-byte aligned (the swizzle atom)
    static constexpr int kStageBytes = kNW * 2 * kSliceBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kOffScales = kRingBytes;  // [stage][warp][K | V][kWT] fp32 (per-token scales)
    static constexpr int kScaleBytes = kStages * kNW * 2 * kWT * 4;
    static constexpr int kOffBars = kOffScales + kScaleBytes;  // full_k[NW][S], full_v[NW][S]
    static constexpr int kOffCnt = kOffBars + 2 * kNW * kStages * 8;
    static constexpr int kOffIds = kOffCnt + kNW * 4;
    static constexpr int kSmemBytes = kOffIds + kMaxIdsPerPartition * 4;
    static constexpr int kAlloc = kSmemBytes + 1024;  // + base alignment
    static constexpr int kThreads = kNW * 32;
    static constexpr int kMergeFloats = kNW * G * kD + 3 * kNW * G;
    static_assert(kWT % 16 == 0 && kNGW >= 1, "whole 16-token groups");
    static_assert(kMergeFloats * 4 <= kRingBytes, "merge area must fit in the ring");
    static_assert(G >= 1 && G <= 8, "one n8 column per query head");
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ float lds32f(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// D += A . B, m16n8k16, f16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A . B, m16n8k16, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool BF>
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    if constexpr (BF)
        mma_bf16_16816(d, a0, a1, a2, a3, b0, b1);
    else
        mma_f16_16816(d, a0, a1, a2, a3, b0, b1);
}

// Transpose of an 8 x 8 matrix of 16-bit elements held one word per lane
// (lane g*4 + t holds row g, columns 2t and 2t + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Swizzled row r, 16-byte chunk c of a 16-row group at byte address base.
__device__ __forceinline__ uint32_t swz16(uint32_t base, int r, int c) {
    return base + r * 128 + (((c ^ r) & 7) << 4);
}

// q fragments of the row this lane's column g reads (qrow; null: a column
// with no query, zeros), for k-steps in the order of the K reads below:
// qf[i][0] = dims d_i, d_i + 1, qf[i][1] = dims d_i + 2, d_i + 3, with d_i =
// 32t + 4i (E4M3) or 64(i / 4) + 16t + 4(i % 4) (bf16). E4M3: q becomes f16
// after a power-of-two rescale that puts the warp's largest |q| in
// [2^14, 2^15) (exact for bf16 q down to 2^-29 of it); bf16: q as is.
// Returns the multiplier of a raw score into base-2 units (score_scale_log2
// times the undoing power of two). Every lane of the warp must call it.
template <bool BF>
__device__ __forceinline__ float load_q_frags(const __nv_bfloat16 *qrow, int t, float score_scale_log2,
                                              uint32_t (&qf)[8][2]) {
    uint32_t qw[16];
    if (qrow) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e0 = BF ? (i >> 1) * 64 + 16 * t + (i & 1) * 8 : 32 * t + 8 * i;
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(qrow + e0));
            qw[4 * i] = w.x;
            qw[4 * i + 1] = w.y;
            qw[4 * i + 2] = w.z;
            qw[4 * i + 3] = w.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) qw[i] = 0u;
    }
    if constexpr (BF) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            qf[i][0] = qw[2 * i];
            qf[i][1] = qw[2 * i + 1];
        }
        return score_scale_log2;
    } else {
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fmaxf(fabsf(bf16lo(qw[i])), fabsf(bf16hi(qw[i]))));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        frexpf(mx, &e);  // mx < 2^e
        const int k = 15 - e;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            qf[i][0] = tc::pack_f16(ldexpf(bf16lo(qw[2 * i]), k), ldexpf(bf16hi(qw[2 * i]), k));
            qf[i][1] = tc::pack_f16(ldexpf(bf16lo(qw[2 * i + 1]), k), ldexpf(bf16hi(qw[2 * i + 1]), k));
        }
        return ldexpf(score_scale_log2, -k);
    }
}

// Raw scores of one 16-token group: c = S^T fragment (tokens g, g + 8 x
// columns 2t, 2t + 1). Two accumulators take alternate k-steps (two
// independent MMA chains) and are added at the end.
template <bool BF>
__device__ __forceinline__ void qk_group(uint32_t kg, int g, int t, const uint32_t (&qf)[8][2], float (&c)[4]) {
    float c2[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (BF) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint4 k0 = lds128(swz16(kg + hh * 2048, g, 2 * t));
            const uint4 k1 = lds128(swz16(kg + hh * 2048, g, 2 * t + 1));
            const uint4 k2 = lds128(swz16(kg + hh * 2048, g + 8, 2 * t));
            const uint4 k3 = lds128(swz16(kg + hh * 2048, g + 8, 2 * t + 1));
            const uint32_t wg[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
            const uint32_t wh[8] = {k2.x, k2.y, k2.z, k2.w, k3.x, k3.y, k3.z, k3.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mma_bf16_16816((i & 1) ? c2 : c, wg[2 * i], wh[2 * i], wg[2 * i + 1], wh[2 * i + 1],
                               qf[4 * hh + i][0], qf[4 * hh + i][1]);
        }
    } else {
        const uint4 k0 = lds128(swz16(kg, g, 2 * t));
        const uint4 k1 = lds128(swz16(kg, g, 2 * t + 1));
        const uint4 k2 = lds128(swz16(kg, g + 8, 2 * t));
        const uint4 k3 = lds128(swz16(kg, g + 8, 2 * t + 1));
        const uint32_t wg[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        const uint32_t wh[8] = {k2.x, k2.y, k2.z, k2.w, k3.x, k3.y, k3.z, k3.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint2 a = tc::e4m3x4_to_f16x4(wg[i]);  // row g: dims +0,+1 | +2,+3
            const uint2 b = tc::e4m3x4_to_f16x4(wh[i]);  // row g + 8
            mma_f16_16816((i & 1) ? c2 : c, a.x, b.x, a.y, b.y, qf[i][0], qf[i][1]);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] += c2[k];
}

// o += P V of one 16-token group. pw: the weights of tokens g, g + 8 x
// columns 2t, 2t + 1 (already times 2^-vexp and the V scale for per-token
// scales). Rows at or past n_valid (of 16) read as zero: stale slots of a
// partial box may hold NaN.
template <bool BF>
__device__ __forceinline__ void pv_group(uint32_t vg, int g, int t, const float (&pw)[4], int n_valid,
                                         float (&o)[8][4]) {
    uint4 r[2][4];
#pragma unroll
    for (int hh = 0; hh < (BF ? 2 : 1); ++hh) {
        const uint32_t vh = vg + hh * 2048;
        r[hh][0] = lds128(swz16(vh, 2 * t, g));
        r[hh][1] = lds128(swz16(vh, 2 * t + 1, g));
        r[hh][2] = lds128(swz16(vh, 2 * t + 8, g));
        r[hh][3] = lds128(swz16(vh, 2 * t + 9, g));
        if (n_valid < 16) {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            if (2 * t >= n_valid) r[hh][0] = z;
            if (2 * t + 1 >= n_valid) r[hh][1] = z;
            if (2 * t + 8 >= n_valid) r[hh][2] = z;
            if (2 * t + 9 >= n_valid) r[hh][3] = z;
        }
    }
    if constexpr (BF) {
        // weights as bf16 hi + lo: p - hi is exact in fp32 and lo keeps the
        // next 8 bits
        const uint32_t h01 = tc::pack_bf16(pw[0], pw[1]), h23 = tc::pack_bf16(pw[2], pw[3]);
        const uint32_t l01 = tc::pack_bf16(pw[0] - bf16lo(h01), pw[1] - bf16hi(h01));
        const uint32_t l23 = tc::pack_bf16(pw[2] - bf16lo(h23), pw[3] - bf16hi(h23));
        const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
        const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t w0[4] = {r[hh][0].x, r[hh][0].y, r[hh][0].z, r[hh][0].w};
            const uint32_t w1[4] = {r[hh][1].x, r[hh][1].y, r[hh][1].z, r[hh][1].w};
            const uint32_t w2[4] = {r[hh][2].x, r[hh][2].y, r[hh][2].z, r[hh][2].w};
            const uint32_t w3[4] = {r[hh][3].x, r[hh][3].y, r[hh][3].z, r[hh][3].w};
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
                // dims 64hh + 8g + 2qd, + 1 of tokens (2t, 2t+1) and (2t+8, 2t+9)
                const uint32_t a0 = __byte_perm(w0[qd], w1[qd], 0x5410);
                const uint32_t a1 = __byte_perm(w0[qd], w1[qd], 0x7632);
                const uint32_t a2 = __byte_perm(w2[qd], w3[qd], 0x5410);
                const uint32_t a3 = __byte_perm(w2[qd], w3[qd], 0x7632);
                mma_bf16_16816(o[4 * hh + qd], a0, a1, a2, a3, bh0, bh1);
                mma_bf16_16816(o[4 * hh + qd], a0, a1, a2, a3, bl0, bl1);
            }
        }
    } else {
        const uint32_t b0 = movmatrix_trans(tc::pack_f16(pw[0], pw[1]));  // tokens 2t, 2t+1 of column g
        const uint32_t b1 = movmatrix_trans(tc::pack_f16(pw[2], pw[3]));  // tokens 2t+8, 2t+9
        const uint32_t w0[4] = {r[0][0].x, r[0][0].y, r[0][0].z, r[0][0].w};
        const uint32_t w1[4] = {r[0][1].x, r[0][1].y, r[0][1].z, r[0][1].w};
        const uint32_t w2[4] = {r[0][2].x, r[0][2].y, r[0][2].z, r[0][2].w};
        const uint32_t w3[4] = {r[0][3].x, r[0][3].y, r[0][3].z, r[0][3].w};
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
            // dims 16g + 4qd .. +3 of tokens (2t, 2t+1) and (2t+8, 2t+9)
            const uint2 x0 = tc::e4m3x4_to_f16x4(__byte_perm(w0[qd], w1[qd], 0x5140));
            const uint2 x1 = tc::e4m3x4_to_f16x4(__byte_perm(w0[qd], w1[qd], 0x7362));
            const uint2 y0 = tc::e4m3x4_to_f16x4(__byte_perm(w2[qd], w3[qd], 0x5140));
            const uint2 y1 = tc::e4m3x4_to_f16x4(__byte_perm(w2[qd], w3[qd], 0x7362));
            mma_f16_16816(o[2 * qd], x0.x, x0.y, y0.x, y0.y, b0, b1);
            mma_f16_16816(o[2 * qd + 1], x1.x, x1.y, y1.x, y1.y, b0, b1);
        }
    }
}

// Softmax of one tile of NG groups in base 2 for the lane's columns 2t, 2t + 1:
// x holds the scaled scores (-inf past the end). The reference maximum moves
// only when the tile maximum exceeds it by more than 8 (so weights stay below
// 2^8); alpha receives the factor the accumulators must take (1 when nothing
// moved, in every lane when the return value is false), l is rescaled and
// takes the new weights pw.
template <int NG>
__device__ __forceinline__ bool tile_softmax(const float (&x)[NG][4], float (&m_ref)[2], float (&l)[2],
                                             float (&alpha)[2], float (&pw)[NG][4]) {
    float mx[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(x[0][h], x[0][2 + h]);
#pragma unroll
        for (int gi = 1; gi < NG; ++gi) mx[h] = fmaxf(mx[h], fmaxf(x[gi][h], x[gi][2 + h]));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], off));
    }
    const bool move = mx[0] > m_ref[0] + 8.f || mx[1] > m_ref[1] + 8.f;
    alpha[0] = alpha[1] = 1.f;
    const bool rescale = __any_sync(0xffffffffu, move);
    if (rescale) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float mn = fmaxf(m_ref[h], mx[h]);
            alpha[h] = m_ref[h] == -CUDART_INF_F ? 0.f : fast_exp2(m_ref[h] - mn);
            m_ref[h] = mn;
        }
    }
    const float mr0 = m_ref[0] == -CUDART_INF_F ? 0.f : m_ref[0];
    const float mr1 = m_ref[1] == -CUDART_INF_F ? 0.f : m_ref[1];
    l[0] *= alpha[0];
    l[1] *= alpha[1];
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
        pw[gi][0] = fast_exp2(x[gi][0] - mr0);
        pw[gi][1] = fast_exp2(x[gi][1] - mr1);
        pw[gi][2] = fast_exp2(x[gi][2] - mr0);
        pw[gi][3] = fast_exp2(x[gi][3] - mr1);
        l[0] += pw[gi][0] + pw[gi][2];
        l[1] += pw[gi][1] + pw[gi][3];
    }
    return rescale;
}

// Per-token V scales (E4M3 with scale pools): the scales of the lane's rows
// g, g + 8 of each group sit at vs_addr + 4 * row (0 past nv). A tile maximum
// at or above 2^vexp raises vexp and folds the exact factor 2^-rise into
// alpha, so that the weights times 2^-vexp stay below 2^9 in f16; the weights
// are multiplied by their token's scale times 2^-vexp.
template <int NG>
__device__ __forceinline__ bool tile_vscale(uint32_t vs_addr, int nv, int g, int &vexp, float &vinv,
                                            float (&alpha)[2], float (&pw)[NG][4]) {
    float vsc[NG][2];
    float vm = 0.f;
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
        const bool v0 = gi * 16 + g < nv, v1 = gi * 16 + g + 8 < nv;
        vsc[gi][0] = v0 ? lds32f(vs_addr + (gi * 16 + g) * 4) : 0.f;
        vsc[gi][1] = v1 ? lds32f(vs_addr + (gi * 16 + g + 8) * 4) : 0.f;
        vm = fmaxf(vm, fmaxf(vsc[gi][0], vsc[gi][1]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
    // vm < 2^ev (vm >= the smallest normal: scales are floored there, and the
    // tile has a valid token); the same in every lane
    const int ev = (int)(__float_as_uint(vm) >> 23) - 126;
    bool rise = false;
    if (ev > vexp) {
        const float f = ldexpf(1.f, vexp - ev);  // 0 for the first rise
        alpha[0] *= f;
        alpha[1] *= f;
        rise = true;
        vexp = ev;
        vinv = ldexpf(1.f, -vexp);
    }
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
        const float f0 = vsc[gi][0] * vinv, f1 = vsc[gi][1] * vinv;
        pw[gi][0] *= f0;
        pw[gi][1] *= f0;
        pw[gi][2] *= f1;
        pw[gi][3] *= f1;
    }
    return rise;
}

__device__ __forceinline__ void rescale_acc(float (&o)[8][4], const float (&alpha)[2]) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        o[jj][0] *= alpha[0];
        o[jj][1] *= alpha[1];
        o[jj][2] *= alpha[0];
        o[jj][3] *= alpha[1];
    }
}

// Dim held by accumulator o[j][0..1] (o[j][2..3]: the next dim) of row
// group g: 16g + 2j (E4M3) or 64(j / 4) + 8g + 2(j % 4) (bf16).
template <bool BF>
__device__ __forceinline__ int acc_dim(int j, int g) {
    return BF ? (j >> 2) * 64 + 8 * g + 2 * (j & 3) : 16 * g + 2 * j;
}

template <int G, bool BF, int MIN_BLOCKS, bool TS>
__global__ void __launch_bounds__(MmaTraits<G, BF>::kThreads, MIN_BLOCKS)
    paged_decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap map_k,
                            const __grid_constant__ CUtensorMap map_v, int box_rows) {
    static_assert(!(BF && TS), "per-token scales exist only for E4M3");
    using T = MmaTraits<G, BF>;
    constexpr int D = T::kD;
    constexpr int NW = T::kNW;
    constexpr int WT = T::kWT;
    constexpr int NGW = T::kNGW;
    constexpr int TILE = T::kTile;
    constexpr int STAGES = T::kStages;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = smem_addr(smem);
    int32_t *ids = reinterpret_cast<int32_t *>(smem + T::kOffIds);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;  // fragment row group
    const int t = lane & 3;   // thread in group

    const int part = blockIdx.x % p.grid_partitions;
    const int rest = blockIdx.x / p.grid_partitions;
    const int kvh = rest % p.num_kv_heads;
    const int seq_slot = rest / p.num_kv_heads;
    const int seq = p.seq_order ? __ldg(p.seq_order + seq_slot) : seq_slot;
    if (seq < 0 || seq >= p.num_seqs) {
        if (tid == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
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
    // Shared-prefix mode: this kernel attends tokens [P, ctx) of the sequence
    // (its group's shared prefix is the prefix kernel's) and always writes a
    // partial, to slot part + 1.
    int P = 0;
    if (p.cu_group_seqs && !bad_len) {
        P = prefix_of(p, seq, ctx);
        if (P < 0) {  // the merge writes zeros for this sequence
            if (tid == 0 && part == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
            return;
        }
    }
    const int pslot = part + (p.cu_group_seqs ? 1 : 0);
    const int start = P + part * p.partition_tokens;
    const int end = bad_len ? start : min(start + p.partition_tokens, ctx);
    const int n_parts_seq = bad_len ? 1 : (ctx - P + p.partition_tokens - 1) / p.partition_tokens;
    const bool single = n_parts_seq == 1 && !p.cu_group_seqs;
    if (!bad_len && start >= end) return;
    if (bad_len && part != 0) return;

    // every block id of the partition is checked; the first ones are staged
    const int first_blk = start >> p.log2_block_size;
    const int n_blk = bad_len ? 0 : ((end - 1) >> p.log2_block_size) - first_blk + 1;
    int bad = bad_len;
    const int32_t *table = p.block_tables + (long long)seq * p.max_blocks_per_seq + first_blk;
    for (int i = tid; i < n_blk; i += T::kThreads) {
        const int32_t id = __ldg(table + i);
        if (i < kMaxIdsPerPartition) ids[i] = id;
        bad |= (id < 0 || (long long)id >= p.num_blocks);
    }
    uint64_t *full_k = reinterpret_cast<uint64_t *>(smem + T::kOffBars) + warp * STAGES;
    uint64_t *full_v = full_k + NW * STAGES;
    int *issued = reinterpret_cast<int *>(smem + T::kOffCnt) + warp;  // tiles this warp issued
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
        }
        fence_barrier_init();
    }
    bad = __syncthreads_or(bad);
    const int qh0 = kvh * G;
    if (bad) {
        if (tid == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
        if (single || bad_len) {
            for (int i = tid; i < G * D; i += T::kThreads)
                p.out[(row * p.num_q_heads + qh0) * D + i] = __float2bfloat16_rn(0.f);
        } else if (tid < G) {
            float *ml = p.part_ml + (((long long)seq * p.num_q_heads + qh0 + tid) * p.num_partitions + pslot) * 2;
            ml[0] = -CUDART_INF_F;
            ml[1] = 0.f;
        }
        return;
    }

    const int n_tiles = (end - start + TILE - 1) / TILE;
    const int bs_mask = p.block_size - 1;
    const int lbs = p.log2_block_size;
    // This warp's rows of tile j: logical tokens [start + j*TILE + warp*WT, ...).
    auto warp_tok0 = [&](int j) { return start + j * TILE + warp * WT; };
    // Issue this warp's K and V boxes (and, TS, scale runs) of tile j into
    // stage s. Only boxes holding at least one valid token are copied; a box
    // never leaves its (block, KV head) run, since box_rows divides 16 and
    // the block size, and groups start on multiples of 16.
    auto issue = [&](int j, int s) {
        const int a0 = warp_tok0(j);
        const int nv = min(end - a0, WT);
        uint32_t bytes = 0;
        for (int a = 0; a < nv; a += box_rows) bytes += box_rows * T::kRowBytes + (TS ? box_rows * 4 : 0);
        mbar_arrive_expect_tx(&full_k[s], bytes);
        mbar_arrive_expect_tx(&full_v[s], bytes);
        const uint32_t sk = sbase + s * T::kStageBytes + warp * 2 * T::kSliceBytes;
        const uint32_t sv = sk + T::kSliceBytes;
        for (int a = 0; a < nv; a += box_rows) {
            const int tok = a0 + a;
            const int bi = (tok >> lbs) - first_blk;
            const long long phys = bi < kMaxIdsPerPartition ? ids[bi] : __ldg(table + bi);
            const long long row = (phys * p.num_kv_heads + kvh) * p.block_size + (tok & bs_mask);
            // group a / 16, rows a % 16 .. of each 128-byte half
            const uint32_t dst = (a >> 4) * T::kGroupBytes + (a & 15) * 128;
#pragma unroll
            for (int hh = 0; hh < T::kHalves; ++hh) {
                tc::tma_load_2d(sk + dst + hh * 2048, &map_k, hh * 64, (int)row, &full_k[s]);
                tc::tma_load_2d(sv + dst + hh * 2048, &map_v, hh * 64, (int)row, &full_v[s]);
            }
            if constexpr (TS) {
                uint8_t *sc = smem + T::kOffScales + ((s * NW + warp) * 2) * WT * 4;
                bulk_g2s(sc + a * 4, p.k_scale + row, box_rows * 4, &full_k[s]);
                bulk_g2s(sc + WT * 4 + a * 4, p.v_scale + row, box_rows * 4, &full_v[s]);
            }
        }
    };
    if (lane == 0) {
        int n = 0;
        for (int j = 0; j < min(STAGES, n_tiles) && warp_tok0(j) < end; ++j, ++n) issue(j, j);
        *issued = n;
    }
    __syncwarp();

    // q of head qh0 + g, dims 32t .. 32t + 31, as f16 pairs in k-step order:
    // qf[i][0] = dims 32t + 4i, +1; qf[i][1] = dims 32t + 4i + 2, +3 (zero
    // for g >= G). Scaled by 2^k so that the largest |q| of the KV head's
    // group lies in [2^14, 2^15): exact for bf16 q down to 2^-29 of it.
    uint32_t qf[8][2];
    const float score_scale = load_q_frags<BF>(
        g < G ? p.q + (row * p.num_q_heads + qh0 + g) * D : nullptr, t,
        (BF || TS) ? p.qk_scale_log2 : p.qk_scale_log2 * __ldg(p.k_scale + kvh), qf);

    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[j][i] = 0.f;
    float m_ref[2] = {-CUDART_INF_F, -CUDART_INF_F};  // heads 2t, 2t + 1 (base-2 units)
    float l[2] = {0.f, 0.f};
    int vexp = -100000;  // TS: weights are scaled by 2^-vexp before rounding
    float vinv = 0.f;    // 2^-vexp

    bool ok = true;
    int s = 0, rnd = 0;
    for (int j = 0; j < n_tiles; ++j) {
        const int a0 = warp_tok0(j);
        const int nv = min(end - a0, WT);  // valid tokens of this warp in tile j
        if (nv <= 0) break;                // only in the last tile
        if (!mbar_wait(&full_k[s], rnd & 1)) {
            ok = false;
            break;
        }
        const uint32_t sk = sbase + s * T::kStageBytes + warp * 2 * T::kSliceBytes;
        const uint32_t sv = sk + T::kSliceBytes;
        const uint32_t ssc = smem_addr(smem + T::kOffScales) + ((s * NW + warp) * 2) * WT * 4;

        // ---- scores of the warp's groups (x: base-2 units)
        float x[NGW][4];
#pragma unroll
        for (int gi = 0; gi < NGW; ++gi) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            if (gi * 16 < nv) qk_group<BF>(sk + gi * T::kGroupBytes, g, t, qf, c);
            float ks0 = score_scale, ks1 = score_scale;
            if constexpr (TS) {
                ks0 *= lds32f(ssc + (gi * 16 + g) * 4);
                ks1 *= lds32f(ssc + (gi * 16 + g + 8) * 4);
            }
            // c: (token g, head 2t), (g, 2t + 1), (g + 8, 2t), (g + 8, 2t + 1)
            const bool v0 = gi * 16 + g < nv, v1 = gi * 16 + g + 8 < nv;
            x[gi][0] = v0 ? c[0] * ks0 : -CUDART_INF_F;
            x[gi][1] = v0 ? c[1] * ks0 : -CUDART_INF_F;
            x[gi][2] = v1 ? c[2] * ks1 : -CUDART_INF_F;
            x[gi][3] = v1 ? c[3] * ks1 : -CUDART_INF_F;
        }
        float alpha[2], pw[NGW][4];
        bool rescale = tile_softmax<NGW>(x, m_ref, l, alpha, pw);
        if (!mbar_wait(&full_v[s], rnd & 1)) {
            ok = false;
            break;
        }
        if constexpr (TS) rescale |= tile_vscale<NGW>(ssc + WT * 4, nv, g, vexp, vinv, alpha, pw);
        if (rescale) rescale_acc(o, alpha);
        // ---- P V
#pragma unroll
        for (int gi = 0; gi < NGW; ++gi) {
            if (gi * 16 < nv) pv_group<BF>(sv + gi * T::kGroupBytes, g, t, pw[gi], nv - gi * 16, o);
        }
        __syncwarp();
        if (lane == 0) {
            const int jn = j + STAGES;
            if (jn < n_tiles && warp_tok0(jn) < end) {
                fence_proxy_async_smem();
                issue(jn, s);
                *issued = jn + 1;
            }
        }
        if (++s == STAGES) {
            s = 0;
            ++rnd;
        }
    }
    if (!ok) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
    (void)rnd;

    // ------------------------------------------------------------- epilogue
    // l: sum over the lanes of the same heads (the g bits).
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
    if (lane == 0) {  // copies of this warp still in flight (only after a timeout)
        const int n_iss = *issued;
        for (int jj = max(0, n_iss - STAGES); jj < n_iss; ++jj) {
            const int ss = jj % STAGES;
            const uint32_t par = (jj / STAGES) & 1;
            if (!mbar_wait(&full_k[ss], par) || !mbar_wait(&full_v[ss], par)) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
        }
    }
    __syncthreads();
    float *merge_acc = reinterpret_cast<float *>(smem);  // [NW][G][D]
    float *merge_m = merge_acc + NW * G * D;            // [NW][G]
    float *merge_l = merge_m + NW * G;                  // [NW][G]
    float *merge_w = merge_l + NW * G;                  // [NW][G]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int head = 2 * t + h;
        if (head < G) {
            const float sc = TS ? ldexpf(1.f, vexp) : 1.f;  // TS: undo the 2^-vexp of the weights
            float *dst = merge_acc + (warp * G + head) * D;
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2) {
                // m-tiles jj, jj + 1 hold dims e, e + 1, e + 2, e + 3
                const int e = acc_dim<BF>(jj, g);
                *reinterpret_cast<float4 *>(dst + e) =
                    make_float4(o[jj][h] * sc, o[jj][2 + h] * sc, o[jj + 1][h] * sc, o[jj + 1][2 + h] * sc);
            }
            if (g == 0) {
                merge_m[warp * G + head] = m_ref[h];
                merge_l[warp * G + head] = l[h];
            }
        }
    }
    __syncthreads();
    if (tid < G) {
        const int h = tid;
        float M = -CUDART_INF_F;
        for (int w = 0; w < NW; ++w) M = fmaxf(M, merge_m[w * G + h]);
        float L = 0.f;
        for (int w = 0; w < NW; ++w) {
            const float e = merge_m[w * G + h] == -CUDART_INF_F ? 0.f : exp2f(merge_m[w * G + h] - M);
            merge_w[w * G + h] = e;
            L += merge_l[w * G + h] * e;
        }
        float post = 1.f / L;
        if constexpr (!TS && !BF) post *= __ldg(p.v_scale + kvh);
        for (int w = 0; w < NW; ++w) merge_w[w * G + h] *= post;
        if (!single) {
            float *ml = p.part_ml + (((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + pslot) * 2;
            ml[0] = M;
            ml[1] = L;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += T::kThreads) {
        const int h = idx / D;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) acc = fmaf(merge_acc[(w * G + h) * D + (idx % D)], merge_w[w * G + h], acc);
        if (single) {
            p.out[(row * p.num_q_heads + qh0) * D + idx] = __float2bfloat16_rn(acc);
        } else {
            p.part_o[(((long long)seq * p.num_q_heads + qh0 + h) * p.num_partitions + pslot) * D + (idx % D)] = acc;
        }
    }
}

// ------------------------------------------------------- shared prefixes
//
// Shared-prefix (cascade) decode, the prefix half. Sequences that share
// their first P cached tokens (the same physical blocks: prefix caching,
// "Nano-vLLM：轻量高效的大模型推理框架", section 三.2(1) 前缀缓存; sharing across
// requests, "DeepSeek复刻vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战")
// attend those tokens here once per group of member sequences instead of
// once each: a thread block takes up to 4 * (8 / G) members of one group and
// one KV head; a producer warp copies the prefix tile by tile (the same
// tensor-map boxes as the decode kernel) into a ring that every consumer
// warp reads; consumer warp w computes the 8 columns (member, head) of its
// 8 / G members with the decode kernel's per-group MMA code, so each K/V
// fragment read from shared memory serves 8 query rows and each tile read
// from L2 or HBM serves all the block's members. Each member gets its
// prefix partial (normalised O, max, sum) in split-K slot 0; the decode
// kernel writes the suffix partials and the merge combines them.
//
// Checks (PKV_DEVERR_BOUNDS; the member's partial gets sum 0, which makes the
// merge write zeros): P a whole number of blocks within the table, the
// leader's block ids inside the pool, every member's context at least P and
// every member's first P / block_size block ids equal to the leader's.

template <bool BF>
struct PrefixTraits {
    static constexpr int kNW = 4;  // consumer warps; warp kNW issues the copies
    static constexpr int kThreads = (kNW + 1) * 32;
    static constexpr int kRowBytes = BF ? 256 : 128;
    static constexpr int kHalves = BF ? 2 : 1;
    static constexpr int kGroupBytes = 16 * kRowBytes;
    static constexpr int kNG = 4;        // 16-token groups per stage
    static constexpr int kTT = 16 * kNG;  // tokens per stage
    static constexpr int kStages = BF ? 3 : 4;
    static constexpr int kHalfBytes = kNG * kGroupBytes;  // K (or V) of one stage
    static constexpr int kStageBytes = 2 * kHalfBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kOffScales = kRingBytes;  // [stage][K | V][kTT] fp32
    static constexpr int kOffBars = kOffScales + kStages * 2 * kTT * 4;  // full_k[S], full_v[S], empty[S]
    static constexpr int kOffFlags = kOffBars + 3 * kStages * 8;
    static constexpr int kOffIds = kOffFlags + 16;
    static constexpr int kSmemBytes = kOffIds + kMaxIdsPerPartition * 4;
    static constexpr int kAlloc = kSmemBytes + 1024;
};

// two blocks per SM: at three the register cap spills (measured slower)
template <int G, bool BF, bool TS>
__global__ void __launch_bounds__(PrefixTraits<BF>::kThreads, 2)
    paged_prefix_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap map_k,
                            const __grid_constant__ CUtensorMap map_v, int box_rows, int max_chunks) {
    static_assert(!(BF && TS), "per-token scales exist only for E4M3");
    using T = PrefixTraits<BF>;
    constexpr int D = 128;
    constexpr int NW = T::kNW;
    constexpr int NG = T::kNG;
    constexpr int TT = T::kTT;
    constexpr int STAGES = T::kStages;
    constexpr int SPW = 8 / G;        // member sequences per consumer warp
    constexpr int MC = NW * SPW;      // member sequences per block
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = smem_addr(smem);
    int32_t *ids = reinterpret_cast<int32_t *>(smem + T::kOffIds);
    unsigned *bad_mask = reinterpret_cast<unsigned *>(smem + T::kOffFlags);
    uint64_t *full_k = reinterpret_cast<uint64_t *>(smem + T::kOffBars);
    uint64_t *full_v = full_k + STAGES;
    uint64_t *empty = full_v + STAGES;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int grp = blockIdx.x / max_chunks;
    const int chunk = blockIdx.x % max_chunks;
    const int kvh = blockIdx.y;
    if (grp >= p.num_groups) return;
    const int m0 = __ldg(p.cu_group_seqs + grp), m1 = __ldg(p.cu_group_seqs + grp + 1);
    if (m0 < 0 || m1 < m0 || m1 > p.num_seqs) {  // members cannot be located safely
        if (tid == 0 && chunk == 0 && kvh == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
        return;
    }
    const int first = m0 + chunk * MC;
    if (first >= m1) return;
    const int last = min(first + MC, m1);
    const int P = __ldg(p.group_prefix + grp);
    if (P == 0) return;  // nothing shared: the decode kernel attends every token

    const int lbs = p.log2_block_size;
    const int bs_mask = p.block_size - 1;
    const int table_cap = p.max_blocks_per_seq << lbs;
    const bool p_ok = P > 0 && (P & bs_mask) == 0 && P <= table_cap;
    const int n_blk = p_ok ? P >> lbs : 0;
    const int32_t *lead = p.block_tables + (long long)m0 * p.max_blocks_per_seq;
    if (tid == 0) *bad_mask = 0u;
    __syncthreads();
    int bad_all = !p_ok;
    for (int i = tid; i < n_blk; i += T::kThreads) {
        const int32_t id = __ldg(lead + i);
        if (i < kMaxIdsPerPartition) ids[i] = id;
        bad_all |= (id < 0 || (long long)id >= p.num_blocks);
    }
    for (int mi = 0; mi < last - first; ++mi) {
        const int m = first + mi;
        const int32_t *row = p.block_tables + (long long)m * p.max_blocks_per_seq;
        int bad_m = 0;
        if (tid == 0) {
            const int c = __ldg(p.context_lens + m);
            bad_m = c < P || c > p.max_context_len || c > table_cap;
        }
        for (int i = tid; i < n_blk; i += T::kThreads) bad_m |= __ldg(row + i) != __ldg(lead + i);
        if (bad_m) atomicOr(bad_mask, 1u << mi);
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
            mbar_init(&empty[s], NW);
        }
        fence_barrier_init();
    }
    bad_all = __syncthreads_or(bad_all);
    const unsigned bmask = *bad_mask;
    const int qh0 = kvh * G;
    if (bad_all || bmask) {
        if (tid == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
    }
    if (bad_all) {  // every member's prefix partial: sum 0 (the merge writes zeros)
        for (int i = tid; i < (last - first) * G; i += T::kThreads) {
            float *ml = p.part_ml + (((long long)(first + i / G) * p.num_q_heads + qh0 + i % G) * p.num_partitions) * 2;
            ml[0] = -CUDART_INF_F;
            ml[1] = 0.f;
        }
        return;
    }

    const int n_tiles = (P + TT - 1) / TT;
    if (warp == NW) {  // ------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&empty[s], ((j / STAGES) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int a0 = j * TT;
                const int nv = min(P - a0, TT);
                uint32_t bytes = 0;
                for (int a = 0; a < nv; a += box_rows) bytes += box_rows * T::kRowBytes + (TS ? box_rows * 4 : 0);
                mbar_arrive_expect_tx(&full_k[s], bytes);
                mbar_arrive_expect_tx(&full_v[s], bytes);
                const uint32_t sk = sbase + s * T::kStageBytes;
                const uint32_t sv = sk + T::kHalfBytes;
                for (int a = 0; a < nv; a += box_rows) {
                    const int tok = a0 + a;
                    const int bi = tok >> lbs;
                    const long long phys = bi < kMaxIdsPerPartition ? ids[bi] : __ldg(lead + bi);
                    const long long row = (phys * p.num_kv_heads + kvh) * p.block_size + (tok & bs_mask);
                    const uint32_t dst = (a >> 4) * T::kGroupBytes + (a & 15) * 128;
#pragma unroll
                    for (int hh = 0; hh < T::kHalves; ++hh) {
                        tc::tma_load_2d(sk + dst + hh * 2048, &map_k, hh * 64, (int)row, &full_k[s]);
                        tc::tma_load_2d(sv + dst + hh * 2048, &map_v, hh * 64, (int)row, &full_v[s]);
                    }
                    if constexpr (TS) {
                        uint8_t *sc = smem + T::kOffScales + s * 2 * TT * 4;
                        bulk_g2s(sc + a * 4, p.k_scale + row, box_rows * 4, &full_k[s]);
                        bulk_g2s(sc + TT * 4 + a * 4, p.v_scale + row, box_rows * 4, &full_v[s]);
                    }
                }
                issued = j + 1;
            }
            if (!ok) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
            // copies still in flight (only when the consumers gave up)
            for (int jj = max(0, issued - STAGES); jj < issued; ++jj) {
                const uint32_t par = (jj / STAGES) & 1;
                if (!mbar_wait(&full_k[jj % STAGES], par) || !mbar_wait(&full_v[jj % STAGES], par))
                    set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
            }
        }
        return;  // no block-wide barrier follows
    }

    // ------------------------------------------------------------ consumers
    // column g of warp w: member first + w * SPW + g / G, head qh0 + g % G
    const int my_member = first + warp * SPW + g / G;
    uint32_t qf[8][2];
    const float score_scale = load_q_frags<BF>(
        my_member < last ? p.q + ((long long)my_member * p.num_q_heads + qh0 + g % G) * D : nullptr, t,
        (BF || TS) ? p.qk_scale_log2 : p.qk_scale_log2 * __ldg(p.k_scale + kvh), qf);
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[j][i] = 0.f;
    float m_ref[2] = {-CUDART_INF_F, -CUDART_INF_F};
    float l[2] = {0.f, 0.f};
    int vexp = -100000;
    float vinv = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        const uint32_t par = (j / STAGES) & 1;
        const int nv = min(P - j * TT, TT);
        if (!mbar_wait(&full_k[s], par)) {
            ok = false;
            break;
        }
        const uint32_t sk = sbase + s * T::kStageBytes;
        const uint32_t sv = sk + T::kHalfBytes;
        const uint32_t ssc = smem_addr(smem + T::kOffScales) + s * 2 * TT * 4;
        float x[NG][4];
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            if (gi * 16 < nv) qk_group<BF>(sk + gi * T::kGroupBytes, g, t, qf, c);
            float ks0 = score_scale, ks1 = score_scale;
            if constexpr (TS) {
                ks0 *= lds32f(ssc + (gi * 16 + g) * 4);
                ks1 *= lds32f(ssc + (gi * 16 + g + 8) * 4);
            }
            const bool v0 = gi * 16 + g < nv, v1 = gi * 16 + g + 8 < nv;
            x[gi][0] = v0 ? c[0] * ks0 : -CUDART_INF_F;
            x[gi][1] = v0 ? c[1] * ks0 : -CUDART_INF_F;
            x[gi][2] = v1 ? c[2] * ks1 : -CUDART_INF_F;
            x[gi][3] = v1 ? c[3] * ks1 : -CUDART_INF_F;
        }
        float alpha[2], pw[NG][4];
        bool rescale = tile_softmax<NG>(x, m_ref, l, alpha, pw);
        if (!mbar_wait(&full_v[s], par)) {
            ok = false;
            break;
        }
        if constexpr (TS) rescale |= tile_vscale<NG>(ssc + TT * 4, nv, g, vexp, vinv, alpha, pw);
        if (rescale) rescale_acc(o, alpha);
#pragma unroll
        for (int gi = 0; gi < NG; ++gi)
            if (gi * 16 < nv) pv_group<BF>(sv + gi * T::kGroupBytes, g, t, pw[gi], nv - gi * 16, o);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!ok) set_error(p.dev_err, PKV_DEVERR_TIMEOUT);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
    // each lane writes its two columns' dims of the slot-0 partial
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int col = 2 * t + h;
        const int member = first + warp * SPW + col / G;
        if (member >= last) continue;
        const bool bad_m = ((bmask >> (member - first)) & 1u) || !ok;
        const long long slot = ((long long)member * p.num_q_heads + qh0 + col % G) * p.num_partitions;
        float inv = bad_m ? 0.f : 1.f / l[h];
        if constexpr (TS) inv *= ldexpf(1.f, vexp);  // undo the 2^-vexp of the weights
        if constexpr (!TS && !BF) inv *= __ldg(p.v_scale + kvh);
        float *dst = p.part_o + slot * D;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int e = acc_dim<BF>(jj, g);
            *reinterpret_cast<float2 *>(dst + e) = make_float2(o[jj][h] * inv, o[jj][2 + h] * inv);
        }
        if (g == 0) {
            p.part_ml[slot * 2] = bad_m ? -CUDART_INF_F : m_ref[h];
            p.part_ml[slot * 2 + 1] = bad_m ? 0.f : l[h];
        }
    }
}

// The E4M3 pool as a 2-D tensor of 128-byte rows (one (block, KV head, slot)
// row each); boxes of 128 bytes x box_rows rows, 128-byte swizzle.
inline bool make_e4m3_pool_map(CUtensorMap *map, const void *pool, long long rows, int box_rows) {
    tc::EncodeTiledFn fn = tc::encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(pool), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bf16 pool as a 2-D tensor of 128-element rows; boxes of 64 elements
// (128 bytes) x box_rows rows, 128-byte swizzle (a row takes two boxes).
inline bool make_bf16_pool_map(CUtensorMap *map, const void *pool, long long rows, int box_rows) {
    tc::EncodeTiledFn fn = tc::encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(pool), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pkv
