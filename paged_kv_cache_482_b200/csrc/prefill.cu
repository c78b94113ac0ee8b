// prefill.cu -- chunked-prefill paged attention on the 5th-generation tensor
// cores (sm_100a): tcgen05.mma with operands in shared memory and fp32
// accumulators in tensor memory.
//
// The operation ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section
// 核心技术改进 2 "Chunked Prefill"; the paged cache of "DeepSeek复刻vLLM反超原版",
// section "vLLM：大模型推理的加速引擎与挑战"): sequence s brings a chunk of
// c = cu_q_lens[s+1] - cu_q_lens[s] query tokens whose K/V are already in the
// cache as the last c of its context_lens[s] positions; token i of the chunk
// (position p = ctx - c + i) attends over positions 0..p. A decode request is
// the case c = 1, so one launch serves a batch that mixes both.
//
// Work unit: one CTA per (sequence, KV head, 128 query rows), 256 threads and
// two CTAs per SM. A row is a (chunk token, query head of the group) pair:
// row r = token r / G, head r % G, so the G heads that share a KV head share
// every K/V tile. This kernel takes the chunks of at most one query tile
// (128 / G tokens, decode requests among them) and prefill_ws.cu the longer
// ones, for every cache type. The CTA walks the sequence's KV in 64-token
// tiles up to its last row's position:
//   1. K/V tiles are gathered through the block table into shared memory,
//      double buffered, in the 128-byte-swizzled layout the tensor core
//      reads: for a bf16 cache one thread issues tensor-map (TMA) copies of
//      whole block runs (a 2-D view of the pool, 64 columns x up to 64 rows
//      per copy, no multicast) and the V rows past the causal end are zeroed
//      on the last tile; an E4M3 cache is loaded and widened by the threads;
//   2. one thread issues S = Q K^T (M 128, N 64, K head_dim) into tensor
//      memory, queued right behind P V of the previous tile;
//   3. two threads per row read half of the row's tensor-memory columns each,
//      apply the causal mask, combine the row maximum through shared memory
//      and write P = exp2(s - m) as bf16 over the K tile S has consumed (or
//      into a buffer of its own for head_dim 64);
//   4. one thread issues O += P V (M 128, N head_dim, K 64; V read MN-major
//      straight from its row layout) into a second tensor-memory buffer. The
//      reference maximum moves only when a tile's maximum exceeds it by more
//      than 8 (log2 domain); then the row's O is rescaled in tensor memory.
//
// Shared-memory operand layout (all four operands): [head_dim / 64 or
// 128 / 64 column blocks][rows][128 bytes], the 16-byte chunk c of row r
// stored at chunk c ^ (r % 8) -- the canonical 128-byte swizzle, so one
// descriptor form serves Q, K and P (K-major) and V (MN-major).
#include <atomic>

#include "tc_common.cuh"

namespace pkv {
namespace {

using namespace tc;

constexpr int kRows = 128;  // MMA M: query rows per CTA
constexpr int kBN = 64;     // KV tokens per tile
constexpr int kThreads = 256;          // two threads per row: each owns half of the tile's score columns
constexpr int kHalfCols = kBN / 2;
constexpr uint32_t kTmemCols = 256;  // S: 64 columns, O: up to 128 columns (two CTAs fill an SM's 512)
constexpr uint32_t kMinSmem = 100u * 1024u;  // at most two CTAs per SM, whatever head_dim
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Layout {
    static constexpr int kHalves = D / 64;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kQBytes = kHalves * kRows * 128;
    static constexpr uint32_t kTileBytes = kHalves * kBN * 128;
    static constexpr uint32_t kK0 = kQ + kQBytes;
    static constexpr uint32_t kV0 = kK0 + kTileBytes;
    static constexpr uint32_t kBufStride = 2 * kTileBytes;  // K1 = K0 + stride, V1 = V0 + stride
    // P (kRows x kBN bf16) overwrites the K tile it was computed from when it
    // fits (head_dim 128): S has consumed that tile by the time P is written.
    // Otherwise P has a buffer of its own, free once the previous P V is done.
    static constexpr uint32_t kPBytes = (kBN / 64) * kRows * 128;
    static constexpr bool kPInK = kPBytes <= kTileBytes;
    static constexpr uint32_t kP = kK0 + 2 * kBufStride;
    static constexpr uint32_t kBar = kP + (kPInK ? 0 : kPBytes);  // 4 mbarriers, TMEM address
    static constexpr uint32_t kTable = kBar + 64;                  // the sequence's first block ids
    static constexpr uint32_t kScales = kTable + kTableCap * 4;    // per-token scales: [2 buffers][K, V][kBN]
    static constexpr uint32_t kRed = kScales + 2 * 2 * kBN * 4;     // row-max halves: [2 tiles][2 halves][kRows]
    static constexpr uint32_t kBytes = kRed + 3 * 2 * kRows * 4;  // + the final l exchange [2][kRows]
    static constexpr uint32_t kAlloc = (kBytes + 1024 > kMinSmem) ? kBytes + 1024 : kMinSmem;  // + base alignment
};

// Stage KV tile j (logical tokens j*kBN ..) of KV head kh into one K/V buffer.
// Tokens at or past kv_end are zero-filled; their scores are masked anyway
// and zeros keep P V finite.
template <int D, bool FP8, bool TS = false>
__device__ __forceinline__ void load_kv_tile(const PrefillArgs &a, const BlockIds &table, int kh, int j, int kv_end,
                                             int log2_bs, uint32_t sk, uint32_t sv, float *scales = nullptr) {
    if constexpr (TS) {
        // K scales of the tile's tokens in scales[0..kBN), 0 past the end (the
        // V scales are applied to V as it is staged, below)
        if (threadIdx.x < kBN) {
            const int t = threadIdx.x;
            const int pos = j * kBN + t;
            float sc = 0.0f;
            if (pos < kv_end) {
                const int64_t blk = table[pos >> log2_bs];
                const int64_t idx = (blk * a.num_kv_heads + kh) * a.block_size + (pos & (a.block_size - 1));
                sc = __ldg(a.k_scale + idx);
            }
            scales[t] = sc;
        }
    }
    constexpr int kChunks = D / 8;             // 16-byte chunks per bf16 row
    constexpr int kTokPerPass = kThreads / kChunks;
    const int c16 = threadIdx.x % kChunks;
    const int t_first = threadIdx.x / kChunks;
    const int bs = a.block_size;
#pragma unroll 4
    for (int t = t_first; t < kBN; t += kTokPerPass) {
        const int pos = j * kBN + t;
        const bool valid = pos < kv_end;
        const int p = valid ? pos : 0;
        const int64_t blk = table[p >> log2_bs];
        const int64_t elem = ((blk * a.num_kv_heads + kh) * bs + (p & (bs - 1))) * D + c16 * 8;
        const uint32_t off = swz(kBN, t, c16);
        if constexpr (FP8) {
            uint2 kw = make_uint2(0, 0), vw = make_uint2(0, 0);
            float vs = 0.0f;
            if (valid) {
                kw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(a.k_cache) + elem));
                vw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(a.v_cache) + elem));
                if constexpr (TS) vs = __ldg(a.v_scale + elem / D);  // the row's V scale
            }
            st_shared16(sk + off, e4m3x8_to_bf16x8(kw));
            // per-token scales: V is dequantised here (bf16 of code x scale), so P needs no scaling
            st_shared16(sv + off, TS ? e4m3x8_scaled_bf16x8(vw, vs) : e4m3x8_to_bf16x8(vw));
        } else {
            const __nv_bfloat16 *kc = static_cast<const __nv_bfloat16 *>(a.k_cache);
            const __nv_bfloat16 *vc = static_cast<const __nv_bfloat16 *>(a.v_cache);
            cp_async16(sk + off, kc + elem, valid ? 16u : 0u);
            cp_async16(sv + off, vc + elem, valid ? 16u : 0u);
        }
    }
}

// One thread: stage KV tile j of KV head kh (bf16 cache) with tensor-map
// copies. The pool is viewed as rows (block * nkv + head) * bs + offset of
// head_dim elements; a copy moves 64 columns (one 128-byte swizzle span) of
// min(bs, kBN) consecutive rows of one block. Blocks wholly past kv_end are
// not copied.
template <int D>
__device__ __forceinline__ void tma_kv_tile(const CUtensorMap *mk, const CUtensorMap *mv, const BlockIds &table, int nkv,
                                            int kh, int bs, int log2_bs, int j, int kv_end, uint32_t sk, uint32_t sv,
                                            uint64_t *bar) {
    constexpr int kHalves = D / 64;
    const int kv0 = j * kBN;
    if (bs >= kBN) {
        const int blk = table[kv0 >> log2_bs];
        const int row = (blk * nkv + kh) * bs + (kv0 & (bs - 1));
        mbar_arrive_expect_tx(bar, 2u * kHalves * kBN * 128u);
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
            tma_load_2d(sk + h * kBN * 128, mk, h * 64, row, bar);
            tma_load_2d(sv + h * kBN * 128, mv, h * 64, row, bar);
        }
    } else {
        const int end = min(kv0 + kBN, kv_end);
        const int nb = (end - kv0 + bs - 1) >> log2_bs;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(2 * kHalves * nb * bs * 128));
        for (int i = 0; i < nb; ++i) {
            const int blk = table[(kv0 >> log2_bs) + i];
            const int row = (blk * nkv + kh) * bs;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
                tma_load_2d(sk + h * kBN * 128 + i * bs * 128, mk, h * 64, row, bar);
                tma_load_2d(sv + h * kBN * 128 + i * bs * 128, mv, h * 64, row, bar);
            }
        }
    }
}

template <int D, int G, bool FP8, bool TS = false>
__global__ void __launch_bounds__(kThreads, 2)
    paged_prefill_kernel(PrefillArgs a, int tiles_per_seq, int log2_bs, const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v) {
    using L = Layout<D>;
    constexpr int TQ = kRows / G;  // chunk tokens per CTA
    constexpr uint32_t kIdescS = idesc_bf16(kRows, kBN, false);
    constexpr uint32_t kIdescPV = idesc_bf16(kRows, D, true);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    uint64_t *bar_s = reinterpret_cast<uint64_t *>(sm + L::kBar);
    uint64_t *bar_pv = bar_s + 1;
    uint64_t *bar_kv = bar_s + 2;  // one per K/V buffer (TMA copies)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bar_s + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    // query-tile-major over the sequences: the last (longest causal range)
    // tiles of every sequence are scheduled first
    const int s = blockIdx.x % a.num_seqs;
    const int tile = tiles_per_seq - 1 - blockIdx.x / a.num_seqs;
    const int kh = blockIdx.y;
    const int nq = a.num_q_heads;

    // ------------------------------------------------ bounds and bookkeeping
    const int q0 = a.cu_q_lens[s];
    const int q1 = a.cu_q_lens[s + 1];
    if (q0 < 0 || q1 < q0 || q1 > a.total_q) {
        if (tid == 0 && tile == 0 && kh == 0) set_error(a.dev_err, PKV_DEVERR_BOUNDS);
        return;  // no row of this sequence can be located safely
    }
    const int c = q1 - q0;
    const int t0 = tile * TQ;
    if (t0 >= c) return;
    if (a.small_cut > 0 && c > a.small_cut) return;  // a longer chunk: the warp-specialised kernel's
    if (c < a.small_min) return;                     // a one-token chunk: the decode kernel's
    const int ctx = a.context_lens[s];
    const int32_t *table_g = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
    int32_t *table_s = reinterpret_cast<int32_t *>(sm + L::kTable);
    bool bad = ctx < c || static_cast<int64_t>(ctx) > static_cast<int64_t>(a.max_blocks_per_seq) * a.block_size ||
               c > a.max_q_len;
    if (!bad) {
        const int nblk_seq = (ctx + a.block_size - 1) >> log2_bs;
        for (int i = tid; i < nblk_seq; i += kThreads) {
            const int32_t b = table_g[i];
            if (b < 0 || b >= a.num_blocks) bad = true;
            if (i < kTableCap) table_s[i] = b;
        }
    }
    const BlockIds table{table_s, table_g};
    // Two threads per row: warps w and w + 4 read the same tensor-memory lanes
    // (32 (w % 4) ..), the first the low half of the score and output
    // columns, the second the high half.
    const int row = tid & (kRows - 1);
    const int half = tid >> 7;
    const int row_tok = t0 + row / G;  // this thread's row
    const int row_head = kh * G + row % G;
    const bool row_live = row_tok < c;
    __nv_bfloat16 *out_row = static_cast<__nv_bfloat16 *>(a.out) +
                             (static_cast<int64_t>(q0 + (row_live ? row_tok : 0)) * nq + row_head) * D + half * (D / 2);
    if (__syncthreads_or(bad)) {
        if (row_live) {
            for (int i = 0; i < D / 2; i += 8) *reinterpret_cast<uint4 *>(out_row + i) = make_uint4(0, 0, 0, 0);
        }
        if (tid == 0) set_error(a.dev_err, PKV_DEVERR_BOUNDS);
        return;
    }
    const int last_tok = min(t0 + TQ, c) - 1;
    const int p_first = ctx - c + t0;  // position of the CTA's first row
    const int p_last = ctx - c + last_tok;
    const int kv_end = p_last + 1;
    const int n_tiles = (kv_end + kBN - 1) / kBN;
    const int row_pos = row_live ? ctx - c + row_tok : p_last;

    // ------------------------------------------------ setup: TMEM, barriers
    if (warp == 0) tmem_alloc(smem_addr(tmem_holder), kTmemCols);
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_pv, 1);
        mbar_init(bar_kv, 1);
        mbar_init(bar_kv + 1, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t tmem_s = tmem;        // S: columns 0..kBN - 1
    const uint32_t tmem_o = tmem + 128;  // O: columns 128..128 + D - 1
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float *red = reinterpret_cast<float *>(sm + L::kRed);  // [2][2][kRows]
    const uint32_t sq = base + L::kQ;
    auto kbuf = [&](int j) { return base + L::kK0 + static_cast<uint32_t>(j & 1) * L::kBufStride; };
    auto sbuf = [&](int j) { return reinterpret_cast<float *>(sm + L::kScales) + (j & 1) * 2 * kBN; };
    auto vbuf = [&](int j) { return base + L::kV0 + static_cast<uint32_t>(j & 1) * L::kBufStride; };

    // S = Q K_j^T, issued by thread 0 once tile j's K is in shared memory
    auto issue_s = [&](int j) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = static_cast<uint32_t>((kk >> 2) * kRows * 128 + (kk & 3) * 32);
            const uint32_t boff = static_cast<uint32_t>((kk >> 2) * kBN * 128 + (kk & 3) * 32);
            mma_bf16(tmem_s, sw128_desc(sq + aoff, 16, 1024), sw128_desc(kbuf(j) + boff, 16, 1024), kIdescS,
                     kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s);
    };

    // Q rows (zero past the chunk) and the first KV tiles
    {
        constexpr int kChunks = D / 8;
        const __nv_bfloat16 *qp = static_cast<const __nv_bfloat16 *>(a.q);
        for (int i = tid; i < kRows * kChunks; i += kThreads) {
            const int r = i / kChunks, c16 = i % kChunks;
            const int tok = t0 + r / G;
            const bool valid = tok < c;
            const int64_t elem = (static_cast<int64_t>(q0 + (valid ? tok : 0)) * nq + kh * G + r % G) * D + c16 * 8;
            cp_async16(sq + swz(kRows, r, c16), qp + elem, valid ? 16u : 0u);
        }
    }
    if constexpr (FP8) {
        load_kv_tile<D, FP8, TS>(a, table, kh, 0, kv_end, log2_bs, kbuf(0), vbuf(0), sbuf(0));
    } else if (tid == 0) {
        tma_kv_tile<D>(&map_k, &map_v, table, a.num_kv_heads, kh, a.block_size, log2_bs, 0, kv_end, kbuf(0), vbuf(0),
                       bar_kv);
        if (n_tiles > 1)
            tma_kv_tile<D>(&map_k, &map_v, table, a.num_kv_heads, kh, a.block_size, log2_bs, 1, kv_end, kbuf(1),
                           vbuf(1), bar_kv + 1);
    }
    cp_async_commit();
    cp_async_wait0();
    fence_proxy_async_smem();
    __syncthreads();
    bool timed_out = false;
    uint64_t *pending = nullptr;  // the barrier a timed-out wait was on
    uint32_t pending_parity = 0;
    if (tid == 0) {
        if (FP8 || mbar_wait(bar_kv, 0)) issue_s(0);
    }

    const float sl2 = a.scale * kLog2e * ((FP8 && !TS) ? __ldg(a.k_scale + kh) : 1.0f);
    float m_run = -INFINITY, l_run = 0.0f;

    for (int j = 0; j < n_tiles; ++j) {
        const uint32_t sk = kbuf(j), sv = vbuf(j);
        const uint32_t sp = L::kPInK ? sk : base + L::kP;  // P replaces this tile's K once S is computed

        // this thread's half of the row's scores (exp2 domain, causal mask) and its maximum
        const bool ok_s = mbar_wait(bar_s, static_cast<uint32_t>(j & 1));
        const int kv0 = j * kBN;
        const int col0 = half * kHalfCols;  // first score column of this thread
        const bool masked = kv0 + kBN - 1 > p_first;  // some row sees a future or absent token
        const float *tsc = sbuf(j);  // this tile's per-token scales (TS)
        float x[kHalfCols];
        float mx = -INFINITY;
        if (ok_s) {
            tc_fence_after();
            float v[32];
            tmem_ld32(tmem_s + lane_base + col0, v);
#pragma unroll
            for (int i = 0; i < kHalfCols; ++i) x[i] = TS ? v[i] * (sl2 * tsc[col0 + i]) : v[i] * sl2;
            if (masked) {
#pragma unroll
                for (int i = 0; i < kHalfCols; ++i)
                    if (kv0 + col0 + i > row_pos) x[i] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
            for (int i = 8; i < kHalfCols; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
            mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            red[((j & 1) * 2 + half) * kRows + row] = mx;
        }
        if (__syncthreads_or(!ok_s)) {
            timed_out = true;
            pending = bar_s;
            pending_parity = static_cast<uint32_t>(j & 1);
            break;
        }
        mx = fmaxf(mx, red[((j & 1) * 2 + (half ^ 1)) * kRows + row]);  // the row's maximum

        // P V of the previous tile has finished: P, O and the other buffer are free
        if (j > 0) {
            const bool ok_pv = mbar_wait(bar_pv, static_cast<uint32_t>((j - 1) & 1));
            if (__syncthreads_or(!ok_pv)) {
                timed_out = true;
                pending = bar_pv;
                pending_parity = static_cast<uint32_t>((j - 1) & 1);
                break;
            }
            tc_fence_after();
        }
        if (j + 1 < n_tiles) {
            if constexpr (FP8) {
                load_kv_tile<D, FP8, TS>(a, table, kh, j + 1, kv_end, log2_bs, kbuf(j + 1), vbuf(j + 1), sbuf(j + 1));
            } else if (tid == 0 && j + 1 >= 2) {  // tiles 0 and 1 were issued up front
                tma_kv_tile<D>(&map_k, &map_v, table, a.num_kv_heads, kh, a.block_size, log2_bs, j + 1, kv_end,
                               kbuf(j + 1), vbuf(j + 1), bar_kv + ((j + 1) & 1));
            }
        }

        // Lazy rescale: the reference maximum moves only when the tile's
        // maximum exceeds it by more than 8 (weights stay below 2^8); the
        // final O / l is the same for any reference.
        if (j == 0) {
            m_run = mx;  // O is written, not accumulated, by the first P V
        } else {
            const bool grow = mx > m_run + 8.0f;
            if (__any_sync(0xffffffffu, grow)) {  // tcgen05.ld/st are warp-wide
                const float alpha = grow ? fast_exp2(m_run - mx) : 1.0f;
                if (grow) {
                    m_run = mx;
                    l_run *= alpha;
                }
#pragma unroll
                for (int ch = 0; ch < D / 64; ++ch) {  // this thread's half of the row's O columns
                    float v[32];
                    tmem_ld32(tmem_o + lane_base + half * (D / 2) + ch * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(tmem_o + lane_base + half * (D / 2) + ch * 32, v);
                }
            }
        }

        // P = exp2(s - m) as bf16 into shared memory; l sums the rounded weights
        // (masked scores are -inf, so their weights are exactly 0)
        float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < kHalfCols / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int i0 = c * 8 + 2 * h;
                w[h] = pack_bf16(fast_exp2(x[i0] - m_run), fast_exp2(x[i0 + 1] - m_run));
                l4[h] += bf16lo(w[h]) + bf16hi(w[h]);
            }
            st_shared16(sp + swz(kRows, row, col0 / 8 + c), make_uint4(w[0], w[1], w[2], w[3]));
        }
        l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);

        if constexpr (!FP8) {
            const int valid_rows = kv_end - kv0;
            if (valid_rows < kBN && mbar_wait(bar_kv + (j & 1), static_cast<uint32_t>((j >> 1) & 1))) {
                // rows past the causal end: zero V so that 0-weight x stale data stays 0
                constexpr int kHalves = D / 64;
                const int n16 = (kBN - valid_rows) * 8;  // 16-byte chunks per half
                for (int i = tid; i < kHalves * n16; i += kThreads) {
                    const int h = i / n16, r = valid_rows + (i % n16) / 8, cc = i % 8;
                    st_shared16(sv + h * kBN * 128 + r * 128 + cc * 16, make_uint4(0, 0, 0, 0));
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();

        // O += P V_j, then S_{j+1} right behind it on the tensor core
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
                const uint32_t aoff = static_cast<uint32_t>((kk >> 2) * kRows * 128 + (kk & 3) * 32);
                mma_bf16(tmem_o, sw128_desc(sp + aoff, 16, 1024),
                         sw128_desc(sv + static_cast<uint32_t>(kk * 16 * 128), kBN * 128, 1024), kIdescPV,
                         (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar_pv);
            if (j + 1 < n_tiles) {
                if (FP8 || mbar_wait(bar_kv + ((j + 1) & 1), static_cast<uint32_t>(((j + 1) >> 1) & 1)))
                    issue_s(j + 1);
            }
        }
    }

    if (!timed_out) {
        const bool ok = mbar_wait(bar_pv, static_cast<uint32_t>((n_tiles - 1) & 1));
        if (__syncthreads_or(!ok)) {
            timed_out = true;
            pending = bar_pv;
            pending_parity = static_cast<uint32_t>((n_tiles - 1) & 1);
        }
    }
    cp_async_wait0();
    if (timed_out) {
        // one more bounded wait for the MMAs in flight before TMEM is freed
        if (tid == 0) {
            set_error(a.dev_err, PKV_DEVERR_TIMEOUT);
            mbar_wait(pending, pending_parity);
        }
    } else {
        tc_fence_after();
        // the row's normaliser: this thread's partial sum plus its partner's
        float *lred = red + 2 * 2 * kRows;  // past the max exchange buffers ([2][kRows] floats)
        lred[half * kRows + row] = l_run;
        __syncthreads();
        const float l_row = l_run + lred[(half ^ 1) * kRows + row];
        const float inv = ((FP8 && !TS) ? __ldg(a.v_scale + kh) : 1.0f) / l_row;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
            float v[32];
            tmem_ld32(tmem_o + lane_base + half * (D / 2) + ch * 32, v);  // warp-wide: every lane loads
            if (row_live) {
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 w = make_uint4(pack_bf16(v[i] * inv, v[i + 1] * inv), pack_bf16(v[i + 2] * inv, v[i + 3] * inv),
                                         pack_bf16(v[i + 4] * inv, v[i + 5] * inv),
                                         pack_bf16(v[i + 6] * inv, v[i + 7] * inv));
                    *reinterpret_cast<uint4 *>(out_row + ch * 32 + i) = w;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, int G, bool FP8, bool TS>
cudaError_t launch_t(const PrefillArgs &a, cudaStream_t stream) {
    constexpr int TQ = kRows / G;
    const int tiles = (a.max_q_len + TQ - 1) / TQ;
    const long long nx = static_cast<long long>(a.num_seqs) * tiles;
    if (nx > 0x7FFFFFFFLL || a.num_kv_heads > 65535) return cudaErrorInvalidConfiguration;
    int log2_bs = 0;
    while ((1 << log2_bs) < a.block_size) ++log2_bs;
    CUtensorMap mk, mv;
    memset(&mk, 0, sizeof(mk));
    memset(&mv, 0, sizeof(mv));
    if (!FP8) {
        // TMA row coordinates are int32
        if (static_cast<long long>(a.num_blocks) * a.num_kv_heads * a.block_size > 0x7FFFFFFFLL)
            return cudaErrorInvalidConfiguration;
        if (!make_pool_map(&mk, a.k_cache, a, kBN) || !make_pool_map(&mv, a.v_cache, a, kBN)) return cudaErrorInvalidValue;
    }
    auto kern = paged_prefill_kernel<D, G, FP8, TS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Layout<D>::kAlloc));
    if (e != cudaSuccess) return e;
    kern<<<dim3(static_cast<unsigned>(nx), a.num_kv_heads), kThreads, Layout<D>::kAlloc, stream>>>(a, tiles, log2_bs,
                                                                                                 mk, mv);
    return cudaGetLastError();
}

template <int D, bool FP8, bool TS = false>
cudaError_t launch_d(const PrefillArgs &a, int g, cudaStream_t stream) {
    switch (g) {
        case 1: return launch_t<D, 1, FP8, TS>(a, stream);
        case 2: return launch_t<D, 2, FP8, TS>(a, stream);
        case 4: return launch_t<D, 4, FP8, TS>(a, stream);
        case 8: return launch_t<D, 8, FP8, TS>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_supported(int head_dim, int group) {
    return (head_dim == 64 || head_dim == 128) && (group == 1 || group == 2 || group == 4 || group == 8);
}

namespace {

// The warp-specialised kernel for the chunks longer than one query tile
// (128 / G tokens); nothing when there are none.
cudaError_t launch_long_chunks(const PrefillArgs &a, int g, cudaStream_t stream) {
    if (a.max_q_len <= kRows / g) return cudaSuccess;
    PrefillArgs large = a;
    large.small_cut = kRows / g;
    return launch_prefill_ws(large, stream);
}

// The one-tile kernel for chunks of 2 .. 128 / G tokens.
cudaError_t launch_short_chunks(const PrefillArgs &a, int g, cudaStream_t stream) {
    PrefillArgs small = a;
    small.small_cut = kRows / g;
    small.small_min = 2;
    small.max_q_len = a.max_q_len < small.small_cut ? a.max_q_len : small.small_cut;
    if (a.fp8 && a.token_scales)
        return a.head_dim == 128 ? launch_d<128, true, true>(small, g, stream)
                                 : launch_d<64, true, true>(small, g, stream);
    if (a.head_dim == 128) return a.fp8 ? launch_d<128, true>(small, g, stream) : launch_d<128, false>(small, g, stream);
    return a.fp8 ? launch_d<64, true>(small, g, stream) : launch_d<64, false>(small, g, stream);
}

}  // namespace

// A low-priority stream per device, created on first use and kept for the
// process. The one-token chunks of a mixed prefill batch run on it, beside
// the chunk kernels, so that their blocks fill the SMs the few long-chunk
// blocks leave idle (the short chunks stay on the caller's stream: moved to
// the side stream they competed with the long chunks for the SMs and the
// batch took 5 % longer); so does the suffix decode of a bf16 cascade, beside
// the shared-prefix kernel (decode.cu). The caller's stream waits for it
// before anything queued later.
cudaStream_t library_side_stream() {
    constexpr int kMaxDevices = 64;
    static std::atomic<cudaStream_t> streams[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    cudaStream_t s = streams[dev].load(std::memory_order_acquire);
    if (s) return s;
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&s, cudaStreamNonBlocking, least) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    cudaStream_t expected = nullptr;
    if (!streams[dev].compare_exchange_strong(expected, s, std::memory_order_acq_rel)) {
        cudaStreamDestroy(s);  // another thread made one first
        return expected;
    }
    return s;
}

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream) {
    const int g = a.num_q_heads / a.num_kv_heads;
    // One-token chunks (decode requests in the batch) go to the decode
    // kernel, which streams their K/V at HBM speed instead of filling 1 / 128
    // of an MMA tile; chunks of more than one query tile (128 / G tokens) go
    // to the warp-specialised kernel (two tiles per CTA, one CTA per SM);
    // the rest to the one-tile kernel, which fits two CTAs per SM. Each
    // kernel skips the others' sequences.
    DecodeArgs d;
    d.q = a.q;
    d.k_cache = a.k_cache;
    d.v_cache = a.v_cache;
    d.block_tables = a.block_tables;
    d.max_blocks_per_seq = a.max_blocks_per_seq;
    d.context_lens = a.context_lens;
    d.seq_order = nullptr;
    d.num_seqs = a.num_seqs;
    d.num_q_heads = a.num_q_heads;
    d.num_kv_heads = a.num_kv_heads;
    d.head_dim = a.head_dim;
    d.block_size = a.block_size;
    d.num_blocks = a.num_blocks;
    d.scale = a.scale;
    d.fp8 = a.fp8;
    d.token_scales = a.token_scales;
    d.k_scale = a.k_scale;
    d.v_scale = a.v_scale;
    d.max_context_len = a.max_blocks_per_seq * a.block_size;  // the table's capacity
    d.partition_tokens = 0;                                   // no split: nothing to allocate
    d.num_partitions = 1;
    d.part_o = nullptr;
    d.part_ml = nullptr;
    d.out = a.out;
    d.dev_err = a.dev_err;
    d.cu_q_lens = a.cu_q_lens;
    d.total_q = a.total_q;
    if (a.max_q_len <= 1) return launch_decode(d, stream);  // decode requests only
    cudaStream_t side = library_side_stream();
    cudaEvent_t fork = nullptr, join = nullptr;
    if (!side || cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();  // no side stream: everything on the caller's stream
        if (fork) cudaEventDestroy(fork);
        cudaError_t e = launch_long_chunks(a, g, stream);
        if (e == cudaSuccess) e = launch_decode(d, stream);
        return e != cudaSuccess ? e : launch_short_chunks(a, g, stream);
    }
    cudaError_t e = cudaEventRecord(fork, stream);
    if (e == cudaSuccess) e = launch_long_chunks(a, g, stream);  // first: its few blocks start first
    if (e == cudaSuccess) e = launch_short_chunks(a, g, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e == cudaSuccess) e = launch_decode(d, side);
    // join even after a failure, so that nothing later on the caller's stream
    // overtakes work already queued on the side stream
    cudaError_t e2 = cudaEventRecord(join, side);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(stream, join, 0);
    cudaEventDestroy(fork);  // released once the waits are resolved
    cudaEventDestroy(join);
    return e != cudaSuccess ? e : e2;
}

}  // namespace pkv
