// prefill_ws.cu -- chunked-prefill paged attention (bf16 or E4M3 cache, one
// scale per KV head or per token), warp-specialised on the 5th-generation
// tensor cores (sm_100a).
//
// Same operation as prefill.cu ("nano-vllm-lite：深入理解LLM推理机制的教育级开源
// 项目", section 核心技术改进 2 "Chunked Prefill"; paged cache of "DeepSeek复刻
// vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战"): token i of a chunk
// of c new tokens (position p = ctx - c + i) attends over positions 0..p.
//
// One CTA per (sequence, KV head, two query tiles of 128 rows each; a row is
// a (chunk token, query head of the group) pair), one CTA per SM. Warp roles:
//   warps 0-3  softmax of query tile A (one row per thread);
//   warps 4-7  softmax of query tile B;
//   warp 8     bf16: producer, tensor-map copies of 128-token K/V tiles into
//              a two-stage ring (and the zeroing of V rows past the causal
//              end on the last tile). E4M3: one of three converter warps
//              (8, 10, 11) that load the codes, widen them to f16 and store
//              them into the ring;
//   warp 9     tensor-memory allocation and the MMA issue:
//                S_A(0), S_B(0), then per tile j
//                PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), ...
//              so that the tensor core works on one query tile while the
//              other tile's softmax runs, and both share every K/V tile.
// The 128-token KV tile makes S an M = N = 128 MMA: per unit of work it
// reads half as much shared memory for the Q operand as N = 64 does, which
// is what paced the tensor pipe with 64-token tiles.
// Tensor memory (512 columns): S_A, S_B (128 columns each) and O_A, O_B
// (128 columns each). P (two 16-bit values per 32-bit column) is written over
// the first 64 columns of the S it came from and P V takes its A operand from
// tensor memory, so P never touches shared memory. S of tile j + 1 reuses
// the columns of P of tile j: it is issued after P V of tile j by the same
// thread, and MMAs from one thread run in issue order. The commit of S(j+1)
// therefore also covers P V(j): a softmax thread that sees S(j+1) may
// rescale O without waiting for anything else.
// A softmax thread takes its row's 128 scores from tensor memory in one
// statement (two loads and their wait), and rescales O only after P is out of
// its registers (168 registers a thread: 320 or 384 threads, one CTA per SM).
// Operand types: bf16 for a bf16 cache. For E4M3, f16: every E4M3 value is
// an f16 value (one conversion per two codes), Q is scaled per row by a power
// of two into f16 range (exact for bf16 input), and P is packed as f16. With
// per-token scales, the converters also stage the tile's K scales, scores are
// scaled by column, and V is dequantised as it is widened (each code times its
// row's scale in fp32, rounded to bf16), so P V runs in bf16 and P needs no
// scaling: the weights are rounded to bf16 and the normaliser sums the
// rounded weights, as for a bf16 cache.
// With a workspace (E4M3 only), a widening kernel first expands the codes of
// the sequences with long chunks once into dense 16-bit rows (K f16; V f16,
// or bf16 with per-token scales; the per-token scales as fp32 rows), one
// run of rows per (sequence, KV head), zeros past the context; warp 8 is then
// a tensor-map producer as for a bf16 cache (one copy per 64-column half of a
// 128-token tile, plus two 512-byte copies of the tile's scales), and no CTA
// widens anything. The operands the MMAs see are the same 16-bit values, so
// the result is the same as with the converter warps.
// Everything between roles goes through mbarriers (full / empty K/V stages,
// S ready, P ready, O done); every wait is bounded (1 s) and reports
// PKV_DEVERR_TIMEOUT. The softmax uses the same arithmetic as prefill.cu:
// exp2 domain, lazy rescale of O in tensor memory (the reference maximum
// moves only when a tile's maximum exceeds it by more than 8), P rounded to
// the operand type and the normaliser summing the rounded weights.
#include "tc_common.cuh"

namespace pkv {
namespace {

using namespace tc;

constexpr int kRowsT = 128;  // rows per query tile (MMA M)
constexpr int kBN = 128;     // KV tokens per tile
constexpr int kStages = 2;   // K/V ring depth
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8;  // bf16: tensor-map producer; E4M3: converter
constexpr int kMmaWarp = 9;
constexpr int kConvWarps = 3;     // E4M3 converters: warps 8, 10, 11
// bf16: softmax + producer + MMA warps; E4M3: softmax + three converters + MMA
template <bool FP8>
constexpr int ws_threads() { return FP8 ? kSoftmaxThreads + 32 * (kConvWarps + 1) : kSoftmaxThreads + 64; }
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct WsLayout {
    static constexpr int kHalves = D / 64;
    static constexpr uint32_t kQTile = kHalves * kRowsT * 128;  // one query tile
    static constexpr uint32_t kKV = kHalves * kBN * 128;        // one K (or V) tile
    static constexpr uint32_t kQ = 0;                           // Q_A, Q_B
    static constexpr uint32_t kRing = kQ + 2 * kQTile;          // stage s: K at kRing + s * 2 kKV, V after it
    static constexpr uint32_t kBar = kRing + kStages * 2 * kKV;
    static constexpr uint32_t kTable = kBar + 256;
    static constexpr uint32_t kScales = kTable + kTableCap * 4;  // per-token E4M3: [stage][K, V][kBN] fp32
    static constexpr uint32_t kBytes = kScales + kStages * 2 * kBN * 4;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

struct Bars {
    uint64_t kv_full[kStages];   // stage written (MMA warp; softmax too, for per-token scales)
    uint64_t kv_empty[kStages];  // P V_B of the stage's tile done: the stage may be refilled
    uint64_t s_full[2];     // [query tile]
    uint64_t p_full[2];     // [query tile]: P of a tile written
    uint64_t o_done[2];     // [query tile]: P V of a tile done
    uint64_t q_full;
    uint64_t vtail;
    uint64_t drained;
    uint32_t tmem;
};

// Producer: stage KV tile j (logical tokens j * kBN ..) into ring stage (sk, sv).
template <int D>
__device__ __forceinline__ void ws_kv_tile(const CUtensorMap *mk, const CUtensorMap *mv, const BlockIds &table,
                                           int nkv, int kh, int bs, int log2_bs, int j, int kv_end, uint32_t sk,
                                           uint32_t sv, uint64_t *bar) {
    constexpr int kHalves = D / 64;
    const int kv0 = j * kBN;
    if (bs >= kBN) {
        const int row = (table[kv0 >> log2_bs] * nkv + kh) * bs + (kv0 & (bs - 1));
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
            const int row = (table[(kv0 >> log2_bs) + i] * nkv + kh) * bs;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
                tma_load_2d(sk + h * kBN * 128 + i * bs * 128, mk, h * 64, row, bar);
                tma_load_2d(sv + h * kBN * 128 + i * bs * 128, mv, h * 64, row, bar);
            }
        }
    }
}

// Dense staging of E4M3 K/V (workspace layout): rows of D 16-bit values,
// row (s * num_kv_heads + kv head) * staging_stride + position; K rows, then V
// rows, then (per-token scales) the K scales as fp32, one per row (V is
// staged dequantised, so its scales are not needed).
struct Staging {
    uint16_t *k;
    uint16_t *v;
    float *k_scale;
};

template <int D>
__host__ __device__ __forceinline__ Staging staging_of(const PrefillArgs &a) {
    const long long rows = static_cast<long long>(a.num_seqs) * a.num_kv_heads * a.staging_stride;
    Staging st;
    st.k = static_cast<uint16_t *>(a.staging);
    st.v = st.k + rows * D;
    st.k_scale = reinterpret_cast<float *>(st.v + rows * D);
    return st;
}

// Widening of the E4M3 K/V codes into the staging rows, one unit = 128 rows
// of one (sequence, KV head), for the sequences whose chunks the
// warp-specialised kernel takes (longer than small_cut). Rows past the
// context are written as zeros; units wholly past it are never read and are
// skipped. Sequences the attention kernel will reject (bad cu_q_lens or
// lengths) are skipped; a block id outside the pool gives zero rows (the
// attention kernel reports it).
constexpr int kWidenThreads = 256;

template <int D, bool TS>
__global__ void __launch_bounds__(kWidenThreads) widen_kv_kernel(PrefillArgs a, int log2_bs, long long units) {
    constexpr int kCPR = D / 16;  // 16-code chunks per row
    const int tiles = a.staging_stride / kBN;
    const Staging st = staging_of<D>(a);
    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
        const int tile = static_cast<int>(u % tiles);
        const long long sk = u / tiles;  // s * num_kv_heads + kv head
        const int kh = static_cast<int>(sk % a.num_kv_heads);
        const int s = static_cast<int>(sk / a.num_kv_heads);
        const int q0 = a.cu_q_lens[s], q1 = a.cu_q_lens[s + 1];
        if (q0 < 0 || q1 < q0 || q1 > a.total_q) continue;
        const int c = q1 - q0;
        if (c <= a.small_cut || c > a.max_q_len) continue;
        const int ctx = a.context_lens[s];
        if (ctx < c || static_cast<long long>(ctx) > static_cast<long long>(a.max_blocks_per_seq) * a.block_size)
            continue;
        const int t0 = tile * kBN;
        if (t0 >= ctx) continue;
        const int32_t *table = a.block_tables + static_cast<long long>(s) * a.max_blocks_per_seq;
        const long long drow0 = sk * a.staging_stride + t0;
        // kIt chunks per thread: every block id, then every code load, then
        // the conversions and stores, so that a thread's loads are in flight
        // together
        constexpr int kIt = kBN * kCPR / kWidenThreads;
        int r[kIt];
        long long prow[kIt];
#pragma unroll
        for (int u = 0; u < kIt; ++u) {
            const int i = threadIdx.x + u * kWidenThreads;
            r[u] = i / kCPR;
            const int t = t0 + r[u];
            prow[u] = -1;
            if (t < ctx) {
                const int b = __ldg(table + (t >> log2_bs));
                if (b >= 0 && b < a.num_blocks)
                    prow[u] = (static_cast<long long>(b) * a.num_kv_heads + kh) * a.block_size + (t & (a.block_size - 1));
            }
        }
        const int cc = threadIdx.x % kCPR;  // the same 16-code column in every chunk of this thread
        uint4 kc[kIt], vc[kIt];
        float vs[kIt];
#pragma unroll
        for (int u = 0; u < kIt; ++u) {
            kc[u] = make_uint4(0, 0, 0, 0);
            vc[u] = kc[u];
            vs[u] = 0.0f;
            if (prow[u] >= 0) {
                kc[u] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.k_cache) + prow[u] * D +
                                                            cc * 16));
                vc[u] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.v_cache) + prow[u] * D +
                                                            cc * 16));
                if constexpr (TS) vs[u] = __ldg(a.v_scale + prow[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kIt; ++u) {
            uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0, v0 = k0, v1 = k0;
            if (prow[u] >= 0) {  // zeros past the context (and for a bad block id)
                const uint2 h0 = e4m3x4_to_f16x4(kc[u].x), h1 = e4m3x4_to_f16x4(kc[u].y);
                const uint2 h2 = e4m3x4_to_f16x4(kc[u].z), h3 = e4m3x4_to_f16x4(kc[u].w);
                k0 = make_uint4(h0.x, h0.y, h1.x, h1.y);
                k1 = make_uint4(h2.x, h2.y, h3.x, h3.y);
                if constexpr (TS) {  // per-token scales: V dequantised (bf16 of code x scale), P V in bf16
                    v0 = e4m3x8_scaled_bf16x8(make_uint2(vc[u].x, vc[u].y), vs[u]);
                    v1 = e4m3x8_scaled_bf16x8(make_uint2(vc[u].z, vc[u].w), vs[u]);
                } else {
                    const uint2 g0 = e4m3x4_to_f16x4(vc[u].x), g1 = e4m3x4_to_f16x4(vc[u].y);
                    const uint2 g2 = e4m3x4_to_f16x4(vc[u].z), g3 = e4m3x4_to_f16x4(vc[u].w);
                    v0 = make_uint4(g0.x, g0.y, g1.x, g1.y);
                    v1 = make_uint4(g2.x, g2.y, g3.x, g3.y);
                }
            }
            uint4 *kd = reinterpret_cast<uint4 *>(st.k + (drow0 + r[u]) * D + cc * 16);
            uint4 *vd = reinterpret_cast<uint4 *>(st.v + (drow0 + r[u]) * D + cc * 16);
            kd[0] = k0;
            kd[1] = k1;
            vd[0] = v0;
            vd[1] = v1;
        }
        if constexpr (TS) {
            for (int rr = threadIdx.x; rr < kBN; rr += blockDim.x) {
                const int t = t0 + rr;
                float ks = 0.0f;
                if (t < ctx) {
                    const int b = __ldg(table + (t >> log2_bs));
                    if (b >= 0 && b < a.num_blocks) {
                        const long long prow = (static_cast<long long>(b) * a.num_kv_heads + kh) * a.block_size +
                                               (t & (a.block_size - 1));
                        ks = __ldg(a.k_scale + prow);
                    }
                }
                st.k_scale[drow0 + rr] = ks;
            }
        }
    }
}

// STG (E4M3 only): K/V tiles come from the staging rows by tensor-map copies
// (map_k / map_v cover the staging instead of the pools); otherwise E4M3
// codes are widened by the converter warps.
// PFX (bf16 cache, shared-prefix decode): a unit is a group of sequences
// that share their first group_prefix[s] cached tokens, its rows are
// (member, query head) pairs (member i's query is q row cu_group_seqs[s] + i),
// the keys are the shared tokens, read through the first member's table, with
// no causal mask, and each row's result is its split-K slot-0 partial
// (normalised O, maximum, sum) for the merge -- the product of the members'
// queries with the shared keys is a dense contraction, run here on the
// tensor cores instead of once per member.
template <int D, int G, bool FP8, bool TS, bool STG, bool PFX>
__global__ void __launch_bounds__(ws_threads<FP8 && !STG>(), 1)
    paged_prefill_ws_kernel(PrefillArgs a, int tiles_per_seq, int log2_bs, const __grid_constant__ CUtensorMap map_k,
                            const __grid_constant__ CUtensorMap map_v) {
    constexpr bool CONV = FP8 && !STG;  // converter warps widen the codes
    using L = WsLayout<D>;
    constexpr int TQ = kRowsT / G;  // chunk tokens per query tile
    // bf16 cache: bf16 operands. E4M3 cache: f16 operands for S (one conversion
    // per two codes; Q is scaled into f16 range per row, see the staging below)
    // and for P V with one scale per KV head. With one scale per token, V is
    // dequantised to bf16 (code times its row's scale), which may leave f16
    // range: P V then runs in bf16 (P and V both bf16).
    constexpr uint32_t kIdescS = FP8 ? idesc_f16(kRowsT, kBN, false) : idesc_bf16(kRowsT, kBN, false);
    constexpr uint32_t kIdescPV = (FP8 && !TS) ? idesc_f16(kRowsT, D, true) : idesc_bf16(kRowsT, D, true);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    Bars *bars = reinterpret_cast<Bars *>(sm + L::kBar);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    // query-tile-major over the sequences (groups): the last (longest causal
    // range) tiles of every sequence are scheduled first
    const int units = PFX ? a.num_groups : a.num_seqs;
    const int s = blockIdx.x % units;
    const int tile = tiles_per_seq - 1 - blockIdx.x / units;
    const int kh = blockIdx.y;
    const int nq = a.num_q_heads;

    // ------------------------------------------------ bounds and bookkeeping
    // rows: the chunk's tokens, or (PFX) the group's members
    const int q0 = PFX ? a.cu_group_seqs[s] : a.cu_q_lens[s];
    const int q1 = PFX ? a.cu_group_seqs[s + 1] : a.cu_q_lens[s + 1];
    if (q0 < 0 || q1 < q0 || q1 > (PFX ? a.num_seqs : a.total_q)) {
        if (tid == 0 && tile == 0 && kh == 0) set_error(a.dev_err, PKV_DEVERR_BOUNDS);
        return;
    }
    const int c = q1 - q0;
    const int t0 = tile * 2 * TQ;  // first chunk token (member) of query tile A
    if (t0 >= c) return;
    if (!PFX && c <= a.small_cut) return;  // a short chunk: the one-tile kernel's
    const int P = PFX ? a.group_prefix[s] : 0;
    if (PFX && P == 0) return;  // nothing shared: the decode kernel attends every token
    const long long cap = static_cast<long long>(a.max_blocks_per_seq) * a.block_size;
    // keys 0 .. ctx - 1: the sequence's context, or the group's shared tokens
    const int ctx = PFX ? P : a.context_lens[s];
    const int32_t *table_g = a.block_tables + static_cast<int64_t>(PFX ? q0 : s) * a.max_blocks_per_seq;
    int32_t *table_s = reinterpret_cast<int32_t *>(sm + L::kTable);
    bool bad = PFX ? (P < 0 || (P & (a.block_size - 1)) != 0 || P > cap)
                   : (ctx < c || static_cast<int64_t>(ctx) > cap || c > a.max_q_len);
    if (!bad) {
        const int nblk_seq = (ctx + a.block_size - 1) >> log2_bs;
        for (int i = tid; i < nblk_seq; i += ws_threads<CONV>()) {
            const int32_t b = table_g[i];
            if (b < 0 || b >= a.num_blocks) bad = true;
            if (i < kTableCap) table_s[i] = b;
        }
    }
    const BlockIds table{table_s, table_g};
    // PFX: a member whose context is shorter than the shared tokens, or whose
    // table does not start with the first member's blocks, gets an empty
    // partial (sum 0: the merge writes zeros) and PKV_DEVERR_BOUNDS; one flag
    // per member of this unit, in the (unused) scale slots
    uint8_t *mflag = sm + L::kScales;
    if constexpr (PFX) {
        const int nm = min(c - t0, 2 * TQ);
        const int nblk = bad ? 0 : P >> log2_bs;
        for (int m = warp; m < nm; m += ws_threads<CONV>() / 32) {
            const int seq = q0 + t0 + m;
            const int cm = __ldg(a.context_lens + seq);
            bool bm = cm < P || cm > a.max_context_len || cm > cap;
            const int32_t *mrow = a.block_tables + static_cast<int64_t>(seq) * a.max_blocks_per_seq;
            for (int i = lane; i < nblk; i += 32) bm |= __ldg(mrow + i) != __ldg(table_g + i);
            bm = __any_sync(0xffffffffu, bm);
            if (lane == 0) mflag[m] = bm ? 1 : 0;
        }
    }

    // softmax threads: query tile X, row r of it
    const int X = (warp >> 2) & 1;
    const int row = tid & (kRowsT - 1);
    const int row_tok = t0 + X * TQ + row / G;
    const bool row_live = warp < 8 && row_tok < c;
    __nv_bfloat16 *out_row = PFX ? nullptr
                                 : static_cast<__nv_bfloat16 *>(a.out) +
                                       (static_cast<int64_t>(q0 + (row_live ? row_tok : 0)) * nq + kh * G + row % G) * D;
    // PFX: this row's slot-0 partial
    const long long pslot =
        PFX ? (static_cast<long long>(q0 + (row_live ? row_tok : 0)) * nq + kh * G + row % G) * a.num_partitions : 0;
    if (__syncthreads_or(bad)) {
        if (row_live) {
            if constexpr (PFX) {
                a.part_ml[pslot * 2] = -INFINITY;
                a.part_ml[pslot * 2 + 1] = 0.0f;
            } else {
                for (int i = 0; i < D; i += 8) *reinterpret_cast<uint4 *>(out_row + i) = make_uint4(0, 0, 0, 0);
            }
        }
        if (tid == 0) set_error(a.dev_err, PKV_DEVERR_BOUNDS);
        return;
    }
    if constexpr (PFX) {
        bool any = false;
        for (int m = tid; m < min(c - t0, 2 * TQ); m += ws_threads<CONV>()) any |= mflag[m] != 0;
        if (any) set_error(a.dev_err, PKV_DEVERR_BOUNDS);
    }
    const int last_tok = min(t0 + 2 * TQ, c) - 1;
    const int p_last = PFX ? P - 1 : ctx - c + last_tok;
    const int kv_end = p_last + 1;
    const int n_tiles = (kv_end + kBN - 1) / kBN;

    // ------------------------------------------------ setup
    if (warp == kMmaWarp) tmem_alloc(smem_addr(&bars->tmem), kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->kv_full[i], CONV ? kConvWarps : 1);
            mbar_init(&bars->kv_empty[i], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_full[x], kRowsT / 32);  // one arrive per softmax warp
            mbar_init(&bars->o_done[x], 1);
        }
        mbar_init(&bars->q_full, kSoftmaxThreads);
        mbar_init(&bars->vtail, 1);
        mbar_init(&bars->drained, 1);
        fence_barrier_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem;
    auto kbuf = [&](int j) { return base + L::kRing + static_cast<uint32_t>(j % kStages) * 2 * L::kKV; };
    auto vbuf = [&](int j) { return kbuf(j) + L::kKV; };
    const uint32_t sq0 = base + L::kQ;

    if (warp < 8) {
        // ================================================ softmax, query tile X
        const uint32_t sq = sq0 + X * L::kQTile;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tmem_s = tmem + X * kBN;  // S (and P over its first 64 columns)
        const uint32_t tmem_o = tmem + 256 + X * 128;
        // E4M3 with one scale per KV head: k_scale folds into the softmax scale
        float sl2 = a.scale * kLog2e * ((FP8 && !TS) ? __ldg(a.k_scale + kh) : 1.0f);
        {
            constexpr int kChunks = D / 8;
            const __nv_bfloat16 *qp = static_cast<const __nv_bfloat16 *>(a.q);
            if constexpr (!FP8) {
                for (int i = row; i < kRowsT * kChunks; i += kRowsT) {
                    const int r = i / kChunks, c16 = i % kChunks;
                    const int tok = t0 + X * TQ + r / G;
                    const bool valid = tok < c;
                    const int64_t elem =
                        (static_cast<int64_t>(q0 + (valid ? tok : 0)) * nq + kh * G + r % G) * D + c16 * 8;
                    cp_async16(sq + swz(kRowsT, r, c16), qp + elem, valid ? 16u : 0u);
                }
                cp_async_commit();
                cp_async_wait0();
            } else {
                // This thread's own row, times 2^kq with kq chosen so that the row's
                // largest |q| lies in [2^14, 2^15): exact in f16 (a bf16 value has 8
                // significant bits) down to 2^-31 of the row maximum. 2^-kq folds
                // into the row's softmax scale. kq >= -114 (|q| < 2^129, infinities
                // included); it is capped at 60 so that 2^-kq times the softmax
                // scale stays a normal float: rows so small that the cap binds
                // have scores below 2^-45 times the key norms, whose softmax is
                // uniform either way.
                const uint4 *qrow = reinterpret_cast<const uint4 *>(
                    qp + (static_cast<int64_t>(q0 + (row_live ? row_tok : 0)) * nq + kh * G + row % G) * D);
                uint4 qv[kChunks];
                float amax = 0.0f;
#pragma unroll
                for (int c16 = 0; c16 < kChunks; ++c16) {
                    qv[c16] = row_live ? __ldg(qrow + c16) : make_uint4(0, 0, 0, 0);
                    const uint32_t wds[4] = {qv[c16].x, qv[c16].y, qv[c16].z, qv[c16].w};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        amax = fmaxf(amax, fmaxf(fabsf(bf16lo(wds[k])), fabsf(bf16hi(wds[k]))));
                }
                const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 126;  // amax < 2^e
                const int kq = min(60, 15 - e);
                const float qs = __int_as_float((kq + 127) << 23);
                sl2 *= __int_as_float((127 - kq) << 23);
#pragma unroll
                for (int c16 = 0; c16 < kChunks; ++c16) {
                    const uint32_t wds[4] = {qv[c16].x, qv[c16].y, qv[c16].z, qv[c16].w};
                    uint32_t h[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) h[k] = pack_f16(bf16lo(wds[k]) * qs, bf16hi(wds[k]) * qs);
                    st_shared16(sq + swz(kRowsT, row, c16), make_uint4(h[0], h[1], h[2], h[3]));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->q_full);
        }
        // position of this tile's first row, and of this row (PFX: every row
        // sees all the shared tokens)
        const int p_first = PFX ? P - 1 : ctx - c + t0 + X * TQ;
        const int row_pos = PFX ? P - 1 : (row_live ? ctx - c + row_tok : p_last);
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            // S_X(j) done implies P V_X(j - 1) done (issued before it): O_X is stable
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[X], static_cast<uint32_t>(j & 1)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int kv0 = j * kBN;
            const bool masked = kv0 + kBN - 1 > p_first;
            // the row's 128 scores (one statement: two loads and their wait)
            float x[kBN];
            tmem_ld128(tmem_s + lane_base, x);
            const float *tsc = reinterpret_cast<const float *>(sm + L::kScales) + (j % kStages) * 2 * kBN;
            if constexpr (TS) {
                // the tile's per-token K scales were staged with its codes: x = s *
                // k_scale of the column (the row's sl2 enters below, as without
                // per-token scales). The stage is refilled only after both query
                // tiles have released this tile, so this wait cannot see a later phase.
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->kv_full[j % kStages],
                                                       static_cast<uint32_t>((j / kStages) & 1)))) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int i = 0; i < kBN / 2; ++i) {
                    const float2 k2 = *reinterpret_cast<const float2 *>(tsc + 2 * i);
                    const float2 v2 = __fmul2_rn(make_float2(x[2 * i], x[2 * i + 1]), k2);
                    x[2 * i] = v2.x;
                    x[2 * i + 1] = v2.y;
                }
            }
            if (masked) {
#pragma unroll
                for (int i = 0; i < kBN; ++i)
                    if (kv0 + i > row_pos) x[i] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = x[k];
#pragma unroll
            for (int i = 8; i < kBN; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
            const float mx = sl2 * fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                         fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            float alpha = 1.0f;
            bool rescale = false;
            if (j == 0) {
                m_run = mx;
            } else {
                const bool grow = mx > m_run + 8.0f;
                rescale = __any_sync(0xffffffffu, grow);
                if (grow) {
                    alpha = fast_exp2(m_run - mx);
                    m_run = mx;
                    l_run *= alpha;
                }
            }
            // P as 16-bit pairs (bf16, or f16 for E4M3 with per-head scales) over
            // columns 0..63 of S: scores 64 hh .. 64 hh + 63 go to columns
            // 32 hh .. 32 hh + 31 (all scores are in registers)
            const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_run, -m_run);
            float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float pw[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float2 t = __ffma2_rn(make_float2(x[hh * 64 + 2 * i], x[hh * 64 + 2 * i + 1]), sl2x2, nm2);
                    uint32_t w;
                    if constexpr (FP8 && !TS) {  // P in f16 (the E4M3 path's operand type)
                        w = pack_f16(fast_exp2(t.x), fast_exp2(t.y));
                        l4[i & 3] = fma_f16x2_acc(w, 0x3C003C00u, l4[i & 3]);
                    } else {
                        w = pack_bf16(fast_exp2(t.x), fast_exp2(t.y));
                        l4[i & 3] = fma_bf16x2_acc(w, 0x3F803F80u, l4[i & 3]);
                    }
                    pw[i] = __uint_as_float(w);
                }
                tmem_st32_async(tmem_s + lane_base + hh * 32, pw);
            }
            l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            // O rescale once the scores are out of the registers; P V of this
            // tile is issued only after the arrive below
            if (rescale) {
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    float v[32];
                    tmem_ld32(tmem_o + lane_base + ch * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32_async(tmem_o + lane_base + ch * 32, v);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[X]);
        }
        if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_done[X], 0))) {
            tc_fence_after();
            const float inv = ((FP8 && !TS) ? __ldg(a.v_scale + kh) : 1.0f) / l_run;
            if constexpr (PFX) {  // the slot-0 partial: O / l, then (maximum, sum)
                const bool bm = row_live && mflag[row_tok - t0] != 0;
                float *dst = a.part_o + pslot * D;
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    float v[32];
                    tmem_ld32(tmem_o + lane_base + ch * 32, v);
                    if (row_live) {
                        const float w = bm ? 0.0f : inv;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(dst + ch * 32 + i) =
                                make_float4(v[i] * w, v[i + 1] * w, v[i + 2] * w, v[i + 3] * w);
                    }
                }
                if (row_live) {
                    a.part_ml[pslot * 2] = bm ? -INFINITY : m_run;
                    a.part_ml[pslot * 2 + 1] = bm ? 0.0f : l_run;
                }
            }
#pragma unroll
            for (int ch = 0; ch < (PFX ? 0 : D / 32); ++ch) {
                float v[32];
                tmem_ld32(tmem_o + lane_base + ch * 32, v);
                if (row_live) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 w = make_uint4(pack_bf16(v[i] * inv, v[i + 1] * inv),
                                             pack_bf16(v[i + 2] * inv, v[i + 3] * inv),
                                             pack_bf16(v[i + 4] * inv, v[i + 5] * inv),
                                             pack_bf16(v[i + 6] * inv, v[i + 7] * inv));
                        *reinterpret_cast<uint4 *>(out_row + ch * 32 + i) = w;
                    }
                }
            }
        } else {
            if (row == 0) set_error(a.dev_err, PKV_DEVERR_TIMEOUT);
            if (PFX && row_live) {  // an empty partial: the merge writes zeros
                a.part_ml[pslot * 2] = -INFINITY;
                a.part_ml[pslot * 2 + 1] = 0.0f;
            }
        }
        __syncwarp();
    } else if (!CONV && warp == kProducerWarp) {
        // ================================================ producer (bf16 pools, or E4M3 staging rows)
        int issued = 0;
        if (lane == 0) {
            const int srow0 = (s * a.num_kv_heads + kh) * a.staging_stride;  // staging: int32 (host-checked)
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % kStages, use = j / kStages;
                if (use > 0 && !mbar_wait(&bars->kv_empty[st], static_cast<uint32_t>((use - 1) & 1))) {
                    set_error(a.dev_err, PKV_DEVERR_TIMEOUT);
                    break;
                }
                if constexpr (STG) {
                    uint64_t *bar = &bars->kv_full[st];
                    const int row = srow0 + j * kBN;
                    mbar_arrive_expect_tx(bar, 2u * (D / 64) * kBN * 128u + (TS ? kBN * 4u : 0u));
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        tma_load_2d(kbuf(j) + h * kBN * 128, &map_k, h * 64, row, bar);
                        tma_load_2d(vbuf(j) + h * kBN * 128, &map_v, h * 64, row, bar);
                    }
                    if constexpr (TS) {
                        const Staging sg = staging_of<D>(a);
                        float *tsc = reinterpret_cast<float *>(sm + L::kScales) + st * 2 * kBN;
                        bulk_g2s(tsc, sg.k_scale + row, kBN * 4, bar);  // V came dequantised
                    }
                } else {
                    ws_kv_tile<D>(&map_k, &map_v, table, a.num_kv_heads, kh, a.block_size, log2_bs, j, kv_end,
                                  kbuf(j), vbuf(j), &bars->kv_full[st]);
                }
                issued = j + 1;
            }
        }
        issued = __shfl_sync(0xffffffffu, issued, 0);
        // V rows past the causal end on the last tile (bf16 pools): zero them,
        // so that a zero weight times stale pool data stays zero. The staging
        // rows past the context are zeros already, and the rows between the
        // causal end and the context hold cached values (finite for finite
        // data), so a zero weight gives zero there too.
        const int last = n_tiles - 1;
        const int valid_rows = kv_end - last * kBN;
        bool tail_ok = issued == n_tiles;
        if (!STG && tail_ok && valid_rows < kBN) {
            tail_ok = mbar_wait(&bars->kv_full[last % kStages], static_cast<uint32_t>((last / kStages) & 1));
            if (tail_ok) {
                constexpr int kHalves = D / 64;
                const int n16 = (kBN - valid_rows) * 8;
                for (int i = lane; i < kHalves * n16; i += 32) {
                    const int h = i / n16, r = valid_rows + (i % n16) / 8, cc = i % 8;
                    st_shared16(vbuf(last) + h * kBN * 128 + r * 128 + cc * 16, make_uint4(0, 0, 0, 0));
                }
                fence_proxy_async_smem();
            }
        }
        __syncwarp();
        if (lane == 0) {
            if (tail_ok) mbar_arrive(&bars->vtail);
            // copies still in flight (only after a timeout): wait for them before the CTA exits
            for (int j = max(0, issued - kStages); j < issued; ++j)
                mbar_wait(&bars->kv_full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
        }
        __syncwarp();
    } else if (CONV && warp != kMmaWarp) {
        // ================================================ E4M3 converters (warps 8, 10, 11)
        // Each thread loads 16-code chunks of the tile's K and V rows, widens
        // them exactly to f16 and stores them into the swizzled stage the
        // MMAs read; rows past the causal end are written as zeros. The next
        // tile's loads are in flight while the thread waits for its stage.
        constexpr int kCW = kConvWarps * 32;
        constexpr int kCPR = D / 16;                  // 16-code chunks per row
        constexpr int kHalf = kBN * kCPR;             // chunks of one operand's tile
        constexpr int kPer = (kHalf + kCW - 1) / kCW;  // per thread and operand
        const int ct = (warp == kProducerWarp ? 0 : warp - kMmaWarp) * 32 + lane;
        uint4 wk[kPer], wv[kPer];
        // scl (V with per-token scales): also each chunk's row scale
        auto load = [&](uint4 (&w)[kPer], const void *pool, int j, float *scl) {
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int idx = ct + u * kCW;
                const int t = j * kBN + idx / kCPR;
                w[u] = make_uint4(0, 0, 0, 0);
                if (scl) scl[u] = 0.0f;
                if (idx < kHalf && t < kv_end) {
                    const int64_t row = (static_cast<int64_t>(table[t >> log2_bs]) * a.num_kv_heads + kh) *
                                            a.block_size + (t & (a.block_size - 1));
                    w[u] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(pool) + row * D +
                                                               (idx % kCPR) * 16));
                    if (scl) scl[u] = __ldg(a.v_scale + row);
                }
            }
        };
        // scl: V with per-token scales, dequantised to bf16 (code x scale)
        auto store = [&](const uint4 (&w)[kPer], uint32_t dst, const float *scl) {
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int idx = ct + u * kCW;
                if (idx < kHalf) {
                    const int r = idx / kCPR, c16 = 2 * (idx % kCPR);
                    if (scl) {
                        st_shared16(dst + swz(kBN, r, c16), e4m3x8_scaled_bf16x8(make_uint2(w[u].x, w[u].y), scl[u]));
                        st_shared16(dst + swz(kBN, r, c16 + 1),
                                    e4m3x8_scaled_bf16x8(make_uint2(w[u].z, w[u].w), scl[u]));
                    } else {
                        const uint2 h0 = e4m3x4_to_f16x4(w[u].x), h1 = e4m3x4_to_f16x4(w[u].y);
                        const uint2 h2 = e4m3x4_to_f16x4(w[u].z), h3 = e4m3x4_to_f16x4(w[u].w);
                        st_shared16(dst + swz(kBN, r, c16), make_uint4(h0.x, h0.y, h1.x, h1.y));
                        st_shared16(dst + swz(kBN, r, c16 + 1), make_uint4(h2.x, h2.y, h3.x, h3.y));
                    }
                }
            }
            fence_proxy_async_smem();  // the tensor core reads these through the async proxy
            __syncwarp();
        };
        // per-token scales of a tile (TS): K at [0, kBN), V at [kBN, 2 kBN), 0 past the end
        constexpr int kSPer = (2 * kBN + kCW - 1) / kCW;
        float sc[kSPer];
        auto load_scales = [&](int j) {
#pragma unroll
            for (int u = 0; u < kSPer; ++u) {
                const int i = ct + u * kCW;
                const int t = j * kBN + (i % kBN);
                sc[u] = 0.0f;
                if (TS && i < 2 * kBN && t < kv_end)
                    sc[u] = __ldg((i < kBN ? a.k_scale : a.v_scale) +
                                  (static_cast<int64_t>(table[t >> log2_bs]) * a.num_kv_heads + kh) * a.block_size +
                                  (t & (a.block_size - 1)));
            }
        };
        auto store_scales = [&](int j) {
            float *dst = reinterpret_cast<float *>(sm + L::kScales) + (j % kStages) * 2 * kBN;
#pragma unroll
            for (int u = 0; u < kSPer; ++u) {
                const int i = ct + u * kCW;
                if (i < 2 * kBN) dst[i] = sc[u];
            }
        };
        float vsc[kPer];  // per-token scales: the V rows' scales of this thread's chunks
        float *vs_ptr = TS ? vsc : nullptr;
        bool ok = true;
        load(wk, a.k_cache, 0, nullptr);
        load(wv, a.v_cache, 0, vs_ptr);
        if (TS) load_scales(0);
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % kStages, use = j / kStages;
            if (use > 0 &&
                !__all_sync(0xffffffffu, mbar_wait(&bars->kv_empty[st], static_cast<uint32_t>((use - 1) & 1)))) {
                ok = false;
                break;
            }
            // K of tile j, then the next tile's K codes load while V is widened
            // (to bf16 with per-token scales, where P V runs in bf16)
            if (TS) store_scales(j);
            store(wk, kbuf(j), nullptr);
            if (j + 1 < n_tiles) load(wk, a.k_cache, j + 1, nullptr);
            store(wv, vbuf(j), vs_ptr);
            if (lane == 0) mbar_arrive(&bars->kv_full[st]);
            if (j + 1 < n_tiles) {
                load(wv, a.v_cache, j + 1, vs_ptr);
                if (TS) load_scales(j + 1);
            }
        }
        if (!ok && lane == 0) set_error(a.dev_err, PKV_DEVERR_TIMEOUT);
        __syncwarp();
    } else {
        // ================================================ MMA issue
        if (lane == 0) {
            bool ok = mbar_wait(&bars->q_full, 0);
            auto issue_s = [&](int x, int j) {
                const uint32_t sq = sq0 + x * L::kQTile, sk = kbuf(j);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t aoff = static_cast<uint32_t>((kk >> 2) * kRowsT * 128 + (kk & 3) * 32);
                    const uint32_t boff = static_cast<uint32_t>((kk >> 2) * kBN * 128 + (kk & 3) * 32);
                    mma_bf16(tmem + x * kBN, sw128_desc(sq + aoff, 16, 1024), sw128_desc(sk + boff, 16, 1024),
                             kIdescS, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[x]);
            };
            auto issue_pv = [&](int x, int j, bool last) {  // A = P_x(j) over the first 64 columns of S_x
                const uint32_t tp = tmem + x * kBN, sv = vbuf(j);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_bf16_ts(tmem + 256 + x * 128, tp + kk * 8,
                                sw128_desc(sv + static_cast<uint32_t>(kk * 16 * 128), kBN * 128, 1024), kIdescPV,
                                (j > 0 || kk > 0) ? 1u : 0u);
                if (last) mma_commit(&bars->o_done[x]);
            };
            auto kv_ready = [&](int j) {
                const bool r = mbar_wait(&bars->kv_full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
                tc_fence_after();
                return r;
            };
            ok = ok && kv_ready(0);
            if (ok) {
                issue_s(0, 0);
                issue_s(1, 0);
            }
            // per tile j: P V_A(j), S_A(j + 1), P V_B(j), S_B(j + 1); K/V of tile
            // j + 1 is awaited only after P V_A(j) is on the tensor pipe
            for (int j = 0; ok && j < n_tiles; ++j) {
                const bool more = j + 1 < n_tiles;
                if (!FP8 && !more) ok = mbar_wait(&bars->vtail, 0);  // E4M3: converters or staging zero the tail
                for (int x = 0; x < 2 && ok; ++x) {
                    if (!mbar_wait(&bars->p_full[x], static_cast<uint32_t>(j & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(x, j, !more);
                    if (x == 1) mma_commit(&bars->kv_empty[j % kStages]);
                    if (more) {
                        if (x == 0 && !kv_ready(j + 1)) {
                            ok = false;
                            break;
                        }
                        issue_s(x, j + 1);  // after P V_x(j): S_x is free
                    }
                }
            }
            if (!ok) set_error(a.dev_err, PKV_DEVERR_TIMEOUT);
            // every MMA issued so far has finished before tensor memory is freed
            mma_commit(&bars->drained);
            mbar_wait(&bars->drained, 0);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The staging rows as a 2-D tensor of 16-bit elements: boxes of 64 columns x
// 128 rows, 128-byte swizzle (the layout the converters write).
inline bool make_staging_map(CUtensorMap *map, const void *base, long long rows, int head_dim) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kBN)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, bool FP8, bool TS>
cudaError_t launch_ws(const PrefillArgs &a, cudaStream_t stream) {
    constexpr int TQ = kRowsT / G;
    const int tiles = (a.max_q_len + 2 * TQ - 1) / (2 * TQ);
    const long long nx = static_cast<long long>(a.num_seqs) * tiles;
    if (nx > 0x7FFFFFFFLL || a.num_kv_heads > 65535) return cudaErrorInvalidConfiguration;
    if (static_cast<long long>(a.num_blocks) * a.num_kv_heads * a.block_size > 0x7FFFFFFFLL)
        return cudaErrorInvalidConfiguration;  // tensor-map row coordinates are int32
    int log2_bs = 0;
    while ((1 << log2_bs) < a.block_size) ++log2_bs;
    CUtensorMap mk, mv;
    memset(&mk, 0, sizeof(mk));
    memset(&mv, 0, sizeof(mv));
    const dim3 grid(static_cast<unsigned>(nx), a.num_kv_heads);
    if (FP8 && a.staging) {
        // widen once into the staging rows, then copy tiles from there
        const long long rows = static_cast<long long>(a.num_seqs) * a.num_kv_heads * a.staging_stride;
        if (rows > 0x7FFFFFFFLL || a.staging_stride % kBN != 0) return cudaErrorInvalidConfiguration;
        const Staging st = staging_of<D>(a);
        if (!make_staging_map(&mk, st.k, rows, D) || !make_staging_map(&mv, st.v, rows, D))
            return cudaErrorInvalidValue;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cudaGetLastError();
        const long long units = rows / kBN;
        const long long wblocks = units < 16LL * sms ? units : 16LL * sms;
        widen_kv_kernel<D, TS><<<static_cast<unsigned>(wblocks), kWidenThreads, 0, stream>>>(a, log2_bs, units);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        auto kern = paged_prefill_ws_kernel<D, G, true, TS, true, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(WsLayout<D>::kAlloc));
        if (e != cudaSuccess) return e;
        kern<<<grid, ws_threads<false>(), WsLayout<D>::kAlloc, stream>>>(a, tiles, log2_bs, mk, mv);
        return cudaGetLastError();
    }
    // the E4M3 path without staging loads the codes with plain loads: no tensor maps
    if (!FP8 && (!make_pool_map(&mk, a.k_cache, a, kBN) || !make_pool_map(&mv, a.v_cache, a, kBN)))
        return cudaErrorInvalidValue;
    auto kern = paged_prefill_ws_kernel<D, G, FP8, TS, false, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(WsLayout<D>::kAlloc));
    if (e != cudaSuccess) return e;
    kern<<<grid, ws_threads<FP8>(), WsLayout<D>::kAlloc, stream>>>(a, tiles, log2_bs, mk, mv);
    return cudaGetLastError();
}

template <int D, bool FP8, bool TS>
cudaError_t launch_ws_g(const PrefillArgs &a, int g, cudaStream_t stream) {
    switch (g) {
        case 1: return launch_ws<D, 1, FP8, TS>(a, stream);
        case 2: return launch_ws<D, 2, FP8, TS>(a, stream);
        case 4: return launch_ws<D, 4, FP8, TS>(a, stream);
        case 8: return launch_ws<D, 8, FP8, TS>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

namespace {

template <int G>
cudaError_t launch_prefix_g(const PrefillArgs &a, cudaStream_t stream) {
    constexpr int TQ = kRowsT / G;
    const int tiles = (a.max_q_len + 2 * TQ - 1) / (2 * TQ);
    const long long nx = static_cast<long long>(a.num_groups) * tiles;
    if (nx <= 0) return cudaSuccess;
    if (nx > 0x7FFFFFFFLL || a.num_kv_heads > 65535) return cudaErrorInvalidConfiguration;
    if (static_cast<long long>(a.num_blocks) * a.num_kv_heads * a.block_size > 0x7FFFFFFFLL)
        return cudaErrorInvalidConfiguration;  // tensor-map row coordinates are int32
    int log2_bs = 0;
    while ((1 << log2_bs) < a.block_size) ++log2_bs;
    CUtensorMap mk, mv;
    memset(&mk, 0, sizeof(mk));
    memset(&mv, 0, sizeof(mv));
    if (!make_pool_map(&mk, a.k_cache, a, kBN) || !make_pool_map(&mv, a.v_cache, a, kBN)) return cudaErrorInvalidValue;
    auto kern = paged_prefill_ws_kernel<128, G, false, false, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(WsLayout<128>::kAlloc));
    if (e != cudaSuccess) return e;
    kern<<<dim3(static_cast<unsigned>(nx), a.num_kv_heads), ws_threads<false>(), WsLayout<128>::kAlloc, stream>>>(
        a, tiles, log2_bs, mk, mv);
    return cudaGetLastError();
}

}  // namespace

bool prefix_tc_supported(int head_dim, int group, bool fp8) {
    return head_dim == 128 && !fp8 && (group == 1 || group == 2 || group == 4 || group == 8);
}

cudaError_t launch_prefix_tc(const DecodeArgs &d, cudaStream_t stream) {
    const int g = d.num_q_heads / d.num_kv_heads;
    if (!d.cu_group_seqs || !prefix_tc_supported(d.head_dim, g, d.fp8)) return cudaErrorInvalidValue;
    PrefillArgs a;
    a.q = d.q;
    a.k_cache = d.k_cache;
    a.v_cache = d.v_cache;
    a.block_tables = d.block_tables;
    a.max_blocks_per_seq = d.max_blocks_per_seq;
    a.cu_q_lens = nullptr;
    a.context_lens = d.context_lens;
    a.num_seqs = d.num_seqs;
    a.total_q = d.num_seqs;
    a.num_q_heads = d.num_q_heads;
    a.num_kv_heads = d.num_kv_heads;
    a.head_dim = d.head_dim;
    a.block_size = d.block_size;
    a.num_blocks = d.num_blocks;
    a.scale = d.scale;
    a.fp8 = false;
    a.token_scales = false;
    a.k_scale = nullptr;
    a.v_scale = nullptr;
    a.max_q_len = d.max_group_seqs;  // members per group: sizes the grid like a chunk length
    a.out = nullptr;
    a.dev_err = d.dev_err;
    a.small_cut = 0;
    a.cu_group_seqs = d.cu_group_seqs;
    a.group_prefix = d.group_prefix;
    a.num_groups = d.num_groups;
    a.max_context_len = d.max_context_len;
    a.part_o = d.part_o;
    a.part_ml = d.part_ml;
    a.num_partitions = d.num_partitions;
    switch (g) {
        case 1: return launch_prefix_g<1>(a, stream);
        case 2: return launch_prefix_g<2>(a, stream);
        case 4: return launch_prefix_g<4>(a, stream);
        default: return launch_prefix_g<8>(a, stream);
    }
}

int prefill_staging_stride(int max_blocks_per_seq, int block_size) {
    const long long cap = static_cast<long long>(max_blocks_per_seq) * block_size;
    const long long stride = (cap + kBN - 1) / kBN * kBN;
    return stride > 0x7FFFFFFFLL ? 0 : static_cast<int>(stride);
}

size_t prefill_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq, int block_size,
                               bool fp8, bool token_scales) {
    if (!fp8 || num_seqs < 1 || num_kv_heads < 1 || head_dim < 1 || max_blocks_per_seq < 1 || block_size < 1)
        return 0;
    const long long stride = prefill_staging_stride(max_blocks_per_seq, block_size);
    const long long rows = static_cast<long long>(num_seqs) * num_kv_heads * stride;
    if (stride == 0 || rows > 0x7FFFFFFFLL) return 0;
    return static_cast<size_t>(rows) * (4u * static_cast<size_t>(head_dim) + (token_scales ? 4u : 0u));
}

cudaError_t launch_prefill_ws(const PrefillArgs &a, cudaStream_t stream) {
    const int g = a.num_q_heads / a.num_kv_heads;
    if (a.head_dim == 128) {
        if (!a.fp8) return launch_ws_g<128, false, false>(a, g, stream);
        return a.token_scales ? launch_ws_g<128, true, true>(a, g, stream) : launch_ws_g<128, true, false>(a, g, stream);
    }
    if (a.head_dim == 64) {
        if (!a.fp8) return launch_ws_g<64, false, false>(a, g, stream);
        return a.token_scales ? launch_ws_g<64, true, true>(a, g, stream) : launch_ws_g<64, true, false>(a, g, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
