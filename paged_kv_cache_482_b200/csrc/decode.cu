// decode.cu -- instantiations and launch of the paged decode kernels: the
// warp-MMA kernels (decode_mma.cuh) at head_dim 128, the CUDA-core kernel
// (decode.cuh) at head_dim 64.
//
// Tile shape: four warps, each taking up to four 32-lane steps of a tile;
// stages hold K and V of one tile and the ring is about 48 KB deep, so that
// four blocks share an SM with well over 100 KB of loads in flight.
#include <atomic>
#include <cstring>

#include "decode.cuh"
#include "decode_mma.cuh"

namespace pkv {

namespace {

unsigned reduce_blocks(const DecodeParams &p) {
    return (unsigned)(((long long)p.num_seqs * p.num_q_heads + kReduceWarps - 1) / kReduceWarps);
}

template <int D, int G, bool FP8, bool TS>
cudaError_t launch_one(const DecodeParams &p, cudaStream_t stream) {
    using T = DecodeTraits<D, G, FP8>;
#ifdef PKV_DECODE_MIN_BLOCKS
    constexpr int MINB = PKV_DECODE_MIN_BLOCKS;
#else
    constexpr int MINB = (G <= 4) ? 4 : 2;  // 4 x 128 threads at 128 registers fill the register file
#endif
    auto kern = paged_decode_kernel<D, G, FP8, MINB, TS>;

    // The opt-in to more than 48 KB of dynamic shared memory is a property of
    // the function on a device; set it once per device.
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long blocks = (long long)p.num_seqs * p.num_kv_heads * p.num_partitions;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, T::kThreads, T::kSmemBytes, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.num_partitions <= 1) return e;
    paged_decode_reduce_kernel<D><<<reduce_blocks(p), 32 * kReduceWarps, 0, stream>>>(p);
    return cudaGetLastError();
}

// head_dim 128: the warp-MMA kernel (decode_mma.cuh), every cache type.
// tc_prefix: the shared prefixes of a cascade are attended elsewhere (on the
// tensor cores, launch_prefix_tc); otherwise the prefix kernel below does it.
// merge: launch the split-K merge after the decode kernel (when one is
// needed); false when the caller launches it (launch_merge) itself.
template <int G, bool BF, bool TS>
cudaError_t launch_mma_one(const DecodeParams &p, cudaStream_t stream, bool tc_prefix, bool merge) {
    using T = MmaTraits<G, BF>;
#ifdef PKV_MMA_MIN_BLOCKS
    constexpr int MINB = PKV_MMA_MIN_BLOCKS;
#else
    constexpr int MINB = 3;
#endif
    auto kern = paged_decode_mma_kernel<G, BF, MINB, TS>;
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kAlloc);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long blocks = (long long)p.num_seqs * p.num_kv_heads * p.grid_partitions;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // tensor-map row coordinates are int32
    const long long rows = p.num_blocks * p.num_kv_heads * p.block_size;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const int box_rows = p.block_size < 16 ? p.block_size : 16;
    CUtensorMap mk, mv;
    std::memset(&mk, 0, sizeof(mk));
    std::memset(&mv, 0, sizeof(mv));
    const bool mapped = BF ? make_bf16_pool_map(&mk, p.k_cache, rows, box_rows) &&
                                 make_bf16_pool_map(&mv, p.v_cache, rows, box_rows)
                           : make_e4m3_pool_map(&mk, p.k_cache, rows, box_rows) &&
                                 make_e4m3_pool_map(&mv, p.v_cache, rows, box_rows);
    if (!mapped) return cudaErrorInvalidValue;
    if (p.cu_group_seqs && !tc_prefix) {  // the shared prefixes first: slot 0 of every member
        using PT = PrefixTraits<BF>;
        auto pk = paged_prefix_mma_kernel<G, BF, TS>;
        static std::atomic<unsigned long long> configured_prefix{0};
        if (!(configured_prefix.load(std::memory_order_acquire) & bit)) {
            e = cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize, PT::kAlloc);
            if (e != cudaSuccess) return e;
            configured_prefix.fetch_or(bit, std::memory_order_acq_rel);
        }
        const int per_block = PT::kNW * (8 / G);
        const long long chunks = ((long long)p.max_group_seqs + per_block - 1) / per_block;
        const long long gx = chunks * p.num_groups;
        if (gx > 0x7fffffffLL || p.num_kv_heads > 65535) return cudaErrorInvalidConfiguration;
        if (gx > 0) {
            pk<<<dim3((unsigned)gx, (unsigned)p.num_kv_heads), PT::kThreads, PT::kAlloc, stream>>>(p, mk, mv, box_rows,
                                                                                                  (int)chunks);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    kern<<<(unsigned)blocks, T::kThreads, T::kAlloc, stream>>>(p, mk, mv, box_rows);
    e = cudaGetLastError();
    if (e != cudaSuccess || !merge || (p.num_partitions <= 1 && !p.cu_group_seqs)) return e;
    paged_decode_reduce_kernel<128><<<reduce_blocks(p), 32 * kReduceWarps, 0, stream>>>(p);
    return cudaGetLastError();
}

// The split-K merge of a head_dim-128 decode whose partials are all written.
cudaError_t launch_merge(const DecodeParams &p, cudaStream_t stream) {
    if (p.num_partitions <= 1 && !p.cu_group_seqs) return cudaSuccess;
    paged_decode_reduce_kernel<128><<<reduce_blocks(p), 32 * kReduceWarps, 0, stream>>>(p);
    return cudaGetLastError();
}

template <bool BF, bool TS>
cudaError_t launch_mma(int group, const DecodeParams &p, cudaStream_t stream, bool tc_prefix = false,
                       bool merge = true) {
    switch (group) {
        case 1: return launch_mma_one<1, BF, TS>(p, stream, tc_prefix, merge);
        case 2: return launch_mma_one<2, BF, TS>(p, stream, tc_prefix, merge);
        case 4: return launch_mma_one<4, BF, TS>(p, stream, tc_prefix, merge);
        case 8: return launch_mma_one<8, BF, TS>(p, stream, tc_prefix, merge);
        default: return cudaErrorInvalidValue;
    }
}

// bf16 cascade: the shared prefixes on the tensor cores, on the caller's
// stream and launched first (one CTA per SM, on far fewer SMs than there are
// at the sizes where prefixes are shared), beside the suffix decode on the
// library's low-priority side stream, which fills the other SMs; the merge
// runs on the caller's stream once both are done. Without a side stream,
// everything in order on the caller's stream.
cudaError_t launch_cascade_tc(int group, const DecodeArgs &a, const DecodeParams &p, cudaStream_t stream) {
    cudaStream_t side = library_side_stream();
    cudaEvent_t fork = nullptr, join = nullptr;
    if (!side || cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        if (fork) cudaEventDestroy(fork);
        const cudaError_t e = launch_prefix_tc(a, stream);
        return e != cudaSuccess ? e : launch_mma<true, false>(group, p, stream, true);
    }
    cudaError_t e = cudaEventRecord(fork, stream);
    if (e == cudaSuccess) e = launch_prefix_tc(a, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e == cudaSuccess) e = launch_mma<true, false>(group, p, side, true, false);
    // join even after a failure, so that nothing later on the caller's stream
    // overtakes work already queued on the side stream
    cudaError_t e2 = cudaEventRecord(join, side);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(stream, join, 0);
    cudaEventDestroy(fork);  // released once the waits are resolved
    cudaEventDestroy(join);
    if (e != cudaSuccess) return e;
    if (e2 != cudaSuccess) return e2;
    return launch_merge(p, stream);
}

template <bool BF>
int mma_tile_of(int group) {
    switch (group) {
        case 1: return MmaTraits<1, BF>::kTile;
        case 2: return MmaTraits<2, BF>::kTile;
        case 4: return MmaTraits<4, BF>::kTile;
        case 8: return MmaTraits<8, BF>::kTile;
        default: return 0;
    }
}

template <int D, bool FP8>
int tile_of(int group) {
    switch (group) {
        case 1: return DecodeTraits<D, 1, FP8>::kTile;
        case 2: return DecodeTraits<D, 2, FP8>::kTile;
        case 4: return DecodeTraits<D, 4, FP8>::kTile;
        case 8: return DecodeTraits<D, 8, FP8>::kTile;
        default: return 0;
    }
}

template <int D, bool FP8, bool TS = false>
cudaError_t launch_group(int group, const DecodeParams &p, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_one<D, 1, FP8, TS>(p, stream);
        case 2: return launch_one<D, 2, FP8, TS>(p, stream);
        case 4: return launch_one<D, 4, FP8, TS>(p, stream);
        case 8: return launch_one<D, 8, FP8, TS>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int decode_tile_tokens(int head_dim, int group, bool fp8) {
    if (head_dim == 128) return fp8 ? mma_tile_of<false>(group) : mma_tile_of<true>(group);
    if (head_dim == 64) return fp8 ? tile_of<64, true>(group) : tile_of<64, false>(group);
    return 0;
}

int decode_max_blocks_per_partition() { return kMaxIdsPerPartition; }

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    DecodeParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k_cache = static_cast<const uint8_t *>(a.k_cache);
    p.v_cache = static_cast<const uint8_t *>(a.v_cache);
    p.block_tables = a.block_tables;
    p.max_blocks_per_seq = a.max_blocks_per_seq;
    p.context_lens = a.context_lens;
    p.seq_order = a.seq_order;
    p.num_seqs = a.num_seqs;
    p.num_q_heads = a.num_q_heads;
    p.num_kv_heads = a.num_kv_heads;
    p.block_size = a.block_size;
    int lg = 0;
    while ((1 << lg) < a.block_size) ++lg;
    p.log2_block_size = lg;
    p.num_blocks = a.num_blocks;
    p.qk_scale_log2 = a.scale * 1.4426950408889634f;  // log2(e)
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.max_context_len = a.max_context_len;
    p.partition_tokens = a.partition_tokens > 0 ? a.partition_tokens : a.max_context_len;
    p.num_partitions = a.partition_tokens > 0 ? a.num_partitions : 1;
    if (a.cu_group_seqs) {  // slot 0 holds the shared prefix; the grid covers the suffix partitions
        if (a.head_dim != 128) return cudaErrorInvalidValue;
        p.num_partitions = a.num_partitions;
    }
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.dev_err = a.dev_err;
    p.cu_q_lens = a.cu_q_lens;
    p.total_q = a.total_q;
    p.cu_group_seqs = a.cu_group_seqs;
    p.group_prefix = a.group_prefix;
    p.num_groups = a.num_groups;
    p.max_group_seqs = a.max_group_seqs;
    p.grid_partitions = a.cu_group_seqs ? p.num_partitions - 1 : p.num_partitions;
    const int group = a.num_q_heads / a.num_kv_heads;
    if (a.head_dim == 128) {
        if (!a.fp8) {
            if (a.cu_group_seqs && prefix_tc_supported(a.head_dim, group, false))
                return launch_cascade_tc(group, a, p, stream);  // bf16 cascade
            return launch_mma<true, false>(group, p, stream);
        }
        return a.token_scales ? launch_mma<false, true>(group, p, stream) : launch_mma<false, false>(group, p, stream);
    }
    if (a.head_dim == 64) {  // the CUDA-core kernel (decode.cuh)
        if (a.fp8 && a.token_scales) return launch_group<64, true, true>(group, p, stream);
        return a.fp8 ? launch_group<64, true>(group, p, stream) : launch_group<64, false>(group, p, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
