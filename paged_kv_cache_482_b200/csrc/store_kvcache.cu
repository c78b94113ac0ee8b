// store_kvcache.cu -- write the step's K/V rows into their pool slots.
//
// Each new token's K and V rows go to slot slot_mapping[t] of the paged pool
// (the block manager gives every request its blocks: "Nano-vLLM：轻量高效的大模型
// 推理框架", section 三.1 "块管理器"; the FP8 cache variant: "nano-vllm-lite",
// section 核心技术改进 3 "FP8 KV Cache量化"; with one scale per KV head, or one
// per (token, KV head) computed here from the row's largest magnitude and
// written to scale pools shaped like the cache without head_dim). One thread
// moves one 16-byte chunk
// (8 bf16 elements) of a (token, KV head) row for both K and V: coalesced
// 16-byte loads, and 16-byte (bf16) or 8-byte (E4M3) stores. All address
// arithmetic is 64-bit: pools exceed 2^31 elements.
#include "pkv_common.cuh"
#include "pkv_launch.h"

namespace pkv {

namespace {

struct StoreParams {
    const uint4 *k;
    const uint4 *v;
    void *k_cache;
    void *v_cache;
    const int32_t *slots;
    long long total_chunks;  // num_tokens * num_kv_heads * chunks_per_row
    int chunks_per_row;      // head_dim / 8
    int num_kv_heads;
    int block_size;
    long long pool_slots;  // num_blocks * block_size
    float *k_scale;  // [num_kv_heads] (per head) or scale pools [num_blocks][num_kv_heads][block_size]
    float *v_scale;
    int *dev_err;
};

// Largest |x| of 8 bf16 elements.
__device__ __forceinline__ float amax8(uint4 x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[j])), fabsf(bf16hi(w[j]))));
    return m;
}

// Per-token scale: the row's largest magnitude / 448 (one IEEE division), at
// least the smallest normal binary32 so that an all-zero row encodes as zeros.
__device__ __forceinline__ float token_scale(float amax) { return fmaxf(__fdiv_rn(amax, 448.0f), 1.17549435e-38f); }

__device__ __forceinline__ uint2 quantise8(uint4 x, float scale) {
    // E4M3 of x / scale for 8 bf16 elements: one IEEE fp32 division each, then
    // round-to-nearest-even with saturation to +-448 (CUDA's conversion).
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = __fdiv_rn(bf16lo(w[j]), scale);
        const float b = __fdiv_rn(bf16hi(w[j]), scale);
        const uint32_t ca = __nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
        const uint32_t cb = __nv_cvt_float_to_fp8(b, __NV_SATFINITE, __NV_E4M3);
        out[j >> 1] |= (ca | (cb << 8)) << ((j & 1) * 16);
    }
    return make_uint2(out[0], out[1]);
}

// MODE 0: bf16 copy; 1: E4M3, a scale per KV head; 2: E4M3, a scale per
// (token, KV head). In mode 2 the chunks_per_row lanes of one row (adjacent
// lanes: the row's chunks are consecutive in i, and chunks_per_row divides
// 32 and the grid stride) reduce the row's amax with width-limited shuffles.
template <int MODE>
__global__ void __launch_bounds__(256) store_kvcache_kernel(StoreParams p) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < p.total_chunks; i += stride) {
        const int chunk = (int)(i % p.chunks_per_row);
        const long long row = i / p.chunks_per_row;  // token * num_kv_heads + head
        const int head = (int)(row % p.num_kv_heads);
        const long long token = row / p.num_kv_heads;
        const long long slot = p.slots[token];
        if (slot < 0) continue;
        if (slot >= p.pool_slots) {
            set_error(p.dev_err, PKV_DEVERR_BOUNDS);
            continue;
        }
        const long long blk = slot / p.block_size;
        const long long off = slot - blk * p.block_size;
        // element index of (blk, head, off, chunk*8) in the HND pool
        const long long dst = ((blk * p.num_kv_heads + head) * p.block_size + off) * (p.chunks_per_row * 8LL) +
                              chunk * 8LL;
        const uint4 kx = __ldg(p.k + i);
        const uint4 vx = __ldg(p.v + i);
        if constexpr (MODE == 2) {
            const int cpr = p.chunks_per_row;
            const int lane = threadIdx.x & 31;
            const unsigned group = (cpr == 32 ? 0xffffffffu : ((1u << cpr) - 1u)) << (lane & ~(cpr - 1));
            float km = amax8(kx), vm = amax8(vx);
            for (int o = cpr >> 1; o > 0; o >>= 1) {
                km = fmaxf(km, __shfl_xor_sync(group, km, o, cpr));
                vm = fmaxf(vm, __shfl_xor_sync(group, vm, o, cpr));
            }
            const float ks = token_scale(km), vs = token_scale(vm);
            if (chunk == 0) {
                const long long sidx = (blk * p.num_kv_heads + head) * p.block_size + off;
                p.k_scale[sidx] = ks;
                p.v_scale[sidx] = vs;
            }
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.k_cache) + dst) = quantise8(kx, ks);
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.v_cache) + dst) = quantise8(vx, vs);
        } else if constexpr (MODE == 1) {
            const float ks = __ldg(p.k_scale + head);
            const float vs = __ldg(p.v_scale + head);
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.k_cache) + dst) = quantise8(kx, ks);
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.v_cache) + dst) = quantise8(vx, vs);
        } else {
            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.k_cache) + dst) = kx;
            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.v_cache) + dst) = vx;
        }
    }
}

}  // namespace

cudaError_t launch_store_kvcache(const void *k, const void *v, void *k_cache, void *v_cache,
                                 const int32_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                 int block_size, int64_t num_blocks, int mode, float *k_scale, float *v_scale,
                                 int *dev_err, int num_sms, cudaStream_t stream) {
    StoreParams p;
    p.k = static_cast<const uint4 *>(k);
    p.v = static_cast<const uint4 *>(v);
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.slots = slot_mapping;
    p.chunks_per_row = head_dim / 8;
    p.total_chunks = (long long)num_tokens * num_kv_heads * p.chunks_per_row;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.pool_slots = (long long)num_blocks * block_size;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.dev_err = dev_err;
    const int threads = 256;
    long long blocks = (p.total_chunks + threads - 1) / threads;
    const long long cap = (long long)num_sms * 16;  // grid-stride beyond 16 blocks per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (mode == 2)
        store_kvcache_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(p);
    else if (mode == 1)
        store_kvcache_kernel<1><<<(unsigned)blocks, threads, 0, stream>>>(p);
    else
        store_kvcache_kernel<0><<<(unsigned)blocks, threads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pkv
