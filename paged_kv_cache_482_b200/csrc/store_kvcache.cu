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

// ------------------------------------------------------------------ RoPE
//
// Rotary position embedding of q and k fused with the store (the rotation of
// the RoFormer paper, Su et al. 2021; the FP8 cache it feeds: "nano-vllm-lite",
// section 核心技术改进 3): pair i of a row at position m turns by the angle
// whose cosine and sine the caller's table holds at cos_sin[m][i] and
// cos_sin[m][d/2 + i]. Pairs are (i, i + d/2) (STYLE 0) or (2i, 2i + 1)
// (STYLE 1). In binary32, one rounding per step, then bf16 round-to-nearest:
//   x' = fma(-y, sin, x * cos),  y' = fma(x, sin, y * cos)
// (the bf16 bits are decided here, so the operation order is part of the
// contract). The rotated k is then stored exactly as store_kvcache stores a
// bf16 row; v is stored as is; q is written rotated to q_out.
//
// One thread handles 8 pairs of one (token, row) -- rows are the q heads,
// then the KV heads -- so a row takes d/16 adjacent lanes: two 16-byte loads
// and stores per tensor, and 2 x 32 bytes of the table.

struct RopeParams {
    const uint4 *q;  // may be null
    uint4 *q_out;
    const uint4 *k;
    const uint4 *v;
    void *k_cache;
    void *v_cache;
    const int32_t *slots;
    const int32_t *positions;
    const float *cos_sin;  // [max_position][head_dim]
    int max_position;
    long long total_units;  // num_tokens * rows * lanes_per_row
    int lanes_per_row;      // head_dim / 16
    int num_q_heads;        // 0 when q is null
    int num_kv_heads;
    int head_dim;
    int block_size;
    long long pool_slots;
    float *k_scale;
    float *v_scale;
    int *dev_err;
};

// 8 pairs: x holds the 8 first and y the 8 second elements (bf16), c/s the
// 8 cosines and sines; returns the rotated x', y' as bf16.
__device__ __forceinline__ void rotate8(uint4 &x, uint4 &y, const float (&c)[8], const float (&s)[8]) {
    uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float xa[2] = {bf16lo(xw[j]), bf16hi(xw[j])}, ya[2] = {bf16lo(yw[j]), bf16hi(yw[j])};
        float xo[2], yo[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float cc = c[2 * j + e], ss = s[2 * j + e];
            xo[e] = __fmaf_rn(-ya[e], ss, __fmul_rn(xa[e], cc));
            yo[e] = __fmaf_rn(xa[e], ss, __fmul_rn(ya[e], cc));
        }
        const __nv_bfloat162 xb = __floats2bfloat162_rn(xo[0], xo[1]);
        const __nv_bfloat162 yb = __floats2bfloat162_rn(yo[0], yo[1]);
        xw[j] = *reinterpret_cast<const uint32_t *>(&xb);
        yw[j] = *reinterpret_cast<const uint32_t *>(&yb);
    }
    x = make_uint4(xw[0], xw[1], xw[2], xw[3]);
    y = make_uint4(yw[0], yw[1], yw[2], yw[3]);
}

// Interleaved pairs: 16 consecutive elements (two 16-byte chunks a, b) ->
// the 8 first elements of the pairs (x) and the 8 second ones (y), and back.
__device__ __forceinline__ void deinterleave(const uint4 &a, const uint4 &b, uint4 &x, uint4 &y) {
    x = make_uint4(__byte_perm(a.x, a.y, 0x5410), __byte_perm(a.z, a.w, 0x5410), __byte_perm(b.x, b.y, 0x5410),
                   __byte_perm(b.z, b.w, 0x5410));
    y = make_uint4(__byte_perm(a.x, a.y, 0x7632), __byte_perm(a.z, a.w, 0x7632), __byte_perm(b.x, b.y, 0x7632),
                   __byte_perm(b.z, b.w, 0x7632));
}
__device__ __forceinline__ void interleave(const uint4 &x, const uint4 &y, uint4 &a, uint4 &b) {
    a = make_uint4(__byte_perm(x.x, y.x, 0x5410), __byte_perm(x.x, y.x, 0x7632), __byte_perm(x.y, y.y, 0x5410),
                   __byte_perm(x.y, y.y, 0x7632));
    b = make_uint4(__byte_perm(x.z, y.z, 0x5410), __byte_perm(x.z, y.z, 0x7632), __byte_perm(x.w, y.w, 0x5410),
                   __byte_perm(x.w, y.w, 0x7632));
}

// Five blocks of 256 threads per SM (at most 48 registers a thread, with
// 12-64 bytes of spill to L1 a thread): with the loads hoisted, the
// compiler's own choice (54-58 registers, four blocks) was up to 25 % slower
// on the E4M3 store.
#ifndef PKV_ROPE_MIN_BLOCKS
#define PKV_ROPE_MIN_BLOCKS 5
#endif

template <int MODE, int STYLE>
__global__ void __launch_bounds__(256, PKV_ROPE_MIN_BLOCKS) store_kvcache_rope_kernel(RopeParams p) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const int L = p.lanes_per_row;
    const int rows = p.num_q_heads + p.num_kv_heads;
    const int cpr = p.head_dim / 8;  // 16-byte chunks per row
    for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < p.total_units; u += stride) {
        const int c = (int)(u % L);
        const long long rowi = u / L;
        const int r = (int)(rowi % rows);
        const long long token = rowi / rows;
        // chunk indices of the two halves this lane handles
        const int ca = STYLE == 1 ? 2 * c : c;
        const int cb = STYLE == 1 ? 2 * c + 1 : c + L;
        // Every load that does not depend on the position or the slot is
        // issued before either is known (all of them are in bounds), so a
        // unit waits for two memory latencies (position, then its cos/sin
        // row) instead of three.
        const bool is_q = r < p.num_q_heads;
        const int head = r - p.num_q_heads;
        const int m = __ldg(p.positions + token);
        long long slot = 0;
        uint4 a, b, va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
        long long base;
        if (is_q) {
            base = (token * p.num_q_heads + r) * cpr;
            a = __ldg(p.q + base + ca);
            b = __ldg(p.q + base + cb);
        } else {
            slot = __ldg(p.slots + token);
            base = (token * p.num_kv_heads + head) * cpr;
            a = __ldg(p.k + base + ca);
            b = __ldg(p.k + base + cb);
            va = __ldg(p.v + base + ca);
            vb = __ldg(p.v + base + cb);
        }
        if (m < 0 || m >= p.max_position) {
            if (c == 0 && r == 0) set_error(p.dev_err, PKV_DEVERR_BOUNDS);
            continue;
        }
        const float4 *cs = reinterpret_cast<const float4 *>(p.cos_sin + (long long)m * p.head_dim + 8 * c);
        const float4 *sn = reinterpret_cast<const float4 *>(p.cos_sin + (long long)m * p.head_dim + p.head_dim / 2 +
                                                            8 * c);
        const float4 c0 = __ldg(cs), c1 = __ldg(cs + 1), s0 = __ldg(sn), s1 = __ldg(sn + 1);
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        if (!is_q) {
            if (slot < 0) continue;
            if (slot >= p.pool_slots) {
                set_error(p.dev_err, PKV_DEVERR_BOUNDS);
                continue;
            }
        }
        if constexpr (STYLE == 1) {
            uint4 x, y;
            deinterleave(a, b, x, y);
            rotate8(x, y, cv, sv);
            interleave(x, y, a, b);
        } else {
            rotate8(a, b, cv, sv);
        }
        if (is_q) {
            p.q_out[base + ca] = a;
            p.q_out[base + cb] = b;
            continue;
        }
        const long long blk = slot / p.block_size;
        const long long off = slot - blk * p.block_size;
        const long long row = (blk * p.num_kv_heads + head) * p.block_size + off;  // pool row
        const long long ea = row * p.head_dim + ca * 8LL, eb = row * p.head_dim + cb * 8LL;  // element offsets
        if constexpr (MODE == 0) {
            __nv_bfloat16 *kc = static_cast<__nv_bfloat16 *>(p.k_cache), *vc = static_cast<__nv_bfloat16 *>(p.v_cache);
            *reinterpret_cast<uint4 *>(kc + ea) = a;
            *reinterpret_cast<uint4 *>(kc + eb) = b;
            *reinterpret_cast<uint4 *>(vc + ea) = va;
            *reinterpret_cast<uint4 *>(vc + eb) = vb;
        } else {
            float ks, vs;
            if constexpr (MODE == 2) {
                // the row's L lanes are adjacent (L divides 32 and the stride)
                const int lane = threadIdx.x & 31;
                const unsigned group = (L == 32 ? 0xffffffffu : ((1u << L) - 1u)) << (lane & ~(L - 1));
                float km = fmaxf(amax8(a), amax8(b)), vm = fmaxf(amax8(va), amax8(vb));
                for (int o = L >> 1; o > 0; o >>= 1) {
                    km = fmaxf(km, __shfl_xor_sync(group, km, o, L));
                    vm = fmaxf(vm, __shfl_xor_sync(group, vm, o, L));
                }
                ks = token_scale(km);
                vs = token_scale(vm);
                if (c == 0) {
                    p.k_scale[row] = ks;
                    p.v_scale[row] = vs;
                }
            } else {
                ks = __ldg(p.k_scale + head);
                vs = __ldg(p.v_scale + head);
            }
            uint8_t *kc = static_cast<uint8_t *>(p.k_cache), *vc = static_cast<uint8_t *>(p.v_cache);
            *reinterpret_cast<uint2 *>(kc + ea) = quantise8(a, ks);
            *reinterpret_cast<uint2 *>(kc + eb) = quantise8(b, ks);
            *reinterpret_cast<uint2 *>(vc + ea) = quantise8(va, vs);
            *reinterpret_cast<uint2 *>(vc + eb) = quantise8(vb, vs);
        }
    }
}

template <int MODE>
void launch_rope_mode(const RopeParams &p, int style, unsigned blocks, cudaStream_t stream) {
    if (style == 1)
        store_kvcache_rope_kernel<MODE, 1><<<blocks, 256, 0, stream>>>(p);
    else
        store_kvcache_rope_kernel<MODE, 0><<<blocks, 256, 0, stream>>>(p);
}

}  // namespace

cudaError_t launch_store_kvcache_rope(const void *q, void *q_out, const void *k, const void *v, void *k_cache,
                                      void *v_cache, const int32_t *slot_mapping, const int32_t *positions,
                                      const float *cos_sin, int max_position, int style, int num_tokens,
                                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                      int64_t num_blocks, int mode, float *k_scale, float *v_scale, int *dev_err,
                                      int num_sms, cudaStream_t stream) {
    RopeParams p;
    p.q = static_cast<const uint4 *>(q);
    p.q_out = static_cast<uint4 *>(q_out);
    p.k = static_cast<const uint4 *>(k);
    p.v = static_cast<const uint4 *>(v);
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.slots = slot_mapping;
    p.positions = positions;
    p.cos_sin = cos_sin;
    p.max_position = max_position;
    p.lanes_per_row = head_dim / 16;
    p.num_q_heads = q ? num_q_heads : 0;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.pool_slots = (long long)num_blocks * block_size;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.dev_err = dev_err;
    p.total_units = (long long)num_tokens * (p.num_q_heads + num_kv_heads) * p.lanes_per_row;
    long long blocks = (p.total_units + 255) / 256;
    const long long cap = (long long)num_sms * 16;  // grid-stride beyond 16 blocks per SM (an uncapped grid measured slower)
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (mode == 2)
        launch_rope_mode<2>(p, style, (unsigned)blocks, stream);
    else if (mode == 1)
        launch_rope_mode<1>(p, style, (unsigned)blocks, stream);
    else
        launch_rope_mode<0>(p, style, (unsigned)blocks, stream);
    return cudaGetLastError();
}

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
