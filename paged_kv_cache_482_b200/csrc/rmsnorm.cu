// rmsnorm.cu -- fused residual add + RMSNorm (sm_100a).
//
// The operation ("nano-vllm-lite：深入理解LLM推理机制的教育级开源项目", section
// 核心技术改进 1 "CUDA融合内核：Add+RMSNorm": the residual add and the RMSNorm
// after it in one kernel, so the sum never makes a round trip through
// memory): for each row of `hidden` elements
//   h = x + residual          (fp32; the residual stream continues as bf16(h))
//   out = weight * h / sqrt(mean(h^2) + eps)
// Without a residual it is a plain RMSNorm of x.
//
// Bandwidth-bound: per element 2 bytes of x, 2 of the residual read and 2
// written, 2 of out written. A persistent grid of CTAs walks the rows; a
// thread owns NV 16-byte vectors of a row, keeps its slice of the weight in
// registers across rows, and loads the next row while the current one is
// reduced. One block reduction per row (warp shuffles, then one warp over
// the per-warp sums), with the per-warp scratch double-buffered by row so
// that a row costs a single barrier pair.
#include "pkv_common.cuh"
#include "pkv_launch.h"

namespace pkv {
namespace {

constexpr int kMaxThreads = 256;
constexpr int kMaxWarps = kMaxThreads / 32;

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
    f[0] = bf16lo(v.x);
    f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y);
    f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z);
    f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w);
    f[7] = bf16hi(v.w);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

template <int NV, bool RES>
__global__ void __launch_bounds__(kMaxThreads) fused_add_rmsnorm_kernel(const __nv_bfloat16 *x, __nv_bfloat16 *residual,
                                                                 const __nv_bfloat16 *weight, __nv_bfloat16 *out,
                                                                 int num_tokens, int hidden, float eps) {
    __shared__ float red[2][kMaxWarps];
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int nwarps = nthr >> 5;
    const int nvec = hidden >> 3;
    const float inv_h = 1.0f / static_cast<float>(hidden);

    uint4 wv[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int v = tid + k * nthr;
        wv[k] = v < nvec ? __ldg(reinterpret_cast<const uint4 *>(weight) + v) : make_uint4(0, 0, 0, 0);
    }

    int row = blockIdx.x;
    uint4 xv[NV], rv[NV];
    auto load_row = [&](int r) {
        const int64_t base = static_cast<int64_t>(r) * nvec;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int v = tid + k * nthr;
            if (v < nvec) {
                xv[k] = ld_stream(reinterpret_cast<const uint4 *>(x) + base + v);
                if (RES) rv[k] = ld_stream(reinterpret_cast<const uint4 *>(residual) + base + v);
            }
        }
    };
    if (row < num_tokens) load_row(row);

    for (int it = 0; row < num_tokens; row += gridDim.x, ++it) {
        // h = x + r for this row, its sum of squares, and the rounded residual
        float h[NV][8];
        float ss = 0.0f;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            if (tid + k * nthr < nvec) {
                unpack8(xv[k], h[k]);
                if (RES) {
                    float r8[8];
                    unpack8(rv[k], r8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) h[k][i] += r8[i];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(h[k][i], h[k][i], ss);
            }
        }
        const int64_t base = static_cast<int64_t>(row) * nvec;
        if (RES) {
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                const int v = tid + k * nthr;
                if (v < nvec)
                    st_stream(reinterpret_cast<uint4 *>(residual) + base + v,
                              make_uint4(pack2(h[k][0], h[k][1]), pack2(h[k][2], h[k][3]), pack2(h[k][4], h[k][5]),
                                         pack2(h[k][6], h[k][7])));
            }
        }
        // the next row's loads overlap this row's reduction
        const int next = row + gridDim.x;
        if (next < num_tokens) load_row(next);

#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        float *rb = red[it & 1];
        if ((tid & 31) == 0) rb[tid >> 5] = ss;
        __syncthreads();
        float tot = (tid & 31) < nwarps ? rb[tid & 31] : 0.0f;  // nwarps <= 8
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        const float inv = rsqrtf(tot * inv_h + eps);

#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int v = tid + k * nthr;
            if (v < nvec) {
                float w8[8];
                unpack8(wv[k], w8);
                st_stream(reinterpret_cast<uint4 *>(out) + base + v,
                          make_uint4(pack2(h[k][0] * inv * w8[0], h[k][1] * inv * w8[1]),
                                     pack2(h[k][2] * inv * w8[2], h[k][3] * inv * w8[3]),
                                     pack2(h[k][4] * inv * w8[4], h[k][5] * inv * w8[5]),
                                     pack2(h[k][6] * inv * w8[6], h[k][7] * inv * w8[7])));
            }
        }
        // red[it & 1] is rewritten two rows later, after the next row's barrier
    }
}

// Persistent grid: as many CTAs as fit on the GPU at once (from the
// occupancy the compiled kernel allows), at most one per row.
template <int NV, bool RES>
cudaError_t launch_nv_res(const NormArgs &a, int threads, int num_sms, cudaStream_t stream) {
    auto kern = fused_add_rmsnorm_kernel<NV, RES>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
    if (e != cudaSuccess) return e;
    long long grid = static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1);
    if (grid > a.num_tokens) grid = a.num_tokens;
    kern<<<static_cast<int>(grid), threads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.x), static_cast<__nv_bfloat16 *>(a.residual),
        static_cast<const __nv_bfloat16 *>(a.weight), static_cast<__nv_bfloat16 *>(a.out), a.num_tokens, a.hidden,
        a.eps);
    return cudaGetLastError();
}

template <int NV>
cudaError_t launch_nv(const NormArgs &a, int threads, int num_sms, cudaStream_t stream) {
    return a.residual ? launch_nv_res<NV, true>(a, threads, num_sms, stream)
                      : launch_nv_res<NV, false>(a, threads, num_sms, stream);
}

}  // namespace

int norm_max_hidden() { return 8 * 8 * kMaxThreads; }  // 8 vectors of 8 per thread

cudaError_t launch_fused_add_rmsnorm(const NormArgs &a, int num_sms, cudaStream_t stream) {
    const int nvec = a.hidden / 8;
    // threads per CTA: one vector per thread up to kMaxThreads threads, then
    // more vectors per thread (NV, up to 8)
    int nv = 1, threads = 32;
    while (threads < nvec && threads < kMaxThreads) threads <<= 1;
    while (nv * threads < nvec) nv <<= 1;
    switch (nv) {
        case 1: return launch_nv<1>(a, threads, num_sms, stream);
        case 2: return launch_nv<2>(a, threads, num_sms, stream);
        case 4: return launch_nv<4>(a, threads, num_sms, stream);
        default: return launch_nv<8>(a, threads, num_sms, stream);
    }
}

}  // namespace pkv
