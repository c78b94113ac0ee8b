// pagedkv_noalloc.cu -- paged decode for callers that cannot allocate device memory.
//
// pkv_paged_attention_decode needs a caller-provided device workspace when it
// splits long contexts (split-K partials). Some callers have no way to provide
// one: an engine that reserves all device memory for its KV pool at start-up
// and forbids later allocations, a plugin that sits behind a host framework
// whose device allocator it cannot reach through a C ABI, or code that must not
// allocate on its serving path. This file gives them an entry point that takes
// the scratch from a fixed-size array owned by the library instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it until the process exits. Host code cannot use the array's
// name as a device address (it names a host-side stand-in), so the device
// address is looked up with cudaGetSymbolAddress once per device, with that
// device current, on the entry point's first call on the device.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "pagedkv.h"

namespace {

// Stated maximum of the library-owned scratch (bytes), PKV_STATIC_SCRATCH_BYTES
// in the header: enough for the split-K partials of, e.g., 64 sequences x 32
// query heads x 32 partitions x 128 dims.
constexpr size_t kStaticScratchBytes = PKV_STATIC_SCRATCH_BYTES;
static_assert(kStaticScratchBytes % 256 == 0, "scratch size");

__device__ __align__(256) uint8_t g_pkv_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Device address of the array on the current device (looked up once per device).
int static_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return PKV_ERR_CUDA;
    }
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_pkv_static_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return PKV_ERR_CUDA;
        }
        g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return PKV_OK;
}

}  // namespace

extern "C" {

int pkv_paged_attention_decode_static_scratch(const void *q, const void *k_cache, const void *v_cache,
                                              const int32_t *block_tables, int max_blocks_per_seq,
                                              const int32_t *context_lens, const int32_t *seq_order,
                                              int num_seqs, int num_q_heads,
                                              int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                                              float scale, int cache_dtype, const float *k_scale,
                                              const float *v_scale, int max_context_len, int partition_request,
                                              void *out, int *dev_err, void *stream) {
    pkv_decode_plan plan;
    int st = pkv_plan_decode(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                             cache_dtype, partition_request, &plan);
    if (st != PKV_OK) return st;
    if (plan.workspace_bytes > kStaticScratchBytes) return PKV_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = static_scratch(&scratch);
    if (st != PKV_OK) return st;
    return pkv_paged_attention_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, seq_order,
                                      num_seqs,
                                      num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                                      cache_dtype, k_scale, v_scale, max_context_len, partition_request, scratch,
                                      kStaticScratchBytes, out, dev_err, stream);
}

}  // extern "C"
