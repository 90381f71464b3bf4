// Allocation-free variant of pkv_paged_attention_decode.
//
// Some callers cannot hand the library a workspace: a serving engine that has
// already reserved nearly all device memory for its KV pool and weights (the
// usual gpu_memory_utilization setting), or code running inside a plugin /
// enqueue hook that must not call cudaMalloc or cudaFree because those can
// synchronise the device and stall every other stream. For them this entry
// point keeps the split-K scratch in a fixed array that lives in the library's
// own device memory, so the call itself allocates nothing.
//
// The array costs PKV_NOALLOC_SCRATCH_BYTES on every GPU that loads this
// library, for the life of the process. Calls share it: two calls that overlap
// on the GPU (different streams, or different host threads) race on it.
// The split-K kernels write every scratch entry they later read; the one part
// that must start at zero, the persistent schedule's arrival counters, is
// cleared on the stream by each call before its launch (a memset, which
// allocates nothing). So the previous call's contents do no harm.
//
// The array's device address is looked up once per device and kept. A device
// reset (cudaDeviceReset) unloads the module and may move the array, so no call
// of this entry point may follow a device reset in the same process.
#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device. Host code only
// sees a host-side stand-in for `g_noalloc_scratch`; the real address has to be
// asked for, once per device, with that device current.
pkv_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PKV_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" pkv_status pkv_paged_attention_decode_noalloc(
    void* out, pkv_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
    pkv_dtype kv_dtype, const int32_t* block_tables, const int32_t* context_lens, float scale, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, int partition_tokens, void* stream) {
    const size_t need = pkv_paged_attention_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                            block_size, max_blocks_per_seq, max_context_len,
                                                            partition_tokens);
    if (need == (size_t)-1) return PKV_ERR_INVALID_ARG;
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_UNSUPPORTED;   // larger than the fixed array
    void* scratch = nullptr;
    if (need > 0) {
        const pkv_status st = scratch_for_current_device(&scratch);
        if (st != PKV_OK) return st;
    }
    return pkv_paged_attention_decode(out, out_dtype, q, k_cache, v_cache, kv_dtype, block_tables, context_lens,
                                      scale, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, max_context_len, partition_tokens, scratch,
                                      need > 0 ? (size_t)PKV_NOALLOC_SCRATCH_BYTES : 0, stream);
}
