// One whole decode step from host buffers, in native code.
//
// The step follows "vLLM PagedAttention 深度解析" §3.3 (decode: write the new
// token's K/V into its logical block through the block table, a new block when
// the last one is full) and §4.1 (a shared partially filled block is copied
// before the write):
//   1. block manager: one slot per sequence, copy-on-write pairs, block tables;
//   2. the metadata goes to the device in one copy from pinned staging, q and
//      the new K/V in one copy each from the caller's host buffers;
//   3. copy_blocks (if any pair), reshape_and_cache, paged decode attention;
//   4. the attention output is copied back to the caller's host buffer.
// Everything is enqueued on the caller's stream; the call returns without
// waiting. The step context owns the device-side buffers and two pinned
// staging slots (so one step's metadata can be written while the previous
// step's copy is still in flight).
#include <cuda_runtime.h>

#include <chrono>
#include <cstring>
#include <new>
#include <vector>

#include "common.cuh"

struct pkv_step_ctx {
    int max_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks, block_size;
    pkv_dtype kv_dtype, out_dtype;
    float k_scale = 1.f, v_scale = 1.f;   // FP8 caches
    size_t meta_bytes, q_bytes, kv_bytes, out_bytes, ws_bytes;
    // device
    unsigned char* d_meta = nullptr;   // slots i64[S] | src i64[S] | dst i64[S] | tables i32[S*MB] | lens i32[S]
    void* d_q = nullptr;
    void* d_k = nullptr;
    void* d_v = nullptr;
    void* d_out = nullptr;
    void* d_ws = nullptr;
    // host
    unsigned char* h_meta[2] = {nullptr, nullptr};
    cudaEvent_t meta_done[2] = {nullptr, nullptr};
    int slot = 0;
    int device = 0;
    // optional phase timing of the last step (pkv_step_ctx_set_timing)
    bool timing = false;
    cudaEvent_t tev[4] = {nullptr, nullptr, nullptr, nullptr};   // before H2D, after H2D, after kernels, after D2H
    float host_ms = 0.f;                                          // block manager + tables, host clock
    bool timed_step = false;
};

namespace {

int elt(pkv_dtype t) { return t == PKV_F32 ? 4 : (t == PKV_BF16 ? 2 : 1); }
// host-side element size of the step's q / new K,V (bf16 for an FP8 cache)
int in_elt(pkv_dtype t) { return t == PKV_F32 ? 4 : 2; }

void release(pkv_step_ctx* c) {
    if (!c) return;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    cudaFree(c->d_meta);
    cudaFree(c->d_q);
    cudaFree(c->d_k);
    cudaFree(c->d_v);
    cudaFree(c->d_out);
    cudaFree(c->d_ws);
    for (int i = 0; i < 2; ++i) {
        if (c->h_meta[i]) cudaFreeHost(c->h_meta[i]);
        if (c->meta_done[i]) cudaEventDestroy(c->meta_done[i]);
    }
    for (int i = 0; i < 4; ++i)
        if (c->tev[i]) cudaEventDestroy(c->tev[i]);
    cudaSetDevice(prev);
    delete c;
}

}  // namespace

extern "C" {

pkv_status pkv_step_ctx_create(int max_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int max_blocks_per_seq, int block_size, pkv_dtype kv_dtype, pkv_dtype out_dtype,
                               int partition_tokens, float k_scale, float v_scale, pkv_step_ctx** out) {
    if (!out || max_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_blocks_per_seq <= 0 || block_size <= 0 || num_q_heads % num_kv_heads != 0 ||
        (kv_dtype != PKV_F32 && kv_dtype != PKV_BF16 && kv_dtype != PKV_FP8_E4M3) ||
        (out_dtype != PKV_F32 && out_dtype != PKV_BF16) ||
        (kv_dtype == PKV_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)))
        return PKV_ERR_INVALID_ARG;
    *out = nullptr;
    pkv_step_ctx* c = new (std::nothrow) pkv_step_ctx();
    if (!c) return PKV_ERR_INVALID_ARG;
    cudaGetDevice(&c->device);
    c->max_seqs = max_seqs;
    c->num_q_heads = num_q_heads;
    c->num_kv_heads = num_kv_heads;
    c->head_dim = head_dim;
    c->max_blocks = max_blocks_per_seq;
    c->block_size = block_size;
    c->kv_dtype = kv_dtype;
    c->out_dtype = out_dtype;
    c->k_scale = k_scale;
    c->v_scale = v_scale;
    const size_t S = (size_t)max_seqs;
    c->meta_bytes = S * 8 * 3 + S * max_blocks_per_seq * 4 + S * 4;
    c->q_bytes = S * num_q_heads * head_dim * in_elt(kv_dtype);
    c->kv_bytes = S * num_kv_heads * head_dim * in_elt(kv_dtype);
    c->out_bytes = S * num_q_heads * head_dim * elt(out_dtype);
    // Largest workspace any step can ask for: a fixed partition length never needs
    // more than at max_seqs and full tables; the library-chosen one is >= 256 tokens.
    const int sizing_part = partition_tokens == 0 ? 256 : partition_tokens;
    const size_t ws = pkv_paged_attention_workspace_bytes(max_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                          max_blocks_per_seq, 0, sizing_part);
    if (ws == (size_t)-1) {
        delete c;
        return PKV_ERR_INVALID_ARG;
    }
    c->ws_bytes = ws;
    bool ok = cudaMalloc(&c->d_meta, c->meta_bytes) == cudaSuccess && cudaMalloc(&c->d_q, c->q_bytes) == cudaSuccess &&
              cudaMalloc(&c->d_k, c->kv_bytes) == cudaSuccess && cudaMalloc(&c->d_v, c->kv_bytes) == cudaSuccess &&
              cudaMalloc(&c->d_out, c->out_bytes) == cudaSuccess &&
              (ws == 0 || cudaMalloc(&c->d_ws, ws) == cudaSuccess);
    for (int i = 0; ok && i < 2; ++i)
        ok = cudaHostAlloc((void**)&c->h_meta[i], c->meta_bytes, cudaHostAllocDefault) == cudaSuccess &&
             cudaEventCreateWithFlags(&c->meta_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        release(c);
        return PKV_ERR_CUDA;
    }
    *out = c;
    return PKV_OK;
}

void pkv_step_ctx_destroy(pkv_step_ctx* ctx) { release(ctx); }

pkv_status pkv_decode_step(pkv_step_ctx* c, pkv_block_manager* bm, const int64_t* seq_ids, int n,
                           const void* q_host, const void* k_host, const void* v_host, void* k_cache, void* v_cache,
                           int num_blocks, float scale, int partition_tokens, void* out_host, void* stream) {
    if (!c || !bm || n < 0 || n > c->max_seqs || (n > 0 && (!seq_ids || !q_host || !k_host || !v_host ||
                                                            !k_cache || !v_cache || !out_host)))
        return PKV_ERR_INVALID_ARG;
    if (pkv_bm_block_size(bm) != c->block_size) return PKV_ERR_INVALID_ARG;
    if (n == 0) return PKV_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t S = (size_t)c->max_seqs;
    const bool timing = c->timing;
    c->timed_step = false;
    const auto t_host0 = std::chrono::steady_clock::now();
    // 1. host metadata into a pinned slot whose previous copy has finished
    const int sl = c->slot;
    c->slot ^= 1;
    if (cudaEventSynchronize(c->meta_done[sl]) != cudaSuccess) return PKV_ERR_CUDA;
    unsigned char* h = c->h_meta[sl];
    int64_t* slots = reinterpret_cast<int64_t*>(h);
    int64_t* src = slots + S;
    int64_t* dst = src + S;
    int32_t* tables = reinterpret_cast<int32_t*>(dst + S);
    int32_t* lens = tables + S * c->max_blocks;
    int ncopy = 0;
    pkv_status s = pkv_bm_append_slots(bm, seq_ids, n, slots, src, dst, &ncopy, nullptr);
    if (s != PKV_OK) return s;
    // tables of the listed sequences, row stride max_blocks
    s = pkv_bm_block_tables(bm, seq_ids, n, c->max_blocks, tables, lens);
    if (s != PKV_OK) return s;
    int max_len = 0;
    for (int i = 0; i < n; ++i) max_len = lens[i] > max_len ? lens[i] : max_len;
    if (timing) {
        c->host_ms = std::chrono::duration<float, std::milli>(std::chrono::steady_clock::now() - t_host0).count();
        if (cudaEventRecord(c->tev[0], st) != cudaSuccess) return PKV_ERR_CUDA;
    }
    // 2. copies to the device
    if (cudaMemcpyAsync(c->d_meta, h, c->meta_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaEventRecord(c->meta_done[sl], st) != cudaSuccess)
        return PKV_ERR_CUDA;
    const size_t qb = (size_t)n * c->num_q_heads * c->head_dim * in_elt(c->kv_dtype);
    const size_t kb = (size_t)n * c->num_kv_heads * c->head_dim * in_elt(c->kv_dtype);
    if (cudaMemcpyAsync(c->d_q, q_host, qb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(c->d_k, k_host, kb, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(c->d_v, v_host, kb, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (timing && cudaEventRecord(c->tev[1], st) != cudaSuccess) return PKV_ERR_CUDA;
    const int64_t* d_slots = reinterpret_cast<const int64_t*>(c->d_meta);
    const int64_t* d_src = d_slots + S;
    const int64_t* d_dst = d_src + S;
    const int32_t* d_tables = reinterpret_cast<const int32_t*>(d_dst + S);
    const int32_t* d_lens = d_tables + S * c->max_blocks;
    // 3. the kernels
    if (ncopy > 0) {
        s = pkv_copy_blocks(k_cache, v_cache, c->kv_dtype, d_src, d_dst, ncopy, c->block_size, c->num_kv_heads, c->head_dim,
                            num_blocks, stream);
        if (s != PKV_OK) return s;
    }
    const bool fp8 = c->kv_dtype == PKV_FP8_E4M3;
    s = fp8 ? pkv_reshape_and_cache_fp8(c->d_k, c->d_v, PKV_BF16, k_cache, v_cache, c->k_scale, c->v_scale, d_slots,
                                        n, c->num_kv_heads, c->head_dim, c->block_size, num_blocks, stream)
            : pkv_reshape_and_cache(c->d_k, c->d_v, k_cache, v_cache, c->kv_dtype, d_slots, n, c->num_kv_heads,
                                    c->head_dim, c->block_size, num_blocks, stream);
    if (s != PKV_OK) return s;
    // workspace sized at creation for max_seqs and the table capacity; this call asks for the
    // same schedule over n sequences, which never needs more
    s = fp8 ? pkv_paged_attention_decode_fp8(c->d_out, c->out_dtype, c->d_q, k_cache, v_cache, c->k_scale,
                                             c->v_scale, d_tables, d_lens, scale, n, c->num_q_heads, c->num_kv_heads,
                                             c->head_dim, c->block_size, c->max_blocks, num_blocks, max_len, partition_tokens,
                                             c->d_ws, c->ws_bytes, stream)
            : pkv_paged_attention_decode(c->d_out, c->out_dtype, c->d_q, k_cache, v_cache, c->kv_dtype, d_tables,
                                         d_lens, scale, n, c->num_q_heads, c->num_kv_heads, c->head_dim, c->block_size,
                                         c->max_blocks, num_blocks, max_len, partition_tokens, c->d_ws, c->ws_bytes,
                                         stream);
    if (s != PKV_OK) return s;
    if (timing && cudaEventRecord(c->tev[2], st) != cudaSuccess) return PKV_ERR_CUDA;
    // 4. the result back to the host
    const size_t ob = (size_t)n * c->num_q_heads * c->head_dim * elt(c->out_dtype);
    if (cudaMemcpyAsync(out_host, c->d_out, ob, cudaMemcpyDeviceToHost, st) != cudaSuccess) return PKV_ERR_CUDA;
    if (timing) {
        if (cudaEventRecord(c->tev[3], st) != cudaSuccess) return PKV_ERR_CUDA;
        c->timed_step = true;
    }
    return PKV_OK;
}

pkv_status pkv_step_ctx_set_timing(pkv_step_ctx* c, int enable) {
    if (!c) return PKV_ERR_INVALID_ARG;
    if (enable && !c->tev[0]) {
        int prev = 0;
        cudaGetDevice(&prev);
        cudaSetDevice(c->device);
        bool ok = true;
        for (int i = 0; i < 4 && ok; ++i) ok = cudaEventCreate(&c->tev[i]) == cudaSuccess;
        cudaSetDevice(prev);
        if (!ok) return PKV_ERR_CUDA;
    }
    c->timing = enable != 0;
    c->timed_step = false;
    return PKV_OK;
}

pkv_status pkv_step_ctx_last_timing(pkv_step_ctx* c, float* out) {
    if (!c || !out) return PKV_ERR_INVALID_ARG;
    if (!c->timed_step) return PKV_ERR_INVALID_ARG;
    if (cudaEventSynchronize(c->tev[3]) != cudaSuccess) return PKV_ERR_CUDA;
    out[0] = c->host_ms;
    for (int i = 0; i < 3; ++i)
        if (cudaEventElapsedTime(&out[1 + i], c->tev[i], c->tev[i + 1]) != cudaSuccess) return PKV_ERR_CUDA;
    return PKV_OK;
}

}  // extern "C"
