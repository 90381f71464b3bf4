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
// The call returns without waiting. The step context owns three streams (host
// to device copies, kernels, device to host copies), two slots of device-side
// step buffers and two pinned metadata staging slots, so consecutive steps
// overlap: step i + 1's inputs cross the host link and step i - 1's output
// comes back while step i's kernels run. Each step starts after the caller's
// prior work on its stream, and the caller's stream passes the step only once
// the step's output is in the host buffer.
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
    // device, two slots (a step uses slot i % 2)
    unsigned char* d_meta[2] = {nullptr, nullptr};   // slots i64[S] | src i64[S] | dst i64[S] | tables i32[S*MB] | lens i32[S]
    void* d_q[2] = {nullptr, nullptr};
    void* d_k[2] = {nullptr, nullptr};
    void* d_v[2] = {nullptr, nullptr};
    void* d_out[2] = {nullptr, nullptr};
    void* d_ws = nullptr;                            // split-K workspace: used by the kernel stream only, in order
    // host
    unsigned char* h_meta[2] = {nullptr, nullptr};
    cudaEvent_t meta_done[2] = {nullptr, nullptr};   // the slot's metadata copy finished (pinned slot reusable)
    // streams and the events that order a slot's use across them
    cudaStream_t s_h2d = nullptr, s_comp = nullptr, s_d2h = nullptr;
    cudaEvent_t ev_caller[2] = {nullptr, nullptr};   // the caller's prior work
    cudaEvent_t ev_in[2] = {nullptr, nullptr};       // the slot's inputs are on the device
    cudaEvent_t ev_comp[2] = {nullptr, nullptr};     // the slot's kernels finished (inputs free, output ready)
    cudaEvent_t ev_d2h[2] = {nullptr, nullptr};      // the slot's output is on the host (output buffer free)
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
    for (cudaStream_t s : {c->s_h2d, c->s_comp, c->s_d2h})
        if (s) cudaStreamSynchronize(s);
    for (int i = 0; i < 2; ++i) {
        cudaFree(c->d_meta[i]);
        cudaFree(c->d_q[i]);
        cudaFree(c->d_k[i]);
        cudaFree(c->d_v[i]);
        cudaFree(c->d_out[i]);
        if (c->h_meta[i]) cudaFreeHost(c->h_meta[i]);
        for (cudaEvent_t e : {c->meta_done[i], c->ev_caller[i], c->ev_in[i], c->ev_comp[i], c->ev_d2h[i]})
            if (e) cudaEventDestroy(e);
    }
    cudaFree(c->d_ws);
    for (cudaStream_t s : {c->s_h2d, c->s_comp, c->s_d2h})
        if (s) cudaStreamDestroy(s);
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
    bool ok = (ws == 0 || cudaMalloc(&c->d_ws, ws) == cudaSuccess) &&
              cudaStreamCreateWithFlags(&c->s_h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&c->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&c->s_d2h, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i) {
        ok = cudaMalloc(&c->d_meta[i], c->meta_bytes) == cudaSuccess && cudaMalloc(&c->d_q[i], c->q_bytes) == cudaSuccess &&
             cudaMalloc(&c->d_k[i], c->kv_bytes) == cudaSuccess && cudaMalloc(&c->d_v[i], c->kv_bytes) == cudaSuccess &&
             cudaMalloc(&c->d_out[i], c->out_bytes) == cudaSuccess &&
             cudaHostAlloc((void**)&c->h_meta[i], c->meta_bytes, cudaHostAllocDefault) == cudaSuccess;
        for (cudaEvent_t* e : {&c->meta_done[i], &c->ev_caller[i], &c->ev_in[i], &c->ev_comp[i], &c->ev_d2h[i]})
            ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    }
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
    if (timing) c->host_ms = std::chrono::duration<float, std::milli>(std::chrono::steady_clock::now() - t_host0).count();
    // 2. copies to the device, on the copy stream: after the caller's prior work,
    //    and once step i - 2's kernels (the slot's last users) have finished
    if (cudaEventRecord(c->ev_caller[sl], st) != cudaSuccess ||
        cudaStreamWaitEvent(c->s_h2d, c->ev_caller[sl], 0) != cudaSuccess ||
        cudaStreamWaitEvent(c->s_comp, c->ev_caller[sl], 0) != cudaSuccess ||
        cudaStreamWaitEvent(c->s_h2d, c->ev_comp[sl], 0) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (timing && cudaEventRecord(c->tev[0], c->s_h2d) != cudaSuccess) return PKV_ERR_CUDA;
    const size_t qb = (size_t)n * c->num_q_heads * c->head_dim * in_elt(c->kv_dtype);
    const size_t kb = (size_t)n * c->num_kv_heads * c->head_dim * in_elt(c->kv_dtype);
    if (cudaMemcpyAsync(c->d_meta[sl], h, c->meta_bytes, cudaMemcpyHostToDevice, c->s_h2d) != cudaSuccess ||
        cudaEventRecord(c->meta_done[sl], c->s_h2d) != cudaSuccess ||
        cudaMemcpyAsync(c->d_q[sl], q_host, qb, cudaMemcpyHostToDevice, c->s_h2d) != cudaSuccess ||
        cudaMemcpyAsync(c->d_k[sl], k_host, kb, cudaMemcpyHostToDevice, c->s_h2d) != cudaSuccess ||
        cudaMemcpyAsync(c->d_v[sl], v_host, kb, cudaMemcpyHostToDevice, c->s_h2d) != cudaSuccess ||
        cudaEventRecord(c->ev_in[sl], c->s_h2d) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (timing && cudaEventRecord(c->tev[1], c->s_h2d) != cudaSuccess) return PKV_ERR_CUDA;
    const int64_t* d_slots = reinterpret_cast<const int64_t*>(c->d_meta[sl]);
    const int64_t* d_src = d_slots + S;
    const int64_t* d_dst = d_src + S;
    const int32_t* d_tables = reinterpret_cast<const int32_t*>(d_dst + S);
    const int32_t* d_lens = d_tables + S * c->max_blocks;
    // 3. the kernels, on the kernel stream: once the inputs are in, and once step
    //    i - 2's output (the slot's output buffer) has been read back
    cudaStream_t sc = c->s_comp;
    if (cudaStreamWaitEvent(sc, c->ev_in[sl], 0) != cudaSuccess || cudaStreamWaitEvent(sc, c->ev_d2h[sl], 0) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (ncopy > 0) {
        s = pkv_copy_blocks(k_cache, v_cache, c->kv_dtype, d_src, d_dst, ncopy, c->block_size, c->num_kv_heads, c->head_dim,
                            num_blocks, sc);
        if (s != PKV_OK) return s;
    }
    const bool fp8 = c->kv_dtype == PKV_FP8_E4M3;
    s = fp8 ? pkv_reshape_and_cache_fp8(c->d_k[sl], c->d_v[sl], PKV_BF16, k_cache, v_cache, c->k_scale, c->v_scale,
                                        d_slots, n, c->num_kv_heads, c->head_dim, c->block_size, num_blocks, sc)
            : pkv_reshape_and_cache(c->d_k[sl], c->d_v[sl], k_cache, v_cache, c->kv_dtype, d_slots, n, c->num_kv_heads,
                                    c->head_dim, c->block_size, num_blocks, sc);
    if (s != PKV_OK) return s;
    // A page-locked out_host is written by the attention kernels themselves
    // (through its device mapping): the output crosses the host link while they
    // run and no copy follows them. Otherwise the output goes to the slot's
    // device buffer and is copied back.
    cudaPointerAttributes oa{};
    const bool direct_out = cudaPointerGetAttributes(&oa, out_host) == cudaSuccess &&
                            oa.type == cudaMemoryTypeHost && oa.devicePointer != nullptr;
    if (!direct_out) cudaGetLastError();                         // a pageable pointer: clear the query's error
    void* attn_out = direct_out ? oa.devicePointer : c->d_out[sl];
    // workspace sized at creation for max_seqs and the table capacity; this call asks for the
    // same schedule over n sequences, which never needs more
    s = fp8 ? pkv_paged_attention_decode_fp8(attn_out, c->out_dtype, c->d_q[sl], k_cache, v_cache, c->k_scale,
                                             c->v_scale, d_tables, d_lens, scale, n, c->num_q_heads, c->num_kv_heads,
                                             c->head_dim, c->block_size, c->max_blocks, num_blocks, max_len, partition_tokens,
                                             c->d_ws, c->ws_bytes, sc)
            : pkv_paged_attention_decode(attn_out, c->out_dtype, c->d_q[sl], k_cache, v_cache, c->kv_dtype, d_tables,
                                         d_lens, scale, n, c->num_q_heads, c->num_kv_heads, c->head_dim, c->block_size,
                                         c->max_blocks, num_blocks, max_len, partition_tokens, c->d_ws, c->ws_bytes, sc);
    if (s != PKV_OK) return s;
    if (cudaEventRecord(c->ev_comp[sl], sc) != cudaSuccess) return PKV_ERR_CUDA;
    if (timing && cudaEventRecord(c->tev[2], sc) != cudaSuccess) return PKV_ERR_CUDA;
    // 4. the result back to the host, on the other copy stream (unless the kernels
    //    wrote it there); the caller's stream passes this step once it is there
    cudaEvent_t done = c->ev_comp[sl];
    if (!direct_out) {
        const size_t ob = (size_t)n * c->num_q_heads * c->head_dim * elt(c->out_dtype);
        if (cudaStreamWaitEvent(c->s_d2h, c->ev_comp[sl], 0) != cudaSuccess ||
            cudaMemcpyAsync(out_host, c->d_out[sl], ob, cudaMemcpyDeviceToHost, c->s_d2h) != cudaSuccess ||
            cudaEventRecord(c->ev_d2h[sl], c->s_d2h) != cudaSuccess)
            return PKV_ERR_CUDA;
        done = c->ev_d2h[sl];
    }
    if (timing) {
        if (cudaEventRecord(c->tev[3], direct_out ? sc : c->s_d2h) != cudaSuccess) return PKV_ERR_CUDA;
        c->timed_step = true;
    }
    if (cudaStreamWaitEvent(st, done, 0) != cudaSuccess) return PKV_ERR_CUDA;
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
