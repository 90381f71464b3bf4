/*
 * pkv.h -- C ABI of the paged KV-cache decode library (libpkv.so, sm_100a).
 *
 * The library implements the data-parallel decode path of PagedAttention:
 *   - pkv_paged_attention_decode : decode attention of one query token per
 *     sequence over a KV cache split into fixed-size physical blocks and
 *     reached through per-sequence block tables (MHA and grouped-query).
 *   - pkv_paged_attention_multi_query : several causal query tokens per
 *     sequence (chunked prefill, speculative verification) over the same cache.
 *   - pkv_reshape_and_cache      : the per-token KV append into the cache.
 *   - pkv_copy_blocks            : physical block copies for copy-on-write forks.
 *   - pkv_swap_blocks            : block moves between the device pool and a
 *     page-locked host pool (preemption by swapping).
 *   - pkv_bm_*                   : a host-side block manager (free list, block
 *     tables, slot mapping, reference counts, copy-on-write) that produces the
 *     block tables, slot mappings and copy lists the kernels consume.
 *
 * Sources of the definitions (web pages on vLLM's PagedAttention):
 *   [BT]  "为什么PagedAttention能让大模型推理吞吐量提升数倍：从KV Cache内存碎片到分页管理的
 *         系统级优化", section "Block Table：GPU上的页表" (block tables, the 7-token
 *         walkthrough) and section "Memory Sharing" (shared blocks, copy-on-write).
 *   [ENG] "LLM 推理引擎内部原理：PagedAttention、Continuous Batching 与现代推理架构剖析",
 *         §2.3 (Block 分配器: free list, allocate, append_slot, free) and §2.4
 *         (CUDA kernel: cache layout [num_blocks, block_size, num_heads, head_dim],
 *         two-level addressing block table -> physical block -> in-block offset).
 *   [VP]  "vLLM PagedAttention 深度解析" (cyqw.cn), §3.3 (single-request prefill and
 *         decode flow), §4.1 (parallel sampling, reference counts, copy-on-write),
 *         §4.2 (beam search, blocks freed when their count reaches 0), §5.2
 *         (preemption: a request's KV blocks swapped out to CPU memory and back).
 *
 * Conventions shared by every call:
 *   - Every data pointer passed to a kernel entry point is a DEVICE pointer
 *     on the current CUDA device. The caller allocates and owns all memory;
 *     no kernel entry point allocates, frees or synchronises (pkv_get_device_error
 *     excepted). Calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).
 *   - Tensors are dense, row-major and 16-byte aligned:
 *       q, out          [num_seqs, num_q_heads, head_dim]
 *       k, v (new)      [num_tokens, num_kv_heads, head_dim]
 *       k_cache,v_cache [num_blocks, block_size, num_kv_heads, head_dim]   ([ENG] §2.4)
 *       block_tables    int32 [num_seqs, max_blocks_per_seq]; entry j of row s is the
 *                       physical block holding tokens [j*block_size, (j+1)*block_size)
 *       context_lens    int32 [num_seqs]
 *       slot_mapping    int64 [num_tokens]; slot = physical_block*block_size + offset
 *   - Supported: head_dim 64 or 128; block_size 8, 16, 32 or 64 ("vLLM
 *     PagedAttention 深度解析" §8.1 names powers of two with 16 the default;
 *     the persistent schedule takes 16 only); num_q_heads a multiple of
 *     num_kv_heads with group size num_q_heads/num_kv_heads in {1, 2, 4, 8, 16}
 *     (other groups return PKV_ERR_UNSUPPORTED; the persistent schedule takes
 *     groups up to 8);
 *     kv dtype f32 or bf16 (q has the kv dtype). Query head h reads KV head
 *     h / group (a reading: the pages do not discuss grouped-query attention).
 *   - Errors detected on the host (bad sizes, null pointers, unsupported shapes,
 *     a launch failure) are returned at once and nothing is launched.
 *     Errors that need device data (a block id or slot outside the pool, a context
 *     longer than the block table) cannot be seen by the host without a
 *     synchronisation: the kernel skips the bad access, records the error in a
 *     device error word and carries on; read it with pkv_get_device_error.
 *     No kernel traps or asserts.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,     /* a size, pointer or alignment is invalid */
    PKV_ERR_UNSUPPORTED = 2,     /* valid but not built (head_dim, block_size, group) */
    PKV_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed */
    PKV_ERR_DEVICE_BOUNDS = 4,   /* (device word) a block id / slot / length was out of range */
    PKV_ERR_OUT_OF_BLOCKS = 5,   /* (block manager) the free list is empty */
    PKV_ERR_DEVICE_TIMEOUT = 6   /* (device word) a bounded wait inside a kernel gave up */
} pkv_status;

typedef enum pkv_dtype {
    PKV_F32 = 0,
    PKV_BF16 = 1,
    PKV_FP8_E4M3 = 2     /* cache storage only: 8-bit e4m3 codes with a per-tensor scale */
} pkv_dtype;

/* partition_tokens value selecting the persistent schedule of the decode call. */
#define PKV_SCHEDULE_PERSISTENT (-1)

/* Human-readable name of a status code (static string, never NULL). */
const char* pkv_status_string(int status);

/* ------------------------------------------------------------------------- */
/* Decode attention                                                          */
/* ------------------------------------------------------------------------- */

/*
 * Decode attention over the paged cache ([ENG] §2.4; [BT] "Block Table"):
 * for every sequence s and query head h (KV head g = h / group),
 *     out[s,h,:] = sum_j softmax_j(scale * q[s,h,:] . K_s[j,g,:]) * V_s[j,g,:]
 * over the first context_lens[s] logical tokens j of sequence s, where token j
 * is read from physical block block_tables[s][j / block_size], offset
 * j % block_size. A sequence with context length 0 gets a zero output.
 *
 * Schedules (`partition_tokens`):
 *   > 0  contexts are cut into partitions of that many tokens (rounded up to a
 *        multiple of block_size), processed in parallel and merged exactly with
 *        a log-sum-exp reduction;
 *   0    the same, with the partition length picked from the shapes: the
 *        fewest partitions (of at least 256 tokens) whose units fill about
 *        one wave of the GPU, each sequence's count estimated from
 *        max_context_len with lengths spread over its upper half;
 *   -1   PKV_SCHEDULE_PERSISTENT: two CTAs per SM, each streaming an equal
 *        share of the batch's (sequence, block) tiles, with split sequences
 *        merged inside the kernel (at most 2048 sequences; block_size 16,
 *        f32 / bf16 caches).
 * With partition_tokens >= 0 and more than one sequence, a small planning
 * kernel first lists the live (sequence, partition) units longest first (full
 * partitions, then each sequence's last partition by decreasing size) and the
 * partition kernel takes them in that order, so long units start first and no
 * CTA is launched for a partition past a sequence's end before those with work.
 * The list and the partial results live in `workspace` (device memory, at least
 * pkv_paged_attention_workspace_bytes(...) bytes, 256-byte aligned; it may be
 * NULL when that size is 0). Its contents need no initialisation and are
 * scratch between calls; two calls in flight at once need two workspaces.
 *
 *   out            device, [num_seqs, num_q_heads, head_dim], out_dtype (f32 or bf16)
 *   q              device, [num_seqs, num_q_heads, head_dim], kv_dtype
 *   k_cache,v_cache device, [num_blocks, block_size, num_kv_heads, head_dim], kv_dtype
 *   block_tables   device int32 [num_seqs, max_blocks_per_seq]
 *   context_lens   device int32 [num_seqs], each in [0, max_blocks_per_seq*block_size]
 *   max_context_len host upper bound of context_lens (sizes the partition grid);
 *                  0 means max_blocks_per_seq*block_size. A length above it or
 *                  above the table's capacity is clamped and flagged
 *                  PKV_ERR_DEVICE_BOUNDS in the device error word.
 *   Block ids outside [0, num_blocks) are flagged the same way and read as zeros.
 */
pkv_status pkv_paged_attention_decode(
    void* out, pkv_dtype out_dtype,
    const void* q, const void* k_cache, const void* v_cache, pkv_dtype kv_dtype,
    const int32_t* block_tables, const int32_t* context_lens, float scale,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, int partition_tokens,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode attention over an FP8 (e4m3) cache written by pkv_reshape_and_cache_fp8
 * ("vLLM PagedAttention 深度解析" §7.4). Same computation and arguments as
 * pkv_paged_attention_decode with K = decode(k code) * k_scale and
 * V = decode(v code) * v_scale; q is bf16 [num_seqs, num_q_heads, head_dim]
 * (converted to f16 for the tensor-core path, so |q| should stay below 65504).
 * head_dim 128; partition_tokens >= 0 (the persistent schedule is not built for
 * fp8). The workspace rule is pkv_paged_attention_workspace_bytes's.
 */
pkv_status pkv_paged_attention_decode_fp8(
    void* out, pkv_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
    float k_scale, float v_scale, const int32_t* block_tables, const int32_t* context_lens, float scale,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, int partition_tokens,
    void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace pkv_paged_attention_decode needs for these sizes (0 when
 * no sequence can span more than one partition). Same partition rule as the
 * decode call; pass the same max_context_len and partition_tokens. Returns
 * (size_t)-1 for invalid sizes. */
size_t pkv_paged_attention_workspace_bytes(
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int partition_tokens);

/* The partition length (tokens) the decode call uses for these sizes, 0 for
 * the persistent schedule, -1 for invalid sizes. */
int pkv_paged_attention_partition_tokens(
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_context_len, int partition_tokens);

/* Size of the fixed scratch array behind pkv_paged_attention_decode_noalloc. */
#define PKV_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * pkv_paged_attention_decode for callers that cannot allocate device memory.
 * (The pages have no counterpart to this call; it is a property of this
 * library's interface, not of the method.)
 *
 * Who needs it: a caller whose device memory is already fully reserved by
 * someone else (a serving engine that hands nearly all of the GPU to its KV
 * pool and weights up front), or code that runs inside a plugin or enqueue
 * hook where cudaMalloc / cudaFree are off limits because they can synchronise
 * the whole device. Such a caller still owns and passes every input and
 * output; only the split-K scratch moves into a fixed array of
 * PKV_NOALLOC_SCRATCH_BYTES that the library keeps in each GPU's memory from
 * the moment the GPU loads the library until the process exits. The call
 * allocates nothing.
 *
 * Arguments and results are exactly those of pkv_paged_attention_decode,
 * without workspace / workspace_bytes. The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current);
 * make that first call before any stream capture on that device.
 *
 * Limit: when pkv_paged_attention_workspace_bytes(...) for these sizes exceeds
 * PKV_NOALLOC_SCRATCH_BYTES the call returns PKV_ERR_UNSUPPORTED and launches
 * nothing (use larger partition_tokens, fewer sequences per call, or the
 * regular entry point with your own workspace).
 *
 * Every call uses the same array and leaves its contents behind. The only part
 * that must start at zero (the persistent schedule's arrival counters) is
 * cleared by each call on `stream` before its kernel runs, so a previous call's
 * leftovers do no harm. Calls whose kernels overlap on the GPU (two streams, two
 * host threads) race on the array: serialise them.
 *
 * The device address is looked up once per device and kept for the life of the
 * process. A device reset (cudaDeviceReset) may move the array, so this entry
 * point must not be called after a device reset in the same process.
 */
pkv_status pkv_paged_attention_decode_noalloc(
    void* out, pkv_dtype out_dtype,
    const void* q, const void* k_cache, const void* v_cache, pkv_dtype kv_dtype,
    const int32_t* block_tables, const int32_t* context_lens, float scale,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, int partition_tokens, void* stream);

/* ------------------------------------------------------------------------- */
/* Cache-side kernels                                                        */
/* ------------------------------------------------------------------------- */

/*
 * KV append ([VP] §3.3, prefill step 3 and decode step 2: each new token's K
 * and V are written to the physical slot its block table maps it to):
 *     k_cache[slot / block_size, slot % block_size, :, :] = k[t, :, :]   (same for v)
 * for every token t with slot = slot_mapping[t] >= 0; negative slots are
 * skipped (padding). Slots >= num_blocks*block_size are skipped and flagged
 * PKV_ERR_DEVICE_BOUNDS. Two tokens with the same slot in one call race.
 *
 *   k, v           device, [num_tokens, num_kv_heads, head_dim], dtype
 *   k_cache,v_cache device, [num_blocks, block_size, num_kv_heads, head_dim], dtype
 *   slot_mapping   device int64 [num_tokens]
 * num_tokens may be 0 (nothing is launched).
 */
pkv_status pkv_reshape_and_cache(
    const void* k, const void* v, void* k_cache, void* v_cache, pkv_dtype dtype,
    const int64_t* slot_mapping, int num_tokens,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, void* stream);

/*
 * Block copy for copy-on-write ([VP] §4.1: the shared physical block is copied
 * to a fresh block for the sample that writes next):
 *     k_cache[dst[i]] = k_cache[src[i]],  v_cache[dst[i]] = v_cache[src[i]]
 * for i < num_pairs, every slot of the block. Destination ids must be distinct
 * and must not appear among the sources of the same call (the copies run in
 * parallel). Ids outside [0, num_blocks) are skipped and flagged
 * PKV_ERR_DEVICE_BOUNDS. dtype may be PKV_FP8_E4M3 (1-byte elements).
 *
 *   src_block_ids, dst_block_ids  device int64 [num_pairs]
 * num_pairs may be 0 (nothing is launched).
 */
pkv_status pkv_copy_blocks(
    void* k_cache, void* v_cache, pkv_dtype dtype,
    const int64_t* src_block_ids, const int64_t* dst_block_ids, int num_pairs,
    int block_size, int num_kv_heads, int head_dim, int num_blocks, void* stream);

/*
 * Block moves of a swap ([VP] §5.2: a preempted request's KV blocks go out to
 * CPU memory, freeing their GPU blocks, and come back when it resumes; [ENG]
 * §3.1 hands them to the cache engine as blocks_to_swap_out / blocks_to_swap_in):
 *     dst_k[dst[i]] = src_k[src[i]],  dst_v[dst[i]] = src_v[src[i]]
 * for i < num_pairs, every slot of the block, between two pools of the same
 * block shape [*, block_size, num_kv_heads, head_dim] and dtype.
 *
 *   src_k_cache, src_v_cache  [src_num_blocks, ...]: device memory, or page-locked
 *                             host memory (cudaHostAlloc / cudaHostRegister; the
 *                             kernel reads it through its mapped device address)
 *   dst_k_cache, dst_v_cache  [dst_num_blocks, ...]: the same choice
 *   src_block_ids, dst_block_ids  int64 [num_pairs], device or page-locked host
 * Swap-out is device -> host, swap-in host -> device; one kernel moves all pairs
 * over the host link, so scattered blocks need no per-block copy calls. Pageable
 * host memory, or K and V of one side in different kinds of memory, return
 * PKV_ERR_INVALID_ARG. Destination ids must be distinct; if both sides are the
 * same pool the rules of pkv_copy_blocks apply. Ids outside their pool are
 * skipped and flagged PKV_ERR_DEVICE_BOUNDS. The caller owns all memory and keeps
 * the host buffers alive until the stream has passed the call. num_pairs may be
 * 0 (nothing is launched); at most 65535 pairs per call.
 */
pkv_status pkv_swap_blocks(
    const void* src_k_cache, const void* src_v_cache, int src_num_blocks,
    void* dst_k_cache, void* dst_v_cache, int dst_num_blocks, pkv_dtype dtype,
    const int64_t* src_block_ids, const int64_t* dst_block_ids, int num_pairs,
    int block_size, int num_kv_heads, int head_dim, void* stream);

/*
 * Multi-query paged attention with a causal mask: several new query tokens per
 * sequence attend over the paged cache ([VP] §7.2 chunked prefill: a long
 * prompt joins the batch chunk by chunk, each chunk's K/V going into the
 * sequence's blocks; [VP] §7.5 and [ENG] §5.2 speculative decoding: the target
 * model checks the draft tokens, whose K/V sit in the same blocks).
 * The queries' own K/V must already be in the cache (pkv_reshape_and_cache), so
 * context_lens[s] counts them. Sequence s owns rows query_start[s] ..
 * query_start[s+1]-1 of q; with n_s = query_start[s+1] - query_start[s] and
 * c_s = context_lens[s], its i-th query sits at position c_s - n_s + i and
 *     out[row, h, :] = sum_{j <= c_s - n_s + i} softmax_j(scale q[row,h] . K_s[j,g]) V_s[j,g]
 * (g = h / group). n_s = 1 with c_s the context is a decode step.
 *
 *   out            device, [num_tokens, num_q_heads, head_dim], out_dtype (f32 or bf16)
 *   q              device, [num_tokens, num_q_heads, head_dim], bf16
 *   k_cache,v_cache device, [num_blocks, block_size, num_kv_heads, head_dim], kv_dtype (bf16)
 *   block_tables   device int32 [num_seqs, max_blocks_per_seq]
 *   context_lens   device int32 [num_seqs]
 *   query_start    device int32 [num_seqs + 1], non-decreasing, query_start[0] >= 0,
 *                  query_start[num_seqs] <= num_tokens
 *   max_query_len  host upper bound of n_s (sizes the grid); max_context_len as in
 *                  pkv_paged_attention_decode (0 = the table capacity)
 *   partition_tokens  > 0 fixed KV partitions, 0 chosen from the shapes (no
 *                  persistent schedule); the workspace is sized by
 *                  pkv_paged_attention_multi_query_workspace_bytes.
 * Supported: bf16 caches, head_dim 64 or 128, groups 1, 2, 4, 8, 16, block sizes 8-64
 * (PKV_ERR_UNSUPPORTED otherwise). A sequence whose n_s, c_s or rows break the
 * rules above (n_s > c_s, n_s > max_query_len, c_s above the capacity, rows
 * outside q) is skipped and flagged PKV_ERR_DEVICE_BOUNDS in the device word; its
 * output rows are not written. Rows of q that belong to no sequence are not
 * written either.
 */
size_t pkv_paged_attention_multi_query_workspace_bytes(
    int num_seqs, int num_tokens, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int max_query_len, int max_context_len, int partition_tokens);

pkv_status pkv_paged_attention_multi_query(
    void* out, pkv_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
    pkv_dtype kv_dtype, const int32_t* block_tables, const int32_t* context_lens,
    const int32_t* query_start, float scale, int num_seqs, int num_tokens, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
    int max_query_len, int max_context_len, int partition_tokens, void* workspace,
    size_t workspace_bytes, void* stream);

/*
 * Decode attention over a batch whose sequences share a prefix (parallel
 * sampling after a copy-on-write fork: "为什么PagedAttention能让大模型推理吞吐量
 * 提升数倍", Memory Sharing). The result is pkv_paged_attention_decode's
 * (softmax over each sequence's whole context), computed as a cascade that
 * reads the shared blocks once instead of once per sequence: the B queries
 * attend to the prefix as one block of B x group rows per KV head (its tokens
 * cut into partitions of whole 128-token tiles, at most one wave of the prefix
 * call's CTAs: KV heads x 128-row tiles x partitions, each writing a partial),
 * then each query to its own tail, longest tail first, merging the prefix's
 * partials into its result by the exact log-sum-exp rule before it writes the
 * output. Three kernels on `stream`, no host synchronisation. The cascade is not
 * a step of the pages' method (their kernel walks each sequence's table).
 *
 *   prefix_tokens  host; the first prefix_tokens / block_size entries of every
 *                  row of block_tables are the same blocks (the caller's
 *                  contract; row 0's are read); a multiple of block_size,
 *                  below max_context_len.
 *   context_lens   device int32 [num_seqs], each in (prefix_tokens,
 *                  max_context_len]; a length outside is flagged
 *                  PKV_ERR_DEVICE_BOUNDS and read as the nearest valid one.
 *   workspace      device, >= pkv_paged_attention_shared_prefix_workspace_bytes
 *                  bytes (for the same batch, heads and prefix_tokens), 256-byte
 *                  aligned; scratch between calls. The size function returns
 *                  (size_t)-1 for arguments it cannot size.
 * Other arguments as pkv_paged_attention_decode. Supported: bf16 caches, head_dim
 * 128, groups 1, 2, 4, 8, 16, block sizes 8-64, num_seqs x group >= 32 (the
 * prefix runs on the tcgen05 multi-query kernel), num_seqs <= 65535;
 * PKV_ERR_UNSUPPORTED otherwise. Host-side argument errors (a prefix that is not
 * whole blocks or reaches max_context_len, a table too narrow for
 * max_context_len, a null or misaligned pointer, a small workspace) return
 * PKV_ERR_INVALID_ARG before any launch.
 */
size_t pkv_paged_attention_shared_prefix_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                                        int head_dim, int prefix_tokens);

pkv_status pkv_paged_attention_decode_shared_prefix(
    void* out, pkv_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int prefix_tokens, float scale,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, void* workspace,
    size_t workspace_bytes, void* stream);

/*
 * FP8 KV append ("vLLM PagedAttention 深度解析" §7.4: K/V stored as FP8 so a block
 * holds twice the tokens). Same addressing as pkv_reshape_and_cache; the caches
 * hold e4m3 codes (1 byte per element) and the stored code of an element x is
 * e4m3(float32(x * float32(1 / scale))), rounded to nearest even, finite values
 * beyond the e4m3 range saturating to +-448. The value a code stands for is
 * decode(code) * scale. One scale per tensor: k_scale for K, v_scale for V
 * (finite, > 0). k, v are bf16 or f32 (in_dtype), [num_tokens, Hkv, D];
 * Hkv * D must be a multiple of 16.
 */
pkv_status pkv_reshape_and_cache_fp8(
    const void* k, const void* v, pkv_dtype in_dtype, void* k_cache, void* v_cache,
    float k_scale, float v_scale, const int64_t* slot_mapping, int num_tokens,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, void* stream);

/*
 * Reads and clears the current device's error word (0 or a pkv_status code set
 * by a kernel). Synchronises `stream` first. `code` is a host pointer.
 */
pkv_status pkv_get_device_error(int* code, void* stream);

/*
 * Test hook for the kernels' bounded waits (no counterpart on the pages; it
 * exists so that a test can watch a wait give up without faulting the GPU).
 * Arms a one-shot change of the NEXT launch of one kernel, made from any host
 * thread:
 *   kernel 0  the partitioned decode kernel of pkv_paged_attention_decode
 *             (partition_tokens >= 0): in its first CTA the producer never issues
 *             the copies of ring stage `index` (16 tokens, 32 for e4m3 caches) nor
 *             arrives on that stage's barrier;
 *   kernel 1  the tcgen05 multi-query kernel of pkv_paged_attention_multi_query
 *             (from 32 query rows per KV head, head_dim 128): in its first CTA
 *             the producer never issues the K copies of 128-token tile `index`.
 * Every bounded wait of that launch then gives up after wait_limit_ns
 * (100 us .. 2 s) instead of 2 s. No copy is left in flight: the withheld one is
 * never issued and the rest are drained. The launch records
 * PKV_ERR_DEVICE_TIMEOUT in the device error word (when the withheld stage is
 * reached, i.e. the first CTA has more than `index` stages or tiles), leaves its
 * output unspecified and releases everything it holds (shared memory, tensor
 * memory), so the next call on the stream runs normally.
 * index -1 disarms. Returns PKV_ERR_INVALID_ARG for another kernel id or a limit
 * outside the range.
 */
pkv_status pkv_test_withhold_copy(int kernel, int index, unsigned long long wait_limit_ns);

/* ------------------------------------------------------------------------- */
/* One decode step from host buffers ([VP] §3.3 decode, §4.1 copy-on-write)  */
/* ------------------------------------------------------------------------- */
/*
 * A step context owns what one decode step needs for up to max_seqs sequences:
 * two slots of device buffers (the step's q / new K,V / metadata / output), the
 * split-K workspace, two pinned metadata staging slots, and three streams (host
 * to device copies, kernels, device to host copies) with the events that order
 * them. Creating it allocates (once); pkv_decode_step allocates nothing.
 * partition_tokens is the schedule the steps will use (same meaning as in
 * pkv_paged_attention_decode). One context serves one caller stream at a time.
 */
typedef struct pkv_step_ctx pkv_step_ctx;
typedef struct pkv_block_manager pkv_block_manager;

/* kv_dtype PKV_FP8_E4M3: the caches hold e4m3 codes, the step's q / new K,V
 * are bf16 on the host, and k_scale / v_scale are the per-tensor scales
 * (ignored for f32 / bf16 caches). block_size: tokens per block of the caches
 * and of the block manager the steps will use (pkv_decode_step refuses a
 * manager with another block size). */
pkv_status pkv_step_ctx_create(int max_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int max_blocks_per_seq, int block_size, pkv_dtype kv_dtype, pkv_dtype out_dtype,
                               int partition_tokens, float k_scale, float v_scale, pkv_step_ctx** out);
void pkv_step_ctx_destroy(pkv_step_ctx* ctx);

/*
 * One decode step for the n listed sequences of `bm` (n <= max_seqs):
 *   1. the block manager appends one token to each sequence (slot mapping,
 *      copy-on-write pairs, block tables and lengths, in pinned staging);
 *   2. metadata, q [n, Hq, D], k and v [n, Hkv, D] are copied to the device
 *      (q_host, k_host, v_host are HOST pointers; pinned memory makes the copies
 *      asynchronous);
 *   3. pkv_copy_blocks for the copy-on-write pairs, pkv_reshape_and_cache for
 *      the new tokens, pkv_paged_attention_decode over the updated contexts;
 *   4. the output [n, Hq, D] (out_dtype of the context) reaches out_host: a
 *      page-locked out_host is written directly by the attention kernels through
 *      its device mapping (no copy after them); pageable memory gets a copy.
 * k_cache / v_cache are the device caches (the context's block_size).
 * Ordering: the step's device work starts after everything enqueued on `stream`
 * before the call, runs on the context's own streams, and `stream` passes the
 * step only once its output is in out_host: synchronise `stream` (or an event
 * recorded on it after the call) before reading out_host. Consecutive steps of
 * one context overlap on the device (step i + 1's host-to-device copies, and a
 * device-to-host copy if there is one, run while step i's kernels run), so a caller that
 * waits for step i - 1 after issuing step i keeps the copies off the critical
 * path; the host buffers of a step must stay untouched until `stream` has passed
 * it. A block manager error (PKV_ERR_OUT_OF_BLOCKS) is returned before anything
 * is enqueued.
 */
pkv_status pkv_decode_step(pkv_step_ctx* ctx, pkv_block_manager* bm, const int64_t* seq_ids, int n,
                           const void* q_host, const void* k_host, const void* v_host,
                           void* k_cache, void* v_cache, int num_blocks, float scale,
                           int partition_tokens, void* out_host, void* stream);

/*
 * Phase timing of the steps of a context (off by default; a measurement aid,
 * not part of the method). When enabled, each pkv_decode_step records the host
 * time of its block-manager work and CUDA events around its H2D copies, its
 * kernels and its D2H copy on the step's stream; pkv_step_ctx_last_timing waits
 * for the last timed step's D2H and writes, in milliseconds,
 *   out[0] host: block-manager append + block tables (host clock),
 *   out[1] H2D copies (metadata, q, new K and V), out[2] kernels (copy_blocks,
 *   KV append, attention), out[3] D2H copy of the output (device events).
 * PKV_ERR_INVALID_ARG if no step ran with timing enabled since it was enabled.
 */
pkv_status pkv_step_ctx_set_timing(pkv_step_ctx* ctx, int enable);
pkv_status pkv_step_ctx_last_timing(pkv_step_ctx* ctx, float* out);

/* ------------------------------------------------------------------------- */
/* Host block manager ([ENG] §2.3; [VP] §3.3, §4.1, §4.2; [BT])              */
/* ------------------------------------------------------------------------- */
/*
 * Plain host memory, not thread-safe (one manager per scheduler thread).
 * Sequences are named by caller-chosen int64 ids. All array arguments here are
 * HOST pointers.
 *
 * Free list: FIFO of block ids, taken from the front, returned to the back
 * ([ENG] §2.3). Reference counts: a block shared by k sequences has count k;
 * a block whose count falls to 0 goes back to the free list ([VP] §4.2).
 */
/* free_order: the initial free-list order (a permutation of 0..num_blocks-1),
 * or NULL for 0,1,2,... The manager copies it. */
pkv_status pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                         pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* bm);

/* New sequence of num_tokens prompt tokens: takes ceil(num_tokens/block_size)
 * blocks and writes the slot of every prompt token to slots_out (may be NULL).
 * PKV_ERR_OUT_OF_BLOCKS (nothing taken) if the free list is too short;
 * PKV_ERR_INVALID_ARG if seq_id already exists. */
pkv_status pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, int num_tokens,
                           int64_t* slots_out);

/* One decode step: appends one token to each listed sequence, in order, and
 * writes its slot to slot_mapping_out[i]. A sequence whose last block still has
 * room writes into it, after a copy-on-write if that block is shared (the
 * (src, dst) pair is appended to copy_src_out/copy_dst_out, capacity n); a full
 * last block gets a new block. *num_copies_out receives the number of pairs.
 * On PKV_ERR_OUT_OF_BLOCKS, *num_done_out sequences were appended and the rest
 * untouched. num_done_out may be NULL. */
pkv_status pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int64_t* slot_mapping_out, int64_t* copy_src_out,
                               int64_t* copy_dst_out, int* num_copies_out, int* num_done_out);

/* Copy-on-write of one logical block of a sequence: if its physical block is
 * shared, the sequence gets a fresh block and (*src, *dst) is the copy to run;
 * otherwise *src = *dst = -1. */
pkv_status pkv_bm_make_writable(pkv_block_manager* bm, int64_t seq_id, int logical_block,
                                int64_t* src, int64_t* dst);

/* child shares all of parent's blocks (each count + 1) and its length. */
pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child);

/* Drops a sequence: each of its blocks' counts falls by one, blocks at 0 return
 * to the back of the free list in table order. */
pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);

/* Block tables and lengths of the listed sequences, rows of max_blocks int32
 * entries padded with 0, ready to copy to the device. PKV_ERR_INVALID_ARG if a
 * sequence has more than max_blocks blocks. context_lens_out may be NULL. */
pkv_status pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int max_blocks, int32_t* tables_out, int32_t* context_lens_out);

/*
 * Host (CPU) block pool for swapping ([VP] §5.2). Set once, before any swap:
 * num_host_blocks ids with their own FIFO free list (free_order or NULL for
 * 0,1,2,...) and reference counts.
 */
pkv_status pkv_bm_set_host_pool(pkv_block_manager* bm, int num_host_blocks, const int32_t* free_order);

/*
 * Swap-out of a group of resident sequences: every distinct device block their
 * tables reference gets one host block (taken in order of first appearance,
 * sequences in the given order, tables in order), written as the pair
 * (dev_blocks_out[i], host_blocks_out[i]) for the copy; each reference moves its
 * count from the device block (freed at 0, so blocks still used by a sequence
 * left behind stay) to the host block. The sequences become swapped out: their
 * tables hold host ids, and append, fork, make_writable and block_tables refuse
 * them (PKV_ERR_INVALID_ARG); pkv_bm_free releases their host blocks.
 * capacity: room in each output array (the group's total block count always
 * suffices). All or nothing: PKV_ERR_OUT_OF_BLOCKS if the host pool has too few
 * free blocks; PKV_ERR_INVALID_ARG for an unknown, repeated or swapped-out id.
 */
pkv_status pkv_bm_swap_out(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* dev_blocks_out,
                           int64_t* host_blocks_out, int capacity, int* num_pairs_out);

/* The mirror image for swapped-out sequences: pairs (host, device). */
pkv_status pkv_bm_swap_in(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* host_blocks_out,
                          int64_t* dev_blocks_out, int capacity, int* num_pairs_out);

int pkv_bm_num_free_host(const pkv_block_manager* bm);
int pkv_bm_host_ref_count(const pkv_block_manager* bm, int block);
/* 1 swapped out, 0 resident, -1 unknown. */
int pkv_bm_is_swapped(const pkv_block_manager* bm, int64_t seq_id);

/* Tokens per block of the manager, or -1 for NULL. */
int pkv_bm_block_size(const pkv_block_manager* bm);
int pkv_bm_num_free(const pkv_block_manager* bm);
int pkv_bm_ref_count(const pkv_block_manager* bm, int block);
/* Number of tokens of a sequence, or -1 if unknown. */
int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
