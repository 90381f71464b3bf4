// Paged decode attention for sm_100a.
//
// What it computes ("LLM 推理引擎内部原理" §2.4; "为什么PagedAttention能让大模型推理吞吐量
// 提升数倍", section "Block Table：GPU上的页表"): for each sequence s and query head
// h, softmax(scale * q[s,h] . K_s^T) V_s over the sequence's logical tokens,
// where logical token j lives in physical block block_tables[s][j / bs] at
// offset j % bs of a cache laid out [num_blocks, bs, Hkv, D].
//
// How (B200 design, not the pages' sketch, which reads one scalar per thread
// per token and leaves the softmax out):
//   * Work item = (sequence, KV head, partition of the context). The grid is
//     (Hkv, partitions, sequences), so the CTAs reading the different heads of
//     the same physical blocks run side by side.
//   * One producer warp walks the partition's slice of the block table (32 ids
//     per coalesced load) and issues one 4-D TMA tile load per block for K and
//     V into a ring of shared-memory stages (mbarrier completion, L2
//     evict-first since the cache is streamed once). No multicast anywhere.
//   * Consumer warps take whole blocks round-robin, each with its own online
//     softmax state (running max m, sum l, accumulator), merged at the end.
//       - SIMT path (fp32 caches, or MHA): 8 lanes per token, 16-byte shared
//         loads, warp-shuffle QK reductions, fp32 FMA.
//       - Tensor-core path (bf16, grouped queries): per block of 16 tokens,
//         S^T = K Q^T with mma.m16n8k16 (16 tokens x 8 query heads), online
//         softmax on the fragments, then O^T += V^T P^T, P split into bf16
//         high + low parts so the probabilities keep ~16 bits.
//   * Partitions: a context longer than one partition is split; each CTA
//     writes (o / l, m, l) for its partition and a second kernel merges them
//     exactly: M = max m_c, w_c = l_c 2^(m_c - M), out = sum w_c o_c / sum w_c.
//     (The split and the log-sum-exp merge are not on the pages; they are the
//     standard exact identity.)
//   * Logits are kept in the log2 domain (scale * log2(e) folded in), so the
//     exponentials are single ex2 instructions.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <type_traits>

#include "attention_common.cuh"
#include "plan_units.cuh"

namespace pkv {
namespace attn {

// Log-sum-exp merge of partition results. grid = (Hq, B), block = GROUPS x D
// threads. The (m, l) pairs are staged in shared memory once (coalesced), the
// weights w_c = l_c 2^(m_c - M) computed once per row; then each group of D
// threads (one thread per dimension) sums over every GROUPS-th partition with
// eight independent loads in flight, and the groups' sums are added. Calls with
// many partitions per context take four groups (one group walking 50
// partitions four loads at a time took 12.5 us of mostly DRAM latency on the
// long-context workload, four groups with eight loads each 9.0 us, ncu); calls
// with a few partitions take one group (fewer threads to launch).
constexpr int kMergeSmemParts = 2048;
constexpr int kMergeManyParts = 8;      // partitions per context from which four groups are launched
//
// Launched as a programmatic dependent of the partition kernel: the launch is
// staged while that kernel runs, and the CTAs wait here until its grid has
// completed and the partials are visible (a no-op for a plain launch). The
// context length is read before that wait: it is an input of the call, final
// before the partition grid started. After the wait every load of the fast
// path is issued at once (each group's first eight partials with the (m, l)
// pairs), so one memory latency, not four dependent ones, separates the wait
// from the sums.
template <int D, int GROUPS>
__global__ void __launch_bounds__(GROUPS * D) merge_partitions_kernel(const Params p) {
    constexpr int NT = GROUPS * D;
    constexpr int kMergeGroups = GROUPS;
    __shared__ float sw[kMergeSmemParts];                        // m_c, then the weights w_c
    __shared__ float sl[kMergeSmemParts];                        // l_c
    __shared__ float s_red[NT / 32];
    __shared__ float s_o[GROUPS > 1 ? GROUPS - 1 : 1][D];
    const int qhead = blockIdx.x, seq = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    const int grp = tid / D, d = tid - grp * D;
    int ctx = p.context_lens[seq];
    ctx = ctx < 0 ? 0 : (ctx > p.ctx_cap ? p.ctx_cap : ctx);
    const int nparts = ((ctx + p.block_size - 1) / p.block_size + p.part_blocks - 1) / p.part_blocks;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (nparts <= 1) return;
    const int64_t qh = (int64_t)seq * p.num_q_heads + qhead;
    const float* ml = p.ws_ml + qh * p.num_parts * 2;
    const float* o = p.ws_o + qh * p.num_parts * D + d;
    float L = 0.f, O = 0.f;
    if (nparts <= kMergeSmemParts) {
        // this group's partitions grp, grp + GROUPS, ...: the first eight loaded now
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = grp + u * kMergeGroups;
            v[u] = c < nparts ? o[(int64_t)c * D] : 0.f;
        }
        // M = max m_c
        float mx = kNegInf;
        for (int c = tid; c < nparts; c += NT) {
            const float2 e = *reinterpret_cast<const float2*>(ml + 2 * c);
            sw[c] = e.x;
            sl[c] = e.y;
            mx = fmaxf(mx, e.x);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) s_red[wid] = mx;
        __syncthreads();
        float M = s_red[0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, s_red[w]);
        __syncthreads();
        if (M != kNegInf) {                                      // uniform over the CTA
            float ls = 0.f;
            for (int c = tid; c < nparts; c += NT) {             // the entries this thread staged
                const float mc = sw[c];
                const float w = mc == kNegInf ? 0.f : sl[c] * fast_exp2(mc - M);
                sw[c] = w;
                ls += w;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
            if (lane == 0) s_red[wid] = ls;
            __syncthreads();
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) L += s_red[w];
            float acc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = grp + u * kMergeGroups;
                acc[u] = c < nparts ? sw[c] * v[u] : 0.f;
            }
            // the rest, eight loads issued before they are used
            int c = grp + 8 * kMergeGroups;
            for (; c + 7 * kMergeGroups < nparts; c += 8 * kMergeGroups) {
                float x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = o[(int64_t)(c + u * kMergeGroups) * D];
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[u] += sw[c + u * kMergeGroups] * x[u];
            }
            for (; c < nparts; c += kMergeGroups) acc[0] += sw[c] * o[(int64_t)c * D];
            O = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        }
        if constexpr (GROUPS > 1) {
            if (grp > 0) s_o[grp - 1][d] = O;
            __syncthreads();
            if (grp > 0) return;
#pragma unroll
            for (int g = 0; g < GROUPS - 1; ++g) O += s_o[g][d];
        }
    } else {
        if (grp > 0) return;
        float M = kNegInf;
        for (int c = 0; c < nparts; ++c) M = fmaxf(M, ml[2 * c]);
        if (M != kNegInf) {
            for (int c = 0; c < nparts; ++c) {
                const float mc = ml[2 * c];
                if (mc == kNegInf) continue;
                const float w = ml[2 * c + 1] * fast_exp2(mc - M);
                L += w;
                O += w * o[(int64_t)c * D];
            }
        }
    }
    store_out(p, qh * D + d, L > 0.f ? O / L : 0.f);
}

// ---------------------------------------------------------------------------
// Longest-first schedule of the partitioned kernel (one CTA; plan_units.cuh).
// It flags lengths outside [0, ctx_cap] and lists them clamped.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads) plan_units_kernel(const Params p) {
    // the partition kernel may start its CTAs now; they wait for the list in-kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int cap = p.ctx_cap;
    list_units(
        [&](int sq, bool first) {
            int ctx = p.context_lens[sq];
            if (ctx < 0 || ctx > cap) {
                if (first) flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                ctx = ctx < 0 ? 0 : cap;
            }
            return ctx;
        },
        p.num_seqs, p.part_blocks, p.block_size, p.units, p.unit_count);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Tensor map over a cache [NB, bs, Hkv, D] of 4-, 2- or 1-byte elements: box =
// piece_rows(bs) tokens of one head (a whole block, or a slice of a block longer
// than a ring stage), the whole row (SIMT) or 128-byte box rows with the 128-byte
// swizzle (tensor-core path).
bool make_cache_map(CUtensorMap* map, const void* base, pkv_dtype dt, int nb, int bs, int hkv, int d, bool mma,
                    int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t eb = dt == PKV_F32 ? 4 : (dt == PKV_BF16 ? 2 : 1);
    const CUtensorMapDataType ty = dt == PKV_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)hkv, (cuuint64_t)bs, (cuuint64_t)nb};
    cuuint64_t strides[3] = {d * eb, (cuuint64_t)hkv * d * eb, (cuuint64_t)bs * hkv * d * eb};
    const int rows = box_rows > 0 ? box_rows : piece_rows(bs, (int)eb);
    if (rows > 256 || bs % rows != 0) return false;
    cuuint32_t box[4] = {(cuuint32_t)(mma ? 128 / eb : d), 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, ty, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    mma ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static std::atomic<int> cached{0};
    int v = cached.load();
    if (v) return v;
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached.store(n);
    return n;
}

struct Plan {
    int ctx_cap, part_tokens, num_parts;
    bool persistent;
    int grid;           // CTAs of the persistent schedule
    int team_size;      // CTAs per team (one KV head each)
    bool longest_first; // partitioned: the plan kernel lists the units (plan_units_kernel)
};

// Bytes of the unit list at the front of the workspace (longest-first schedule).
size_t units_bytes(int num_seqs, const Plan& pl) {
    if (!pl.longest_first) return 0;
    return (((size_t)num_seqs * pl.num_parts * sizeof(uint2) + sizeof(int)) + 255) & ~size_t(255);
}

// Schedule for one call.
//   partition_tokens > 0  : fixed partitions of that many tokens (+ merge kernel).
//   partition_tokens == 0 : fixed partitions chosen here: the fewest that still
//                           give about one wave of work items (see below).
//                           Measured on B200: fewer, longer partitions stream
//                           fastest (no merge pass, fewer CTA start-ups).
//   partition_tokens == -1: the persistent, evenly split schedule (at most 2048
//                           sequences and < 2^31 tiles).
bool plan(int num_seqs, int num_kv_heads, int block_size, int max_blocks, int max_context_len,
          int partition_tokens, Plan* pl) {
    if (num_seqs <= 0 || num_kv_heads <= 0 || !block_size_built(block_size) || max_blocks <= 0 ||
        partition_tokens < -1 || (partition_tokens == -1 && block_size != 16))
        return false;
    const int BS = block_size;
    const int64_t cap_tbl = (int64_t)max_blocks * block_size;
    if (cap_tbl > INT32_MAX) return false;
    int cap = (int)cap_tbl;
    if (max_context_len > 0) cap = std::min(cap, max_context_len);
    pl->ctx_cap = cap;
    pl->persistent = false;
    pl->grid = 0;
    pl->team_size = 0;
    pl->longest_first = false;
    if (partition_tokens == -1) {
        const int64_t max_tiles = (int64_t)num_seqs * num_kv_heads * ((cap + BS - 1) / BS);
        if (num_seqs > persistent_max_seqs() || max_tiles >= INT32_MAX) return false;
        pl->persistent = true;
        // teams of Hkv CTAs (one KV head each); as many whole teams as fit two CTAs per SM
        const int slots = num_sms() * persistent_ctas_per_sm();
        pl->team_size = num_kv_heads;
        pl->grid = std::max(1, slots / num_kv_heads) * num_kv_heads;
        pl->part_tokens = 0;
        pl->num_parts = 1;
        return true;
    }
    int pt = partition_tokens;
    if (pt == 0) {
        // The fewest partitions whose units fill about one wave of the decode
        // kernel (three CTAs per SM), never shorter than 256 tokens (when even
        // those give less than a wave, the shortest split that stays at or above
        // 256 tokens, so no ragged sliver is left over). A sequence's
        // partitions are estimated with context lengths spread evenly over
        // [cap / 2, cap] (16 sample lengths), or at cap for a single sequence.
        // With the longest-first order one wave of long units streams faster
        // than more, shorter ones plus their merge (B200, 70B-shaped GQA: 128
        // sequences 6179 GB/s with one partition vs 5703 with two; 32 sequences
        // 4829 with two vs 3405 with one and 4324 with four).
        const int64_t target = 3ll * num_sms();
        pt = std::max(256, (cap + BS - 1) / BS * BS);
        for (int nparts = 1; nparts <= 65535; ++nparts) {
            const int cand = (int)(((int64_t)(cap + nparts - 1) / nparts + BS - 1) / BS * BS);
            if (cand < 256) break;
            pt = cand;
            int64_t per_seq16 = 0;                                  // 16 x a sequence's expected partitions
            for (int i = 0; i < 16; ++i) {
                const int64_t len = num_seqs == 1 ? cap : cap / 2 + ((int64_t)cap * (2 * i + 1)) / 64;
                per_seq16 += (len + cand - 1) / cand;
            }
            if ((int64_t)num_seqs * num_kv_heads * per_seq16 >= 16 * target) break;
        }
    }
    pt = ((pt + BS - 1) / BS) * BS;
    int parts = (cap + pt - 1) / pt;
    if (parts < 1) parts = 1;
    if (parts > 65535) return false;
    pl->part_tokens = pt;
    pl->num_parts = parts;
    // Longest-first order whenever there is more than one sequence to order and
    // the unit list fits a grid dimension (65535 rows).
    pl->longest_first = num_seqs >= 2 && (int64_t)num_seqs * parts <= 65535 && pt / BS <= kPlanMaxBins;
    return true;
}

size_t ws_bytes_for(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, const Plan& pl) {
    if (pl.persistent) {
        const int group = num_q_heads / num_kv_heads;
        const size_t parts = (((size_t)2 * pl.grid * group * (head_dim + 2) * 4) + 255) & ~size_t(255);
        return parts + (size_t)num_seqs * num_kv_heads * 8;
    }
    const size_t ub = units_bytes(num_seqs, pl);
    if (pl.num_parts <= 1) return ub;
    const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
    const size_t o_bytes = ((rows * head_dim * 4) + 255) & ~size_t(255);
    return ub + o_bytes + rows * 2 * 4;
}

}  // namespace attn
}  // namespace pkv

extern "C" {

size_t pkv_paged_attention_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq, int max_context_len,
                                           int partition_tokens) {
    pkv::attn::Plan pl;
    if (num_q_heads <= 0 || head_dim <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        !pkv::attn::plan(num_seqs, num_kv_heads, block_size, max_blocks_per_seq, max_context_len,
                         partition_tokens, &pl))
        return (size_t)-1;
    return pkv::attn::ws_bytes_for(num_seqs, num_q_heads, num_kv_heads, head_dim, pl);
}

int pkv_paged_attention_partition_tokens(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                         int block_size, int max_blocks_per_seq, int max_context_len,
                                         int partition_tokens) {
    (void)num_q_heads;
    (void)head_dim;
    pkv::attn::Plan pl;
    if (!pkv::attn::plan(num_seqs, num_kv_heads, block_size, max_blocks_per_seq, max_context_len,
                         partition_tokens, &pl))
        return -1;
    return pl.part_tokens;
}

}  // extern "C"

namespace pkv {
namespace attn {

// One decode call. kv_dtype: the cache storage (f32, bf16 or fp8 e4m3); q is
// kv_dtype for f32 / bf16 caches and bf16 for an fp8 cache, whose K and V
// scales fold into the logit scale and the output.
pkv_status decode_tails_with_prefix(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* block_tables, const uint2* units,
                                    float scale, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int num_blocks, int ctx_cap,
                                    const float* pre_o, const float* pre_ml, int pre_parts, cudaStream_t st) {
    const int group = num_q_heads / num_kv_heads;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    const bool use_mma = group >= 2;
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, k_cache, PKV_BF16, num_blocks, block_size, num_kv_heads, head_dim, use_mma) ||
        !make_cache_map(&mv, v_cache, PKV_BF16, num_blocks, block_size, num_kv_heads, head_dim, use_mma))
        return PKV_ERR_CUDA;
    Params p{};
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = nullptr;                                   // each unit carries its (tail) length
    p.err = err;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out_scale = 1.0f;
    p.out_f32 = out_dtype == PKV_F32;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.max_blocks = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.ctx_cap = ctx_cap;
    p.block_size = block_size;
    p.part_blocks = std::max(1, (ctx_cap + block_size - 1) / block_size);   // one partition per sequence
    p.num_parts = 1;
    p.num_seqs = num_seqs;
    p.units = const_cast<uint2*>(units);
    p.unit_count = const_cast<int*>(reinterpret_cast<const int*>(units + num_seqs));
    p.pre_o = pre_o;
    p.pre_ml = pre_ml;
    p.pre_parts = pre_parts;
    p.withhold = -1;
    p.wait_ns = kDefaultWaitNs;
    const dim3 grid(num_kv_heads, num_seqs, 1);                 // row y takes listed unit y
    cudaError_t e;
    switch (block_size) {
        case 8: e = dispatch_partitioned<8>(PKV_BF16, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        case 16: e = dispatch_partitioned<16>(PKV_BF16, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        case 32: e = dispatch_partitioned<32>(PKV_BF16, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        default: e = dispatch_partitioned<64>(PKV_BF16, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
    }
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status decode_impl(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
                       pkv_dtype kv_dtype, float k_scale, float v_scale, const int32_t* block_tables,
                       const int32_t* context_lens, float scale, int num_seqs, int num_q_heads, int num_kv_heads,
                       int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len,
                       int partition_tokens, void* workspace, size_t workspace_bytes, void* stream) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
        max_context_len < 0 || partition_tokens < -1 || !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if (out_dtype != PKV_F32 && out_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    const bool fp8 = kv_dtype == PKV_FP8_E4M3;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (fp8 && (head_dim != 128 || partition_tokens == -1)) return PKV_ERR_UNSUPPORTED;
    if (!block_size_built(block_size) || (partition_tokens == -1 && block_size != 16)) return PKV_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return PKV_ERR_UNSUPPORTED;
    if (partition_tokens == -1 && group > 8) return PKV_ERR_UNSUPPORTED;   // persistent: one 8-wide head tile
    if (num_seqs == 0) return PKV_OK;
    if (num_seqs > 65535) return PKV_ERR_UNSUPPORTED;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    auto al = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; };
    if (!al(out) || !al(q) || !al(k_cache) || !al(v_cache)) return PKV_ERR_INVALID_ARG;

    Plan pl;
    if (!plan(num_seqs, num_kv_heads, block_size, max_blocks_per_seq, max_context_len, partition_tokens, &pl))
        return PKV_ERR_INVALID_ARG;
    const size_t need = ws_bytes_for(num_seqs, num_q_heads, num_kv_heads, head_dim, pl);
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return PKV_ERR_INVALID_ARG;

    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;

    const bool bf16 = kv_dtype == PKV_BF16;
    // tensor cores for grouped bf16 and for every e4m3 cache (MHA included: the
    // f16 MMA path decodes codes with one cvt per pair, measured 2-3 % faster than
    // the CUDA-core consumer at group 1)
    const bool use_mma = (bf16 && group >= 2) || fp8;
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, k_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, use_mma) ||
        !make_cache_map(&mv, v_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, use_mma))
        return PKV_ERR_CUDA;

    Params p{};
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.err = err;
    p.scale_log2 = scale * 1.4426950408889634f * (fp8 ? k_scale : 1.0f);
    p.out_scale = fp8 ? v_scale : 1.0f;
    p.out_f32 = out_dtype == PKV_F32;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.max_blocks = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.ctx_cap = pl.ctx_cap;
    p.block_size = block_size;
    p.part_blocks = pl.part_tokens / block_size;
    p.num_parts = pl.num_parts;
    p.num_seqs = num_seqs;
    p.withhold = -1;
    p.wait_ns = kDefaultWaitNs;
    if (!pl.persistent) take_wait_hook(0, &p.withhold, &p.wait_ns);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (pl.persistent) {
        static std::atomic<unsigned long long> epoch{1};
        p.ws_part = static_cast<float*>(workspace);
        p.counters = reinterpret_cast<unsigned long long*>(
            static_cast<uint8_t*>(workspace) +
            ((((size_t)2 * pl.grid * group * (head_dim + 2) * 4) + 255) & ~size_t(255)));
        p.epoch = epoch.fetch_add(1) & ((1ull << 40) - 1);
        p.team_size = pl.team_size;
        // The arrival counters start at zero on every call. The epoch tag alone
        // cannot tell a counter from other bytes a previous call (a split-K call
        // sharing this workspace) left there, so they are cleared on the stream.
        if (cudaMemsetAsync(p.counters, 0, (size_t)num_seqs * num_kv_heads * sizeof(unsigned long long), st) !=
            cudaSuccess)
            return PKV_ERR_CUDA;
        if (launch_persistent(bf16, use_mma, head_dim, group, mk, mv, p, pl.grid, st) != cudaSuccess)
            return PKV_ERR_CUDA;
        return PKV_OK;
    }
    const size_t ub = units_bytes(num_seqs, pl);
    if (pl.num_parts > 1) {
        const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
        p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ub);
        p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ub +
                                           (((rows * head_dim * 4) + 255) & ~size_t(255)));
    }
    dim3 grid(num_kv_heads, pl.num_parts, num_seqs);
    cudaError_t e;
    if (pl.longest_first) {
        p.units = static_cast<uint2*>(workspace);
        p.unit_count = reinterpret_cast<int*>(p.units + (size_t)num_seqs * pl.num_parts);
        plan_units_kernel<<<1, kPlanThreads, 0, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return PKV_ERR_CUDA;
        grid = dim3(num_kv_heads, num_seqs * pl.num_parts, 1);
    }
    switch (block_size) {
        case 8: e = dispatch_partitioned<8>(kv_dtype, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        case 16: e = dispatch_partitioned<16>(kv_dtype, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        case 32: e = dispatch_partitioned<32>(kv_dtype, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
        default: e = dispatch_partitioned<64>(kv_dtype, use_mma, head_dim, group, num_kv_heads, mk, mv, p, grid, st); break;
    }
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    if (pl.num_parts > 1) {
        // programmatic dependent launch: the merge grid's CTAs wait for the
        // partition grid in-kernel instead of behind a full kernel boundary
        cudaLaunchConfig_t cfg = {};
        const int groups = pl.num_parts >= kMergeManyParts ? 4 : 1;
        cfg.gridDim = dim3(num_q_heads, num_seqs);
        cfg.blockDim = dim3(groups * head_dim);
        cfg.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (groups == 4)
            e = head_dim == 128 ? cudaLaunchKernelEx(&cfg, merge_partitions_kernel<128, 4>, p)
                                : cudaLaunchKernelEx(&cfg, merge_partitions_kernel<64, 4>, p);
        else
            e = head_dim == 128 ? cudaLaunchKernelEx(&cfg, merge_partitions_kernel<128, 1>, p)
                                : cudaLaunchKernelEx(&cfg, merge_partitions_kernel<64, 1>, p);
        if (e != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // namespace attn
}  // namespace pkv

extern "C" {

pkv_status pkv_paged_attention_decode(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                      const void* v_cache, pkv_dtype kv_dtype, const int32_t* block_tables,
                                      const int32_t* context_lens, float scale, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                      int num_blocks, int max_context_len, int partition_tokens,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    if (kv_dtype != PKV_F32 && kv_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    return pkv::attn::decode_impl(out, out_dtype, q, k_cache, v_cache, kv_dtype, 1.0f, 1.0f, block_tables,
                                  context_lens, scale, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                  max_blocks_per_seq, num_blocks, max_context_len, partition_tokens, workspace,
                                  workspace_bytes, stream);
}

pkv_status pkv_paged_attention_decode_fp8(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                          const void* v_cache, float k_scale, float v_scale,
                                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                                          int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_blocks_per_seq, int num_blocks,
                                          int max_context_len, int partition_tokens, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
        return PKV_ERR_INVALID_ARG;
    return pkv::attn::decode_impl(out, out_dtype, q, k_cache, v_cache, PKV_FP8_E4M3, k_scale, v_scale, block_tables,
                                  context_lens, scale, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                  max_blocks_per_seq, num_blocks, max_context_len, partition_tokens, workspace,
                                  workspace_bytes, stream);
}

}  // extern "C"
