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

namespace pkv {
namespace attn {

// ---------------------------------------------------------------------------
// The pipelined kernel.
//   PATH 0: SIMT, block-split (each consumer warp takes whole blocks, HPW = group)
//   PATH 1: SIMT, head-split (every warp reads every block, HPW = group / NCW)
//   PATH 2: tensor cores, block-split (group <= 8)
// ---------------------------------------------------------------------------
template <typename T, int D, int PATH, int HPW, int STAGES, int KPC = 1>
struct Kern {
    static constexpr bool kMma = PATH == 2;
    static constexpr int TILE = BS * D * (int)sizeof(T);              // one block, one head, K or V
    static constexpr int BOX = 128 / (int)sizeof(T);                   // elements per swizzled 128-byte box row
    static constexpr int NBOX = D * (int)sizeof(T) / 128;              // boxes per row (tensor-core path)
    // FP8 tiles are half the size: two physical blocks share a stage, so a stage
    // is 8 KB and a consumer folds 32 tokens per step (K rows of both blocks
    // first, then V rows).
    static constexpr int BPS = sizeof(T) == 1 ? 2 : 1;                  // blocks per stage
    static constexpr int TOK = BS * BPS;
    // KPC KV heads per CTA: their tiles are loaded back to back, so a token row's
    // neighbouring heads (adjacent in HBM) are read together; consumer warps split
    // by head (WPH warps per head). Stage layout: K [head][block][tile], then V.
    static constexpr int WPH = NCW / KPC;
    static constexpr int STAGE_BYTES = 2 * BPS * KPC * TILE;
    static_assert(PATH != 1 || KPC == 1, "head-split consumers serve one KV head");
    static constexpr int RING = STAGES * STAGE_BYTES;
    static constexpr int NSLOT = PATH == 1 ? 1 : NCW;                  // partial states to merge
    static constexpr int MAXG = PATH == 2 ? 8 : (PATH == 1 ? HPW * NCW : HPW);
    static constexpr int RED = NSLOT * MAXG * (D + 2) * 4;
    static constexpr int BODY = RING > RED ? RING : RED;
    static constexpr int SMEM = 1024 /*align slack*/ + BODY + 2 * STAGES * 8;
    static_assert(RED <= BODY, "reduction scratch must fit");
    // Block-split consumers take tiles round-robin; with STAGES a multiple of NCW
    // every round of a stage goes to the same warp, so no warp can wait on a ring
    // phase two rounds ahead of the producer (the parity wait would pass early).
    static_assert(PATH == 1 || STAGES % WPH == 0, "ring depth must be a multiple of the warps per head");
};

template <typename T, int D, int PATH, int HPW, int STAGES, int KPC>
__global__ void __launch_bounds__(NTHREADS, 3)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const Params p) {
    using K = Kern<T, D, PATH, HPW, STAGES, KPC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::BODY);
    uint64_t* empty = full + STAGES;
    __shared__ volatile int s_abort;

    const int kvh = blockIdx.x * KPC, part = blockIdx.y, seq = blockIdx.z;   // first KV head of this CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    int ctx = p.context_lens[seq];
    if (ctx < 0 || ctx > p.ctx_cap) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
        ctx = ctx < 0 ? 0 : p.ctx_cap;
    }
    const int nblk_seq = (ctx + BS - 1) / BS;
    const int nparts = (nblk_seq + p.part_blocks - 1) / p.part_blocks;
    if (part > 0 && part >= nparts) return;                       // beyond this sequence's context
    const int blk0 = part * p.part_blocks;
    const int nblk = max(0, min(p.part_blocks, nblk_seq - blk0));
    const int group = p.group;
    const int64_t qh0 = (int64_t)kvh * group;                     // first query head of this KV head

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], PATH == 1 ? NCW : KPC);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    float* red_o = reinterpret_cast<float*>(smem);
    float* red_m = red_o + K::NSLOT * K::MAXG * D;
    float* red_l = red_m + K::NSLOT * K::MAXG;

    if (warp == 0) {
        // ---------------- producer ----------------
        const uint64_t pol = l2_policy_evict_first();
        const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks + blk0;
        int issued = 0;
        bool ok = true;
        for (int j0 = 0; j0 < nblk && ok; j0 += 32) {
            int id = 0;
            if (j0 + lane < nblk) {
                id = __ldg(bt + j0 + lane);
                if (id < 0 || id >= p.num_blocks) {
                    flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                    id = p.num_blocks;                            // TMA fills an out-of-range tile with zeros
                }
            }
            const int jn = min(32, nblk - j0);
            for (int jj = 0; jj < jn; ++jj) {
                const int pb = __shfl_sync(0xffffffffu, id, jj);
                if (lane == 0 && ok) {
                    const int j = j0 + jj, si = j / K::BPS, b = j - si * K::BPS, st = si % STAGES;
                    if (b == 0) {                                 // first block of a stage: claim it
                        if (!mbar_wait_bounded(&empty[st], ((si / STAGES) & 1) ^ 1, p.err)) {
                            ok = false;
                            s_abort = 1;
                        } else {
                            mbar_arrive_expect_tx(&full[st], min(K::BPS, nblk - j) * 2 * KPC * K::TILE);
                            ++issued;
                        }
                    }
                    if (ok) {
#pragma unroll
                        for (int hd = 0; hd < KPC; ++hd) {
                            uint8_t* dst = smem + st * K::STAGE_BYTES + (hd * K::BPS + b) * K::TILE;
                            uint8_t* vdst = dst + KPC * K::BPS * K::TILE;
                            if constexpr (K::kMma) {
#pragma unroll
                                for (int h = 0; h < K::NBOX; ++h) {
                                    tma_load_4d(dst + h * (BS * 128), &tm_k, &full[st], h * K::BOX, kvh + hd, 0, pb,
                                                pol);
                                    tma_load_4d(vdst + h * (BS * 128), &tm_v, &full[st], h * K::BOX, kvh + hd, 0, pb,
                                                pol);
                                }
                            } else {
                                tma_load_4d(dst, &tm_k, &full[st], 0, kvh + hd, 0, pb, pol);
                                tma_load_4d(vdst, &tm_v, &full[st], 0, kvh + hd, 0, pb, pol);
                            }
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
            }
        }
        if (lane == 0 && !ok) {
            // Drain: wait (bounded) for every copy still in flight before the CTA exits.
            for (int j = max(0, issued - STAGES); j < issued; ++j)
                mbar_wait_bounded(&full[j % STAGES], (j / STAGES) & 1, p.err);
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 1;
        const int hd = cw / K::WPH, sub = cw - hd * K::WPH;               // this warp's KV head, and its turn
        using TQ = std::conditional_t<sizeof(T) == 1, __nv_bfloat16, T>;   // an fp8 cache takes bf16 queries
        const TQ* qbase = static_cast<const TQ*>(p.q) + ((int64_t)seq * p.num_q_heads + qh0 + hd * group) * D;
        const int nstage = (nblk + K::BPS - 1) / K::BPS;
        const int kofs = hd * K::BPS * K::TILE, vofs = (KPC + hd) * K::BPS * K::TILE;
        if constexpr (PATH == 2) {
            using Cons = std::conditional_t<sizeof(T) == 1, MmaConsumerFp8<K::BPS>, MmaConsumer<D>>;
            Cons c;
            c.init(reinterpret_cast<const __nv_bfloat16*>(qbase), group, lane);
            for (int j = sub; j < nstage; j += K::WPH) {
                const int st = j % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (j / STAGES) & 1, p.err);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {   // warp-uniform exit
                    s_abort = 1;
                    break;
                }
                uint8_t* stage = smem + st * K::STAGE_BYTES;
                const int nvalid = min(K::TOK, ctx - (blk0 + j * K::BPS) * BS);
                uint8_t* vst = stage + vofs;
                c.consume(smem_u32(stage + kofs), smem_u32(vst), vst, nvalid, p.scale_log2, lane);
                if (nvalid < K::TOK) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            consumers_barrier();      // every consumer is done with the stage ring it aliases
            c.finish(red_o + cw * K::MAXG * D, red_m + cw * K::MAXG, red_l + cw * K::MAXG, group, lane);
        } else {
            constexpr int HPWc = HPW;
            const int hbase = PATH == 1 ? cw * HPWc : 0;
            SimtConsumer<T, D, HPWc, TQ, K::TOK> c;
            c.init(qbase + (int64_t)hbase * D, p.scale_log2, lane);
            const int jstart = PATH == 1 ? 0 : sub, jstep = PATH == 1 ? 1 : K::WPH;
            for (int j = jstart; j < nstage; j += jstep) {
                const int st = j % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (j / STAGES) & 1, p.err);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {
                    s_abort = 1;
                    break;
                }
                const uint8_t* stage = smem + st * K::STAGE_BYTES;
                c.consume(stage + kofs, stage + vofs, min(K::TOK, ctx - (blk0 + j * K::BPS) * BS), lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            consumers_barrier();
            const int slot = PATH == 1 ? 0 : cw;
            c.finish(red_o + (slot * K::MAXG + hbase) * D, red_m + slot * K::MAXG + hbase,
                     red_l + slot * K::MAXG + hbase, lane);
        }
    }
    __syncthreads();
    if (s_abort) return;

    // ---------------- merge consumer states, write output or partial ----------------
    // KV head hd of this CTA: its states are in warp slots [hd * NSLOT / KPC, (hd + 1) * NSLOT / KPC).
    constexpr int SPH = K::NSLOT / KPC;
    const int C = p.num_parts;
    for (int idx = threadIdx.x; idx < KPC * group * D; idx += NTHREADS) {
        const int hd = idx / (group * D), rem = idx - hd * group * D;
        const int h = rem / D, d = rem - h * D;
        float M = kNegInf;
#pragma unroll
        for (int w = hd * SPH; w < (hd + 1) * SPH; ++w) M = fmaxf(M, red_m[w * K::MAXG + h]);
        float L = 0.f, O = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = hd * SPH; w < (hd + 1) * SPH; ++w) {
                const float mw = red_m[w * K::MAXG + h];
                if (mw == kNegInf) continue;
                const float sc = fast_exp2(mw - M);
                L += red_l[w * K::MAXG + h] * sc;
                O += red_o[(w * K::MAXG + h) * D + d] * sc;
            }
        }
        const float val = L > 0.f ? O / L : 0.f;
        const int64_t qh = (int64_t)seq * p.num_q_heads + qh0 + hd * group + h;
        if (nparts <= 1) {
            store_out(p, qh * D + d, val);
        } else {
            p.ws_o[(qh * C + part) * D + d] = val;
            if (d == 0) {
                p.ws_ml[(qh * C + part) * 2 + 0] = M;
                p.ws_ml[(qh * C + part) * 2 + 1] = L;
            }
        }
    }
}

// Log-sum-exp merge of partition results. grid = (Hq, B), block = D threads.
template <int D>
__global__ void __launch_bounds__(D) merge_partitions_kernel(const Params p) {
    const int qhead = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
    int ctx = p.context_lens[seq];
    ctx = ctx < 0 ? 0 : (ctx > p.ctx_cap ? p.ctx_cap : ctx);
    const int nparts = ((ctx + BS - 1) / BS + p.part_blocks - 1) / p.part_blocks;
    if (nparts <= 1) return;
    const int64_t qh = (int64_t)seq * p.num_q_heads + qhead;
    const float* ml = p.ws_ml + qh * p.num_parts * 2;
    const float* o = p.ws_o + qh * p.num_parts * D;
    float M = kNegInf;
    for (int c = 0; c < nparts; ++c) M = fmaxf(M, ml[2 * c]);
    float L = 0.f, O = 0.f;
    if (M != kNegInf) {
        for (int c = 0; c < nparts; ++c) {
            const float mc = ml[2 * c];
            if (mc == kNegInf) continue;
            const float w = ml[2 * c + 1] * fast_exp2(mc - M);
            L += w;
            O += w * o[(int64_t)c * D + d];
        }
    }
    store_out(p, qh * D + d, L > 0.f ? O / L : 0.f);
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

// Tensor map over a cache [NB, BS, Hkv, D] of 4-, 2- or 1-byte elements: box =
// one block of one head, the whole row (SIMT) or 128-byte box rows with the
// 128-byte swizzle (tensor-core path).
bool make_cache_map(CUtensorMap* map, const void* base, pkv_dtype dt, int nb, int hkv, int d, bool mma) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t eb = dt == PKV_F32 ? 4 : (dt == PKV_BF16 ? 2 : 1);
    const CUtensorMapDataType ty = dt == PKV_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)hkv, (cuuint64_t)BS, (cuuint64_t)nb};
    cuuint64_t strides[3] = {d * eb, (cuuint64_t)hkv * d * eb, (cuuint64_t)BS * hkv * d * eb};
    cuuint32_t box[4] = {(cuuint32_t)(mma ? 128 / eb : d), 1, (cuuint32_t)BS, 1};
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
};

// Schedule for one call.
//   partition_tokens > 0  : fixed partitions of that many tokens (+ merge kernel).
//   partition_tokens == 0 : fixed partitions chosen here: the largest of
//                           2048/1024/512/256 tokens that still gives about two
//                           waves of work items (estimated from the longest
//                           context, assuming lengths spread down to ~half of it).
//                           Measured on B200: fewer, longer partitions stream
//                           fastest (no merge pass, fewer CTA start-ups).
//   partition_tokens == -1: the persistent, evenly split schedule (at most 2048
//                           sequences and < 2^31 tiles).
bool plan(int num_seqs, int num_kv_heads, int block_size, int max_blocks, int max_context_len,
          int partition_tokens, Plan* pl) {
    if (num_seqs <= 0 || num_kv_heads <= 0 || block_size != BS || max_blocks <= 0 || partition_tokens < -1)
        return false;
    const int64_t cap_tbl = (int64_t)max_blocks * block_size;
    if (cap_tbl > INT32_MAX) return false;
    int cap = (int)cap_tbl;
    if (max_context_len > 0) cap = std::min(cap, max_context_len);
    pl->ctx_cap = cap;
    pl->persistent = false;
    pl->grid = 0;
    pl->team_size = 0;
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
        // Fewest partitions of at most kMaxAutoPartition tokens that still give
        // about two waves of work items (estimated with lengths spread down to
        // ~half of the longest); never shorter than 256 tokens.
        constexpr int kMaxAutoPartition = 2560;
        const int64_t target = 2ll * 3 * num_sms();             // ~two waves of 3 CTAs per SM
        pt = 256;
        for (int nparts = 1; nparts <= 65535; ++nparts) {
            const int cand = (int)(((int64_t)(cap + nparts - 1) / nparts + BS - 1) / BS * BS);
            if (cand < 256) break;
            if (cand > kMaxAutoPartition) continue;
            const int64_t est = (int64_t)num_seqs * num_kv_heads * std::max<int64_t>(1, (nparts + 1) / 2);
            if (est >= target) { pt = cand; break; }
        }
    }
    pt = ((pt + BS - 1) / BS) * BS;
    int parts = (cap + pt - 1) / pt;
    if (parts < 1) parts = 1;
    if (parts > 65535) return false;
    pl->part_tokens = pt;
    pl->num_parts = parts;
    return true;
}

size_t ws_bytes_for(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, const Plan& pl) {
    if (pl.persistent) {
        const int group = num_q_heads / num_kv_heads;
        const size_t parts = (((size_t)2 * pl.grid * group * (head_dim + 2) * 4) + 255) & ~size_t(255);
        return parts + (size_t)num_seqs * num_kv_heads * 8;
    }
    if (pl.num_parts <= 1) return 0;
    const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
    const size_t o_bytes = ((rows * head_dim * 4) + 255) & ~size_t(255);
    return o_bytes + rows * 2 * 4;
}

template <typename T, int D, int PATH, int HPW, int STAGES, int KPC = 1>
cudaError_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t stream) {
    using K = Kern<T, D, PATH, HPW, STAGES, KPC>;
    auto kern = paged_decode_kernel<T, D, PATH, HPW, STAGES, KPC>;
    grid.x /= KPC;
    // Opt in to >48 KB dynamic shared memory once per device.
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(done_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
        if (e != cudaSuccess) return e;
        done_mask.fetch_or(bit);
    }
    kern<<<grid, NTHREADS, K::SMEM, stream>>>(mk, mv, p);
    return cudaGetLastError();
}

// Ring depth: about 64 KB of stages per CTA (8 KB per stage for bf16 D=128),
// so three CTAs fit on an SM with ~190 KB of KV in flight.
template <typename T, int D, int KPC = 1>
constexpr int stages_for() {
    constexpr int sb = 2 * (sizeof(T) == 1 ? 2 : 1) * KPC * BS * D * (int)sizeof(T);   // Kern::STAGE_BYTES
    constexpr int n = 65536 / sb;
    return n < 4 ? 4 : (n > 16 ? 16 : n);
}

template <typename T, int D, int KPC = 1>
cudaError_t dispatch_simt(int group, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t st) {
    switch (group) {
        case 1: return launch_decode<T, D, 0, 1, stages_for<T, D, KPC>(), KPC>(mk, mv, p, grid, st);
        case 2: return launch_decode<T, D, 0, 2, stages_for<T, D, KPC>(), KPC>(mk, mv, p, grid, st);
        case 4: return KPC == 1 ? launch_decode<T, D, 1, 1, stages_for<T, D>()>(mk, mv, p, grid, st)
                                : cudaErrorInvalidValue;
        case 8: return KPC == 1 ? launch_decode<T, D, 1, 2, stages_for<T, D>()>(mk, mv, p, grid, st)
                                : cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
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
    if (block_size != BS) return PKV_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_UNSUPPORTED;
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
    const bool use_mma = (bf16 || fp8) && group >= 2;
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, k_cache, kv_dtype, num_blocks, num_kv_heads, head_dim, use_mma) ||
        !make_cache_map(&mv, v_cache, kv_dtype, num_blocks, num_kv_heads, head_dim, use_mma))
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
    p.part_blocks = pl.part_tokens / BS;
    p.num_parts = pl.num_parts;
    p.num_seqs = num_seqs;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (pl.persistent) {
        static std::atomic<unsigned long long> epoch{1};
        p.ws_part = static_cast<float*>(workspace);
        p.counters = reinterpret_cast<unsigned long long*>(
            static_cast<uint8_t*>(workspace) +
            ((((size_t)2 * pl.grid * group * (head_dim + 2) * 4) + 255) & ~size_t(255)));
        p.epoch = epoch.fetch_add(1) & ((1ull << 40) - 1);
        p.team_size = pl.team_size;
        if (launch_persistent(bf16, use_mma, head_dim, group, mk, mv, p, pl.grid, st) != cudaSuccess)
            return PKV_ERR_CUDA;
        return PKV_OK;
    }
    if (need > 0) {
        const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
        p.ws_o = static_cast<float*>(workspace);
        p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           (((rows * head_dim * 4) + 255) & ~size_t(255)));
    }

    dim3 grid(num_kv_heads, pl.num_parts, num_seqs);
    cudaError_t e;
    if (fp8) {
        // Two KV heads per CTA where the SIMT path splits by block (groups 1, 2)
        // or on tensor cores: each token's 256 contiguous bytes of K (and of V)
        // are fetched in one go instead of two 128-byte halves by different CTAs.
        const bool pair = num_kv_heads % 2 == 0 && (use_mma || group <= 2);
        if (use_mma)
            e = pair ? launch_decode<uint8_t, 128, 2, 8, stages_for<uint8_t, 128, 2>(), 2>(mk, mv, p, grid, st)
                     : launch_decode<uint8_t, 128, 2, 8, stages_for<uint8_t, 128>()>(mk, mv, p, grid, st);
        else
            e = pair ? dispatch_simt<uint8_t, 128, 2>(group, mk, mv, p, grid, st)
                     : dispatch_simt<uint8_t, 128>(group, mk, mv, p, grid, st);
    } else if (use_mma) {
        e = head_dim == 128
                ? launch_decode<__nv_bfloat16, 128, 2, 8, stages_for<__nv_bfloat16, 128>()>(mk, mv, p, grid, st)
                : launch_decode<__nv_bfloat16, 64, 2, 8, stages_for<__nv_bfloat16, 64>()>(mk, mv, p, grid, st);
    } else if (bf16) {
        e = head_dim == 128 ? dispatch_simt<__nv_bfloat16, 128>(group, mk, mv, p, grid, st)
                            : dispatch_simt<__nv_bfloat16, 64>(group, mk, mv, p, grid, st);
    } else {
        e = head_dim == 128 ? dispatch_simt<float, 128>(group, mk, mv, p, grid, st)
                            : dispatch_simt<float, 64>(group, mk, mv, p, grid, st);
    }
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    if (pl.num_parts > 1) {
        dim3 g2(num_q_heads, num_seqs);
        if (head_dim == 128) merge_partitions_kernel<128><<<g2, 128, 0, st>>>(p);
        else merge_partitions_kernel<64><<<g2, 64, 0, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
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
