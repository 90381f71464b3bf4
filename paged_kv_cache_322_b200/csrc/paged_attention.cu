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

#include "common.cuh"

namespace pkv {
namespace attn {

constexpr int BS = 16;          // tokens per physical block (the only size built)
constexpr int NCW = 4;          // consumer warps per CTA
constexpr int NTHREADS = 32 * (NCW + 1);
constexpr float kNegInf = -INFINITY;

struct Params {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;        // [B, Hq, C, D] partition outputs (normalised)
    float* ws_ml;       // [B, Hq, C, 2] partition (m, l), m in log2 units
    int* err;
    float scale_log2;   // scale * log2(e)
    int out_f32;
    int num_q_heads, num_kv_heads, group;
    int max_blocks, num_blocks;
    int ctx_cap;        // clamp for context_lens
    int part_blocks;    // blocks per partition
    int num_parts;      // grid.y
};

__device__ __forceinline__ void store_out(const Params& p, int64_t idx, float v) {
    if (p.out_f32) static_cast<float*>(p.out)[idx] = v;
    else static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------------------
// SIMT consumer: HPW query heads per warp, 8 lanes per token, 4 tokens per
// round, fp32 math. T = float or __nv_bfloat16.
// ---------------------------------------------------------------------------
template <typename T, int D, int HPW>
struct SimtConsumer {
    static constexpr int RB = D * (int)sizeof(T);          // row bytes
    static constexpr int NCH = RB / 16;                     // 16-byte chunks per row
    static constexpr int CPL = NCH / 8;                     // chunks per lane
    static constexpr int EPC = 16 / (int)sizeof(T);         // elements per chunk
    static constexpr int EPL = CPL * EPC;                   // elements per lane
    static constexpr int ROUNDS = BS / 4;
    static_assert(NCH % 8 == 0, "row must hold a multiple of 8 chunks");

    float q[HPW][EPL];
    float acc[HPW][EPL];
    float m[HPW], l[HPW];

    __device__ __forceinline__ static void unpack(const uint4& raw, float* f) {
        if constexpr (sizeof(T) == 4) {
            f[0] = __uint_as_float(raw.x); f[1] = __uint_as_float(raw.y);
            f[2] = __uint_as_float(raw.z); f[3] = __uint_as_float(raw.w);
        } else {
            f[0] = bf16lo(raw.x); f[1] = bf16hi(raw.x); f[2] = bf16lo(raw.y); f[3] = bf16hi(raw.y);
            f[4] = bf16lo(raw.z); f[5] = bf16hi(raw.z); f[6] = bf16lo(raw.w); f[7] = bf16hi(raw.w);
        }
    }

    // q_rows points at query head (first head of this warp) of this sequence.
    __device__ __forceinline__ void init(const T* q_rows, float scale_log2, int lane) {
        const int li = lane & 7;
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
            const uint4* row = reinterpret_cast<const uint4*>(q_rows + (int64_t)h * D);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                float f[EPC];
                unpack(__ldg(row + c * 8 + li), f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) q[h][c * EPC + e] = f[e] * scale_log2;
            }
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
            m[h] = kNegInf;
            l[h] = 0.f;
        }
    }

    __device__ __forceinline__ void consume(const uint8_t* ks, const uint8_t* vs, int nvalid, int lane) {
        const int li = lane & 7, tg = lane >> 3;
        float x[ROUNDS][HPW];
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            const uint4* row = reinterpret_cast<const uint4*>(ks + (r * 4 + tg) * RB);
            float part[HPW];
#pragma unroll
            for (int h = 0; h < HPW; ++h) part[h] = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                float f[EPC];
                unpack(row[c * 8 + li], f);
#pragma unroll
                for (int h = 0; h < HPW; ++h)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) part[h] = fmaf(q[h][c * EPC + e], f[e], part[h]);
            }
#pragma unroll
            for (int h = 0; h < HPW; ++h) {
                part[h] += __shfl_xor_sync(0xffffffffu, part[h], 1);
                part[h] += __shfl_xor_sync(0xffffffffu, part[h], 2);
                part[h] += __shfl_xor_sync(0xffffffffu, part[h], 4);
                x[r][h] = (r * 4 + tg < nvalid) ? part[h] : kNegInf;
            }
        }
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
            float bm = x[0][h];
#pragma unroll
            for (int r = 1; r < ROUNDS; ++r) bm = fmaxf(bm, x[r][h]);
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            const float mn = fmaxf(m[h], bm);     // finite: every block has a valid token
            const float alpha = fast_exp2(m[h] - mn);
            m[h] = mn;
            float ps = 0.f;
#pragma unroll
            for (int r = 0; r < ROUNDS; ++r) {
                x[r][h] = fast_exp2(x[r][h] - mn);
                ps += x[r][h];
            }
            l[h] = l[h] * alpha + ps;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[h][e] *= alpha;
        }
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            if (r * 4 + tg < nvalid) {         // never touch rows past the context
                const uint4* row = reinterpret_cast<const uint4*>(vs + (r * 4 + tg) * RB);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    float f[EPC];
                    unpack(row[c * 8 + li], f);
#pragma unroll
                    for (int h = 0; h < HPW; ++h)
#pragma unroll
                        for (int e = 0; e < EPC; ++e)
                            acc[h][c * EPC + e] = fmaf(x[r][h], f[e], acc[h][c * EPC + e]);
                }
            }
        }
    }

    // Sum over the 4 token groups; lanes 0..7 write acc, lane 0 writes m and l.
    __device__ __forceinline__ void finish(float* red_o, float* red_m, float* red_l, int lane) {
        const int li = lane & 7;
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
            float lh = l[h];
            lh += __shfl_xor_sync(0xffffffffu, lh, 8);
            lh += __shfl_xor_sync(0xffffffffu, lh, 16);
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                float a = acc[h][e];
                a += __shfl_xor_sync(0xffffffffu, a, 8);
                a += __shfl_xor_sync(0xffffffffu, a, 16);
                acc[h][e] = a;
            }
            if (lane < 8) {
#pragma unroll
                for (int c = 0; c < CPL; ++c)
#pragma unroll
                    for (int e = 0; e < EPC; ++e)
                        red_o[h * D + (c * 8 + li) * EPC + e] = acc[h][c * EPC + e];
            }
            if (lane == 0) {
                red_m[h] = m[h];
                red_l[h] = lh;
            }
        }
    }
};

// ---------------------------------------------------------------------------
// Tensor-core consumer (bf16, up to 8 query heads per KV head).
// Stage layout: for K then V, D/64 half-tiles of [16 rows x 128 B], each
// written by TMA with the 128-byte swizzle (16-byte chunk c of row r lives at
// chunk c ^ (r & 7)), so ldmatrix reads are bank-conflict free.
// ---------------------------------------------------------------------------
template <int D>
struct MmaConsumer {
    static constexpr int KS = D / 16;          // k-steps of S^T = K Q^T
    static constexpr int MT = D / 16;          // m-tiles of O^T
    static constexpr int HALF = BS * 128;      // bytes of one 64-wide half tile

    uint32_t qb[KS][2];                        // Q^T as B fragments (N = 8 query heads)
    float o[MT][4];                            // O^T fragments: dims x heads
    float m0, m1, l0, l1;                      // heads 2t, 2t+1

    __device__ __forceinline__ void init(const __nv_bfloat16* q_rows, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t* row = reinterpret_cast<const uint32_t*>(q_rows + (int64_t)g * D);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            if (g < group) {
                qb[ks][0] = __ldg(row + (ks * 16 + 2 * t) / 2);
                qb[ks][1] = __ldg(row + (ks * 16 + 2 * t + 8) / 2);
            } else {
                qb[ks][0] = qb[ks][1] = 0u;
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        m0 = m1 = kNegInf;
        l0 = l1 = 0.f;
    }

    __device__ __forceinline__ void consume(uint32_t ks_base, uint32_t vs_base, uint8_t* vs_ptr, int nvalid,
                                            float scale_log2, int lane) {
        const int g = lane >> 2, t = lane & 3;
        // Rows past the context may hold anything (NaN included): zero them in V,
        // so that p = 0 times the row stays 0. K rows are masked by select.
        if (nvalid < BS) {
            for (int i = lane; i < (BS - nvalid) * (D / 8); i += 32) {
                const int r = nvalid + i / (D / 8), cc = i % (D / 8);
                const int half = cc >> 3, c = cc & 7;
                *reinterpret_cast<uint4*>(vs_ptr + half * HALF + r * 128 + ((c ^ (r & 7)) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int r = lane & 15;
            const int c = ((ks & 3) << 1) + (lane >> 4);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, ks_base + (ks >> 2) * HALF + r * 128 + ((c ^ (r & 7)) << 4));
            mma_bf16_16816(s, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
        // s[0]: (token g, head 2t)  s[1]: (g, 2t+1)  s[2]: (g+8, 2t)  s[3]: (g+8, 2t+1)
        float x0 = g < nvalid ? s[0] * scale_log2 : kNegInf;
        float x1 = g < nvalid ? s[1] * scale_log2 : kNegInf;
        float x2 = g + 8 < nvalid ? s[2] * scale_log2 : kNegInf;
        float x3 = g + 8 < nvalid ? s[3] * scale_log2 : kNegInf;
        float b0 = fmaxf(x0, x2), b1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, off));
            b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, off));
        }
        const float n0 = fmaxf(m0, b0), n1 = fmaxf(m1, b1);
        const float al0 = fast_exp2(m0 - n0), al1 = fast_exp2(m1 - n1);
        m0 = n0;
        m1 = n1;
        const float p0 = fast_exp2(x0 - n0), p1 = fast_exp2(x1 - n1);
        const float p2 = fast_exp2(x2 - n0), p3 = fast_exp2(x3 - n1);
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
        }
        // P^T as B fragments (k = token, n = head), high and low bf16 parts.
        const uint32_t h02 = pack_bf16(p0, p2), h13 = pack_bf16(p1, p3);
        const uint32_t e02 = pack_bf16(p0 - bf16lo(h02), p2 - bf16hi(h02));
        const uint32_t e13 = pack_bf16(p1 - bf16lo(h13), p3 - bf16hi(h13));
        const int srcA = (2 * t) * 4 + (g >> 1), srcB = srcA + 4;
        const bool odd = g & 1;
        uint32_t ya, yb, za, zb;
        {
            const uint32_t u0 = __shfl_sync(0xffffffffu, h02, srcA), u1 = __shfl_sync(0xffffffffu, h13, srcA);
            const uint32_t v0 = __shfl_sync(0xffffffffu, h02, srcB), v1 = __shfl_sync(0xffffffffu, h13, srcB);
            ya = odd ? u1 : u0;
            yb = odd ? v1 : v0;
        }
        {
            const uint32_t u0 = __shfl_sync(0xffffffffu, e02, srcA), u1 = __shfl_sync(0xffffffffu, e13, srcA);
            const uint32_t v0 = __shfl_sync(0xffffffffu, e02, srcB), v1 = __shfl_sync(0xffffffffu, e13, srcB);
            za = odd ? u1 : u0;
            zb = odd ? v1 : v0;
        }
        const uint32_t bh0 = __byte_perm(ya, yb, 0x5410), bh1 = __byte_perm(ya, yb, 0x7632);
        const uint32_t bl0 = __byte_perm(za, zb, 0x5410), bl1 = __byte_perm(za, zb, 0x7632);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int mi = lane >> 3;
            const int tok = (lane & 7) + ((mi >> 1) << 3);
            const int c = (((mt * 16) & 63) >> 3) + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(a0, a1, a2, a3,
                              vs_base + ((mt * 16) >> 6) * HALF + tok * 128 + ((c ^ (tok & 7)) << 4));
            mma_bf16_16816(o[mt], a0, a1, a2, a3, bh0, bh1);
            mma_bf16_16816(o[mt], a0, a1, a2, a3, bl0, bl1);
        }
    }

    __device__ __forceinline__ void finish(float* red_o, float* red_m, float* red_l, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
        const int h0 = 2 * t, h1 = 2 * t + 1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            if (h0 < group) {
                red_o[h0 * D + mt * 16 + g] = o[mt][0];
                red_o[h0 * D + mt * 16 + g + 8] = o[mt][2];
            }
            if (h1 < group) {
                red_o[h1 * D + mt * 16 + g] = o[mt][1];
                red_o[h1 * D + mt * 16 + g + 8] = o[mt][3];
            }
        }
        if (g == 0) {
            if (h0 < group) { red_m[h0] = m0; red_l[h0] = l0; }
            if (h1 < group) { red_m[h1] = m1; red_l[h1] = l1; }
        }
    }
};

// ---------------------------------------------------------------------------
// The pipelined kernel.
//   PATH 0: SIMT, block-split (each consumer warp takes whole blocks, HPW = group)
//   PATH 1: SIMT, head-split (every warp reads every block, HPW = group / NCW)
//   PATH 2: tensor cores, block-split (group <= 8)
// ---------------------------------------------------------------------------
template <typename T, int D, int PATH, int HPW, int STAGES>
struct Kern {
    static constexpr bool kMma = PATH == 2;
    static constexpr int TILE = BS * D * (int)sizeof(T);              // one block, one head, K or V
    static constexpr int STAGE_BYTES = 2 * TILE;
    static constexpr int RING = STAGES * STAGE_BYTES;
    static constexpr int NSLOT = PATH == 1 ? 1 : NCW;                  // partial states to merge
    static constexpr int MAXG = PATH == 2 ? 8 : (PATH == 1 ? HPW * NCW : HPW);
    static constexpr int RED = NSLOT * MAXG * (D + 2) * 4;
    static constexpr int BODY = RING > RED ? RING : RED;
    static constexpr int SMEM = 1024 /*align slack*/ + BODY + 2 * STAGES * 8;
    static_assert(RED <= BODY, "reduction scratch must fit");
};

__device__ __forceinline__ void consumers_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

template <typename T, int D, int PATH, int HPW, int STAGES>
__global__ void __launch_bounds__(NTHREADS, 3)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const Params p) {
    using K = Kern<T, D, PATH, HPW, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::BODY);
    uint64_t* empty = full + STAGES;
    __shared__ volatile int s_abort;

    const int kvh = blockIdx.x, part = blockIdx.y, seq = blockIdx.z;
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
            mbar_init(&empty[i], PATH == 1 ? NCW : 1);
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
                    const int j = j0 + jj, st = j % STAGES;
                    if (!mbar_wait_bounded(&empty[st], ((j / STAGES) & 1) ^ 1, p.err)) {
                        ok = false;
                        s_abort = 1;
                    } else {
                        mbar_arrive_expect_tx(&full[st], K::STAGE_BYTES);
                        uint8_t* dst = smem + st * K::STAGE_BYTES;
                        if constexpr (K::kMma) {
#pragma unroll
                            for (int h = 0; h < D / 64; ++h) {
                                tma_load_4d(dst + h * (BS * 128), &tm_k, &full[st], h * 64, kvh, 0, pb, pol);
                                tma_load_4d(dst + K::TILE + h * (BS * 128), &tm_v, &full[st], h * 64, kvh, 0, pb, pol);
                            }
                        } else {
                            tma_load_4d(dst, &tm_k, &full[st], 0, kvh, 0, pb, pol);
                            tma_load_4d(dst + K::TILE, &tm_v, &full[st], 0, kvh, 0, pb, pol);
                        }
                        ++issued;
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
        const T* qbase = static_cast<const T*>(p.q) + ((int64_t)seq * p.num_q_heads + qh0) * D;
        if constexpr (PATH == 2) {
            MmaConsumer<D> c;
            c.init(reinterpret_cast<const __nv_bfloat16*>(qbase), group, lane);
            for (int j = cw; j < nblk; j += NCW) {
                const int st = j % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (j / STAGES) & 1, p.err);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {   // warp-uniform exit
                    s_abort = 1;
                    break;
                }
                uint8_t* stage = smem + st * K::STAGE_BYTES;
                const int nvalid = min(BS, ctx - (blk0 + j) * BS);
                c.consume(smem_u32(stage), smem_u32(stage + K::TILE), stage + K::TILE, nvalid, p.scale_log2, lane);
                if (nvalid < BS) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            consumers_barrier();      // every consumer is done with the stage ring it aliases
            c.finish(red_o + cw * K::MAXG * D, red_m + cw * K::MAXG, red_l + cw * K::MAXG, group, lane);
        } else {
            constexpr int HPWc = HPW;
            const int hbase = PATH == 1 ? cw * HPWc : 0;
            SimtConsumer<T, D, HPWc> c;
            c.init(qbase + (int64_t)hbase * D, p.scale_log2, lane);
            const int jstart = PATH == 1 ? 0 : cw, jstep = PATH == 1 ? 1 : NCW;
            for (int j = jstart; j < nblk; j += jstep) {
                const int st = j % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (j / STAGES) & 1, p.err);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {
                    s_abort = 1;
                    break;
                }
                const uint8_t* stage = smem + st * K::STAGE_BYTES;
                c.consume(stage, stage + K::TILE, min(BS, ctx - (blk0 + j) * BS), lane);
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
    const int nheads = group;
    const int C = p.num_parts;
    for (int idx = threadIdx.x; idx < nheads * D; idx += NTHREADS) {
        const int h = idx / D, d = idx - h * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < K::NSLOT; ++w) M = fmaxf(M, red_m[w * K::MAXG + h]);
        float L = 0.f, O = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = 0; w < K::NSLOT; ++w) {
                const float mw = red_m[w * K::MAXG + h];
                if (mw == kNegInf) continue;
                const float sc = fast_exp2(mw - M);
                L += red_l[w * K::MAXG + h] * sc;
                O += red_o[(w * K::MAXG + h) * D + d] * sc;
            }
        }
        const float val = L > 0.f ? O / L : 0.f;
        const int64_t qh = (int64_t)seq * p.num_q_heads + qh0 + h;
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

// Tensor map over a cache [NB, BS, Hkv, D]: box = one block of one head, the
// whole row (SIMT) or a 64-element half row with the 128-byte swizzle (MMA).
bool make_cache_map(CUtensorMap* map, const void* base, bool bf16, int nb, int hkv, int d, bool mma) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t eb = bf16 ? 2 : 4;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)hkv, (cuuint64_t)BS, (cuuint64_t)nb};
    cuuint64_t strides[3] = {d * eb, (cuuint64_t)hkv * d * eb, (cuuint64_t)BS * hkv * d * eb};
    cuuint32_t box[4] = {(cuuint32_t)(mma ? 64 : d), 1, (cuuint32_t)BS, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
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
};

bool plan(int num_seqs, int num_kv_heads, int block_size, int max_blocks, int max_context_len,
          int partition_tokens, Plan* pl) {
    if (num_seqs <= 0 || num_kv_heads <= 0 || block_size != BS || max_blocks <= 0) return false;
    const int64_t cap_tbl = (int64_t)max_blocks * block_size;
    if (cap_tbl > INT32_MAX) return false;
    int cap = (int)cap_tbl;
    if (max_context_len > 0) cap = std::min(cap, max_context_len);
    int pt = partition_tokens;
    if (pt <= 0) {
        // Default: 512-token partitions once there are enough (sequence, KV head)
        // items to fill the GPU several times over, 256 below that.
        const int64_t items = (int64_t)num_seqs * num_kv_heads;
        pt = items >= 4 * num_sms() ? 512 : 256;
    }
    pt = ((pt + BS - 1) / BS) * BS;
    if (pt <= 0) return false;
    int parts = (cap + pt - 1) / pt;
    if (parts < 1) parts = 1;
    if (parts > 65535) return false;
    pl->ctx_cap = cap;
    pl->part_tokens = pt;
    pl->num_parts = parts;
    return true;
}

size_t ws_bytes_for(int num_seqs, int num_q_heads, int head_dim, const Plan& pl) {
    if (pl.num_parts <= 1) return 0;
    const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
    const size_t o_bytes = ((rows * head_dim * 4) + 255) & ~size_t(255);
    return o_bytes + rows * 2 * 4;
}

template <typename T, int D, int PATH, int HPW, int STAGES>
cudaError_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t stream) {
    using K = Kern<T, D, PATH, HPW, STAGES>;
    auto kern = paged_decode_kernel<T, D, PATH, HPW, STAGES>;
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
template <typename T, int D>
constexpr int stages_for() {
    constexpr int sb = 2 * BS * D * (int)sizeof(T);
    constexpr int n = 65536 / sb;
    return n < 4 ? 4 : (n > 16 ? 16 : n);
}

template <typename T, int D>
cudaError_t dispatch_simt(int group, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t st) {
    switch (group) {
        case 1: return launch_decode<T, D, 0, 1, stages_for<T, D>()>(mk, mv, p, grid, st);
        case 2: return launch_decode<T, D, 0, 2, stages_for<T, D>()>(mk, mv, p, grid, st);
        case 4: return launch_decode<T, D, 1, 1, stages_for<T, D>()>(mk, mv, p, grid, st);
        case 8: return launch_decode<T, D, 1, 2, stages_for<T, D>()>(mk, mv, p, grid, st);
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
    if (num_q_heads <= 0 || head_dim <= 0 ||
        !pkv::attn::plan(num_seqs, num_kv_heads, block_size, max_blocks_per_seq, max_context_len,
                         partition_tokens, &pl))
        return (size_t)-1;
    return pkv::attn::ws_bytes_for(num_seqs, num_q_heads, head_dim, pl);
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

pkv_status pkv_paged_attention_decode(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                      const void* v_cache, pkv_dtype kv_dtype, const int32_t* block_tables,
                                      const int32_t* context_lens, float scale, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                      int num_blocks, int max_context_len, int partition_tokens,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    using namespace pkv;
    using namespace pkv::attn;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
        max_context_len < 0 || !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if ((out_dtype != PKV_F32 && out_dtype != PKV_BF16) || (kv_dtype != PKV_F32 && kv_dtype != PKV_BF16))
        return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
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
    const size_t need = ws_bytes_for(num_seqs, num_q_heads, head_dim, pl);
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return PKV_ERR_INVALID_ARG;

    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;

    const bool bf16 = kv_dtype == PKV_BF16;
    const bool use_mma = bf16 && group >= 2;
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, k_cache, bf16, num_blocks, num_kv_heads, head_dim, use_mma) ||
        !make_cache_map(&mv, v_cache, bf16, num_blocks, num_kv_heads, head_dim, use_mma))
        return PKV_ERR_CUDA;

    Params p{};
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.err = err;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out_f32 = out_dtype == PKV_F32;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.max_blocks = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.ctx_cap = pl.ctx_cap;
    p.part_blocks = pl.part_tokens / BS;
    p.num_parts = pl.num_parts;
    if (need > 0) {
        const size_t rows = (size_t)num_seqs * num_q_heads * pl.num_parts;
        p.ws_o = static_cast<float*>(workspace);
        p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           (((rows * head_dim * 4) + 255) & ~size_t(255)));
    }

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid(num_kv_heads, pl.num_parts, num_seqs);
    cudaError_t e;
    if (use_mma) {
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

}  // extern "C"
