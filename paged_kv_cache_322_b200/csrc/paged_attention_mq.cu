// Multi-query paged attention with a causal mask, for sm_100a: several new
// query tokens per sequence (a chunk of a long prompt, "vLLM PagedAttention 深度
// 解析" §7.2 Chunked Prefill; or the draft tokens a target model verifies, §7.5
// and "LLM 推理引擎内部原理" §5.2) attend over the paged cache, which already holds
// their own K/V. Query i of a sequence with n queries and context c sits at
// position c - n + i and sees cache tokens 0 .. c - n + i.
//
// B200 design (bf16 caches, head_dim 64 / 128, groups 1-8, block sizes 8-64):
//   * A CTA serves one KV head of one sequence and 64 "query rows" (query
//     token x query head of the group: row r = token r / G, head r % G), one
//     partition of the KV range. Grid (Hkv, partitions, sequences x row tiles).
//   * The producer warp streams the partition's K/V with 4-D TMA pieces into a
//     ring of 16-token stages (the decode kernel's scheme); the KV range stops at
//     the CTA's last visible position. L2 evict-normal: the KV of a sequence is
//     re-read by each of its row tiles.
//   * Each of the 4 consumer warps owns 16 rows (two 8-row MMA n-tiles) and
//     folds EVERY stage: S^T = K Q^T with mma.m16n8k16 (16 tokens x 16 rows),
//     the causal / context mask, online softmax per row, O^T += V^T P^T with P
//     split into bf16 high + low parts. Rows are disjoint, so no cross-warp
//     merge: each warp writes its rows (out, or the partition's partial).
//   * Partitions: as in decode, partial (o / l, m, l) per row and partition, and
//     an exact log-sum-exp merge over the partitions a row can see.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "attention_common.cuh"
#include "plan_units.cuh"

namespace pkv {
namespace attn {
namespace {

constexpr int MQ_ROWS_PER_WARP = 16;
// Consumer warps form NCW / wpr row groups of 16 rows; the wpr warps of a group
// share its rows and split the KV stages among them (wpr = 1: every warp has
// its own rows and folds every stage; wpr = 4: one group of 16 rows, the KV
// range split 4 ways, as a decode step with few query rows wants).
__host__ __device__ constexpr int mq_rows_per_tile(int wpr) { return NCW / wpr * MQ_ROWS_PER_WARP; }

struct MqParams {
    void* out;                    // [T, Hq, D]
    const __nv_bfloat16* q;       // [T, Hq, D]
    const int32_t* block_tables;
    const int32_t* context_lens;  // cache tokens per sequence, the queries' own included
    const int32_t* query_start;   // [B + 1]
    float* ws_o;                  // [T * Hq, C, D]
    float* ws_ml;                 // [T * Hq, C, 2]
    int* err;
    float scale_log2;
    int out_f32;
    int num_seqs, num_tokens, num_q_heads, num_kv_heads, group;
    int max_blocks, num_blocks, ctx_cap, max_query_len;
    int block_size, part_blocks, num_parts, row_tiles;
    int wpr;                      // warps per row group: 1, 2 or 4
    int causal;                   // 1: query i sees positions <= c - n + i; 0: every query sees the whole context
    int slot;                     // >= 0: write only normalised partials (o / l, m, l), partition k at index
                                  // slot + k of num_parts (the shared-prefix cascade); -1: output or partitions
    unsigned long long wait_ns;   // limit of every mbarrier wait (2 s unless the test hook shortened it)
    int withhold;                 // test hook: KV tile whose K copies the first CTA never issues (-1: none)
};

// One normalised output value of row qh (sequence-level token row x head),
// written to out (one partition) or to the partition's partial.
template <int D>
__device__ __forceinline__ void mq_store(const MqParams& p, int64_t qh, int part, bool direct, int d, float v) {
    if (direct) {
        if (p.out_f32) static_cast<float*>(p.out)[qh * D + d] = v;
        else static_cast<__nv_bfloat16*>(p.out)[qh * D + d] = __float2bfloat16_rn(v);
    } else {
        p.ws_o[(qh * p.num_parts + part) * D + d] = v;
    }
}

__device__ __forceinline__ void mq_consumers_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Sequence s's query count n and context c, both checked: 0 <= n <= c <= cap (with
// the causal mask off, 0 < c <= cap) and the queries inside [0, T). A bad entry
// flags PKV_ERR_DEVICE_BOUNDS and the sequence is skipped (n = 0).
__device__ __forceinline__ void mq_sequence(const MqParams& p, int s, int& q0, int& n, int& c) {
    q0 = p.query_start[s];
    const int q1 = p.query_start[s + 1];
    c = p.context_lens[s];
    n = q1 - q0;
    if (q0 < 0 || n < 0 || q1 > p.num_tokens || n > p.max_query_len || (p.causal && c < n) || c > p.ctx_cap ||
        (!p.causal && c <= 0)) {
        if (threadIdx.x == 0) flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
        n = 0;
        c = 0;
        q0 = 0;
    }
}

// One warp's 16 query rows (two n-tiles of 8) against 16-token K/V tiles.
template <int D>
struct MqConsumer {
    static constexpr int KS = D / 16;
    static constexpr int MT = D / 16;
    static constexpr int HALF = TILE_ROWS * 128;

    uint32_t qb[KS][2][2];        // Q^T B fragments per k-step and n-tile
    float o[MT][2][4];            // O^T fragments
    float m[2][2], l[2][2];       // [n-tile][column 2t / 2t+1]
    int pos[2][2];                // position of each of the thread's columns (-1: padding row)

    // rows: this warp's first row (sequence-relative); q0, n, c: the sequence.
    __device__ __forceinline__ void init(const MqParams& p, int row0, int kvh, int q0, int n, int c, int lane) {
        const int g = lane >> 2, t = lane & 3;
        const int G = p.group;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r = row0 + nt * 8 + g;                    // the row whose Q this thread loads
            const int i = r / G, h = r - (r / G) * G;
            const bool live = i < n;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                p.q + ((int64_t)(q0 + (live ? i : 0)) * p.num_q_heads + kvh * G + h) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qb[ks][nt][0] = live ? qrow[(ks * 16 + 2 * t) / 2] : 0u;
                qb[ks][nt][1] = live ? qrow[(ks * 16 + 2 * t + 8) / 2] : 0u;
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int rc = row0 + nt * 8 + 2 * t + cc;      // the row of fragment column 2t + cc
                const int ic = rc / G;
                pos[nt][cc] = ic < n ? (p.causal ? c - n + ic : c - 1) : -1;
                m[nt][cc] = kNegInf;
                l[nt][cc] = 0.f;
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
        }
    }

    // tok0: position of the tile's first token; nvalid: tokens of the tile inside the range.
    __device__ __forceinline__ void consume(uint32_t ks_base, uint32_t vs_base, int tok0, int nvalid,
                                            float scale_log2, int lane) {
        const int g = lane >> 2, t = lane & 3;
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int r = lane & 15;
            const int c = ((ks & 3) << 1) + (lane >> 4);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, ks_base + (ks >> 2) * HALF + r * 128 + ((c ^ (r & 7)) << 4));
            mma_bf16_16816(s[0], a0, a1, a2, a3, qb[ks][0][0], qb[ks][0][1]);
            mma_bf16_16816(s[1], a0, a1, a2, a3, qb[ks][1][0], qb[ks][1][1]);
        }
        const int ja = tok0 + g, jb = tok0 + g + 8;             // positions of the thread's two tokens
        const bool va = g < nvalid, vb = g + 8 < nvalid;
        uint32_t bh[2][2], bl[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            // s[nt][0]: (token g, col 2t)  [1]: (g, 2t+1)  [2]: (g+8, 2t)  [3]: (g+8, 2t+1)
            const float x0 = (va && ja <= pos[nt][0]) ? s[nt][0] * scale_log2 : kNegInf;
            const float x1 = (va && ja <= pos[nt][1]) ? s[nt][1] * scale_log2 : kNegInf;
            const float x2 = (vb && jb <= pos[nt][0]) ? s[nt][2] * scale_log2 : kNegInf;
            const float x3 = (vb && jb <= pos[nt][1]) ? s[nt][3] * scale_log2 : kNegInf;
            float b0 = fmaxf(x0, x2), b1 = fmaxf(x1, x3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, off));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, off));
            }
            const float n0 = fmaxf(m[nt][0], b0), n1 = fmaxf(m[nt][1], b1);
            // a column that has seen no visible token yet keeps m = -inf: use 0 as
            // the reference so that no -inf - -inf appears (its o and l stay 0)
            const float r0 = n0 == kNegInf ? 0.f : n0, r1 = n1 == kNegInf ? 0.f : n1;
            const float al0 = fast_exp2(m[nt][0] - r0), al1 = fast_exp2(m[nt][1] - r1);
            m[nt][0] = n0;
            m[nt][1] = n1;
            const float p0 = fast_exp2(x0 - r0), p1 = fast_exp2(x1 - r1);
            const float p2 = fast_exp2(x2 - r0), p3 = fast_exp2(x3 - r1);
            l[nt][0] = l[nt][0] * al0 + (p0 + p2);
            l[nt][1] = l[nt][1] * al1 + (p1 + p3);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                o[mt][nt][0] *= al0; o[mt][nt][1] *= al1; o[mt][nt][2] *= al0; o[mt][nt][3] *= al1;
            }
            // P^T as B fragments (k = token, n = row), high and low bf16 parts
            const uint32_t h02 = pack_bf16(p0, p2), h13 = pack_bf16(p1, p3);
            const uint32_t e02 = pack_bf16(p0 - bf16lo(h02), p2 - bf16hi(h02));
            const uint32_t e13 = pack_bf16(p1 - bf16lo(h13), p3 - bf16hi(h13));
            const int srcA = (2 * t) * 4 + (g >> 1), srcB = srcA + 4;
            const bool odd = g & 1;
            const uint32_t u0 = __shfl_sync(0xffffffffu, h02, srcA), u1 = __shfl_sync(0xffffffffu, h13, srcA);
            const uint32_t w0 = __shfl_sync(0xffffffffu, h02, srcB), w1 = __shfl_sync(0xffffffffu, h13, srcB);
            const uint32_t y0 = __shfl_sync(0xffffffffu, e02, srcA), y1 = __shfl_sync(0xffffffffu, e13, srcA);
            const uint32_t z0 = __shfl_sync(0xffffffffu, e02, srcB), z1 = __shfl_sync(0xffffffffu, e13, srcB);
            const uint32_t ya = odd ? u1 : u0, yb = odd ? w1 : w0;
            const uint32_t za = odd ? y1 : y0, zb = odd ? z1 : z0;
            bh[nt][0] = __byte_perm(ya, yb, 0x5410);
            bh[nt][1] = __byte_perm(ya, yb, 0x7632);
            bl[nt][0] = __byte_perm(za, zb, 0x5410);
            bl[nt][1] = __byte_perm(za, zb, 0x7632);
        }
        // V rows past the range may hold anything (NaN included) and every warp
        // reads this stage, so nothing is zeroed in shared memory: the V^T
        // fragment's token columns 2t, 2t+1 (a0, a1) and 2t+8, 2t+9 (a2, a3) are
        // masked in registers instead (p = 0 there, but 0 * NaN would not be 0).
        const uint32_t m01 = (2 * t < nvalid ? 0x0000ffffu : 0u) | (2 * t + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t m23 = (2 * t + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * t + 9 < nvalid ? 0xffff0000u : 0u);
        const bool partial = nvalid < TILE_ROWS;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int mi = lane >> 3;
            const int tok = (lane & 7) + ((mi >> 1) << 3);
            const int c = (((mt * 16) & 63) >> 3) + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(a0, a1, a2, a3, vs_base + ((mt * 16) >> 6) * HALF + tok * 128 + ((c ^ (tok & 7)) << 4));
            if (partial) {
                a0 &= m01; a1 &= m01; a2 &= m23; a3 &= m23;
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
                mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
            }
        }
    }

    // Writes the warp's rows: the output (one partition) or the partition's partial.
    __device__ __forceinline__ void finish(const MqParams& p, int row0, int kvh, int q0, int n, int part,
                                           bool direct, int lane) {
        const int g = lane >> 2, t = lane & 3;
        const int G = p.group;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float lsum = l[nt][cc];
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
                const int r = row0 + nt * 8 + 2 * t + cc;
                const int i = r / G, h = r - (r / G) * G;
                if (i >= n) continue;
                const int64_t qh = (int64_t)(q0 + i) * p.num_q_heads + kvh * G + h;
                const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    mq_store<D>(p, qh, part, direct, mt * 16 + g, o[mt][nt][cc] * inv);
                    mq_store<D>(p, qh, part, direct, mt * 16 + g + 8, o[mt][nt][2 + cc] * inv);
                }
                if (!direct && g == 0) {
                    p.ws_ml[(qh * p.num_parts + part) * 2 + 0] = m[nt][cc];
                    p.ws_ml[(qh * p.num_parts + part) * 2 + 1] = lsum;
                }
            }
        }
    }

    // The warp's unnormalised state for a cross-warp merge: so [16 rows][D],
    // sm / sl [16 rows] (m and the full l of each row).
    __device__ __forceinline__ void spill(float* so, float* sm, float* sl, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float lsum = l[nt][cc];
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
                const int r = nt * 8 + 2 * t + cc;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    so[r * D + mt * 16 + g] = o[mt][nt][cc];
                    so[r * D + mt * 16 + g + 8] = o[mt][nt][2 + cc];
                }
                if (g == 0) {
                    sm[r] = m[nt][cc];
                    sl[r] = lsum;
                }
            }
        }
    }
};

template <int D, int BSZ, int STAGES>
struct MqKern {
    static constexpr int TOK = TILE_ROWS;                       // tokens per stage
    static constexpr int R = piece_rows(BSZ, 2);
    static constexpr int BPS = TOK / R;
    static constexpr int PPB = BSZ / R;
    static constexpr int NBOX = D * 2 / 128;
    static constexpr int PIECE = R * D * 2;
    static constexpr int REGION = TOK * D * 2;                  // K (or V) of one stage
    static constexpr int STAGE_BYTES = 2 * REGION;
    static constexpr int MERGE = NCW * MQ_ROWS_PER_WARP * (D + 2) * 4;   // cross-warp merge scratch
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2 * STAGES * 8;
    static_assert(MERGE <= STAGES * STAGE_BYTES, "the merge scratch reuses the ring");
    static_assert(STAGES % 4 == 0, "ring depth must be a multiple of every warps-per-group choice");
    static_assert(BPS * R == TOK && PPB * R == BSZ, "block size must be a power of two >= 8");
};

template <int D, int BSZ, int STAGES>
__global__ void __launch_bounds__(NTHREADS, 2)
paged_mq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const MqParams p) {
    using K = MqKern<D, BSZ, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * K::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    __shared__ volatile int s_abort;

    const int kvh = blockIdx.x, part = blockIdx.y;
    const int seq = blockIdx.z / p.row_tiles, tile = blockIdx.z - seq * p.row_tiles;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int q0, n, c;
    mq_sequence(p, seq, q0, n, c);
    const int wpr = p.wpr, rows_per_tile = mq_rows_per_tile(wpr);
    const int row_begin = tile * rows_per_tile;
    if (row_begin >= n * p.group) return;                          // no live rows in this tile
    // last visible position of the tile's rows, and this partition's KV range
    const int last_tok = min(n - 1, (row_begin + rows_per_tile - 1) / p.group);
    const int kv_end = p.causal ? c - n + last_tok + 1 : c;        // tokens [0, kv_end) are visible to some row
    const int pt = p.part_blocks * BSZ;
    const int kv0 = part * pt;
    if (kv0 >= kv_end) return;                                     // no row of the tile sees this partition
    const int ntok = min(pt, kv_end - kv0);
    const int npiece = (ntok + K::R - 1) / K::R;
    const int nblk = (ntok + BSZ - 1) / BSZ;
    const int blk0 = part * p.part_blocks;
    const bool direct = p.slot < 0 && (c + pt - 1) / pt <= 1;      // the whole context is one partition
    const int opart = p.slot >= 0 ? p.slot + part : part;          // the partial's index in the workspace

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NCW / wpr);                       // one warp of each row group
        }
        s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- producer: the decode kernel's piece walk ----------------
        const uint64_t pol = l2_policy_evict_normal();
        const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks + blk0;
        int issued = 0;
        bool ok = true;
        for (int q0p = 0; q0p < npiece && ok; q0p += 32 * K::PPB) {
            const int j0 = q0p / K::PPB;
            int id = 0;
            if (j0 + lane < nblk) {
                id = __ldg(bt + j0 + lane);
                if (id < 0 || id >= p.num_blocks) {
                    flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                    id = p.num_blocks;                              // TMA fills an out-of-range tile with zeros
                }
            }
            const int qn = min(32 * K::PPB, npiece - q0p);
            for (int qq = 0; qq < qn; ++qq) {
                const int pb = __shfl_sync(0xffffffffu, id, qq / K::PPB);
                if (lane == 0 && ok) {
                    const int q = q0p + qq, sub = qq % K::PPB;
                    const int si = q / K::BPS, b = q - si * K::BPS, st = si % STAGES;
                    if (b == 0) {
                        if (!mbar_wait_bounded(&empty[st], ((si / STAGES) & 1) ^ 1, p.err, p.wait_ns)) {
                            ok = false;
                            s_abort = 1;
                        } else {
                            mbar_arrive_expect_tx(&full[st], min(K::BPS, npiece - q) * 2 * K::PIECE);
                            ++issued;
                        }
                    }
                    if (ok) {
                        uint8_t* dst = smem + st * K::STAGE_BYTES;
                        uint8_t* vdst = dst + K::REGION;
#pragma unroll
                        for (int h = 0; h < K::NBOX; ++h) {
                            const int off = h * (K::TOK * 128) + b * (K::R * 128);
                            tma_load_4d(dst + off, &tm_k, &full[st], h * 64, kvh, sub * K::R, pb, pol);
                            tma_load_4d(vdst + off, &tm_v, &full[st], h * 64, kvh, sub * K::R, pb, pol);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
            }
        }
        if (lane == 0 && !ok) {
            for (int j = max(0, issued - STAGES); j < issued; ++j)
                mbar_wait_bounded(&full[j % STAGES], (j / STAGES) & 1, p.err, p.wait_ns);
        }
    } else {
        // ---------------- consumers: row group rg, turn sub of its wpr warps ----------------
        const int cw = warp - 1;
        const int rg = cw / wpr, sub = cw - rg * wpr;
        const int row0 = row_begin + rg * MQ_ROWS_PER_WARP;
        MqConsumer<D> cons;
        cons.init(p, row0, kvh, q0, n, c, lane);
        const int nstage = (npiece + K::BPS - 1) / K::BPS;
        // With STAGES a multiple of wpr, every round of a stage goes to the same
        // warp of each group, so no warp can run a ring phase ahead of the producer.
        for (int j = sub; j < nstage; j += wpr) {
            const int st = j % STAGES;
            const bool got = mbar_wait_bounded(&full[st], (j / STAGES) & 1, p.err, p.wait_ns);
            if (__any_sync(0xffffffffu, !got || s_abort != 0)) {
                s_abort = 1;
                break;
            }
            uint8_t* stage = smem + st * K::STAGE_BYTES;
            const int nvalid = min(K::TOK, ntok - j * K::TOK);
            cons.consume(smem_u32(stage), smem_u32(stage + K::REGION), kv0 + j * K::TOK, nvalid, p.scale_log2, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (wpr == 1) {
            if (!s_abort) cons.finish(p, row0, kvh, q0, n, opart, direct, lane);
        } else {
            // merge the wpr partial states of each row group through shared memory
            // (the ring is free once every consumer is past its last stage)
            mq_consumers_barrier();
            if (!s_abort) {
                float* so = reinterpret_cast<float*>(smem);
                float* sm = so + NCW * MQ_ROWS_PER_WARP * D;
                float* sl = sm + NCW * MQ_ROWS_PER_WARP;
                cons.spill(so + cw * MQ_ROWS_PER_WARP * D, sm + cw * MQ_ROWS_PER_WARP, sl + cw * MQ_ROWS_PER_WARP,
                           lane);
                mq_consumers_barrier();
                const int G = p.group;
                for (int idx = threadIdx.x - 32; idx < NCW / wpr * MQ_ROWS_PER_WARP * D; idx += NCW * 32) {
                    const int grp = idx / (MQ_ROWS_PER_WARP * D), rem = idx - grp * MQ_ROWS_PER_WARP * D;
                    const int rr = rem / D, d = rem - rr * D;
                    const int r = row_begin + grp * MQ_ROWS_PER_WARP + rr;
                    const int i = r / G, h = r - i * G;
                    if (i >= n) continue;
                    float M = kNegInf;
                    for (int w = grp * wpr; w < (grp + 1) * wpr; ++w) M = fmaxf(M, sm[w * MQ_ROWS_PER_WARP + rr]);
                    float L = 0.f, O = 0.f;
                    if (M != kNegInf) {
                        for (int w = grp * wpr; w < (grp + 1) * wpr; ++w) {
                            const float mw = sm[w * MQ_ROWS_PER_WARP + rr];
                            if (mw == kNegInf) continue;
                            const float sc = fast_exp2(mw - M);
                            L += sl[w * MQ_ROWS_PER_WARP + rr] * sc;
                            O += so[(w * MQ_ROWS_PER_WARP + rr) * D + d] * sc;
                        }
                    }
                    const int64_t qh = (int64_t)(q0 + i) * p.num_q_heads + kvh * G + h;
                    mq_store<D>(p, qh, opart, direct, d, L > 0.f ? O / L : 0.f);
                    if (!direct && d == 0) {
                        p.ws_ml[(qh * p.num_parts + opart) * 2 + 0] = M;
                        p.ws_ml[(qh * p.num_parts + opart) * 2 + 1] = L;
                    }
                }
            }
        }
    }
}

// Log-sum-exp merge over the partitions each row sees. grid = (Hq, T), block = D.
template <int D>
__global__ void __launch_bounds__(D) merge_mq_kernel(const MqParams p) {
    const int head = blockIdx.x, tok = blockIdx.y, d = threadIdx.x;
    // the sequence of token `tok`: last s with query_start[s] <= tok
    int lo = 0, hi = p.num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.query_start[mid] <= tok) lo = mid;
        else hi = mid - 1;
    }
    int q0, n, c;
    mq_sequence(p, lo, q0, n, c);
    const int i = tok - q0;
    if (i < 0 || i >= n) return;
    const int pt = p.part_blocks * p.block_size;
    if ((c + pt - 1) / pt <= 1) return;                            // written directly
    const int pos = c - n + i;
    const int nparts = pos / pt + 1;                               // partitions holding tokens 0..pos
    const int64_t qh = (int64_t)tok * p.num_q_heads + head;
    const float* ml = p.ws_ml + qh * p.num_parts * 2;
    const float* o = p.ws_o + qh * p.num_parts * D;
    float M = kNegInf;
    for (int k = 0; k < nparts; ++k) M = fmaxf(M, ml[2 * k]);
    float L = 0.f, O = 0.f;
    if (M != kNegInf) {
        for (int k = 0; k < nparts; ++k) {
            const float mk = ml[2 * k];
            if (mk == kNegInf) continue;
            const float w = ml[2 * k + 1] * fast_exp2(mk - M);
            L += w;
            O += w * o[(int64_t)k * D + d];
        }
    }
    const float v = L > 0.f ? O / L : 0.f;
    if (p.out_f32) static_cast<float*>(p.out)[qh * D + d] = v;
    else static_cast<__nv_bfloat16*>(p.out)[qh * D + d] = __float2bfloat16_rn(v);
}

}  // namespace
}  // namespace attn
}  // namespace pkv

#include "paged_attention_mq_tc.cuh"

namespace pkv {
namespace attn {
namespace {

template <int BSZ>
// pdl: launched as a programmatic dependent of the kernel before it on the
// stream (its CTAs wait for that grid in-kernel).
cudaError_t launch_mq_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const MqParams& p,
                         dim3 grid, cudaStream_t st, bool pdl) {
    auto kern = tc::paged_mq_tc_kernel<BSZ>;
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(done_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM);
        if (e != cudaSuccess) return e;
        done_mask.fetch_or(bit);
    }
    if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(tc::THREADS);
        cfg.dynamicSmemBytes = tc::SMEM;
        cfg.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p);
    }
    kern<<<grid, tc::THREADS, tc::SMEM, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

cudaError_t launch_mq_tc_bs(int bs, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const MqParams& p, dim3 grid, cudaStream_t st, bool pdl = false) {
    switch (bs) {
        case 8: return launch_mq_tc<8>(mq, mk, mv, p, grid, st, pdl);
        case 16: return launch_mq_tc<16>(mq, mk, mv, p, grid, st, pdl);
        case 32: return launch_mq_tc<32>(mq, mk, mv, p, grid, st, pdl);
        default: return launch_mq_tc<64>(mq, mk, mv, p, grid, st, pdl);
    }
}

// Tensor map over q [T, Hq, D] (bf16): box (64 dims, G heads, 128 / G tokens),
// 128-byte swizzle, so one 128-row query tile lands as the K-major operand of
// the tcgen05 kernel (row = token x G + head).
bool make_q_map(CUtensorMap* map, const void* q, int T, int hq, int d, int group) {
    cudaDriverEntryPointQueryResult qr;
    void* f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || !f)
        return false;
    auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hq, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hq * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(tc::ROWS / group)};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BSZ>
cudaError_t launch_mq(const CUtensorMap& mk, const CUtensorMap& mv, const MqParams& p, dim3 grid, cudaStream_t st) {
    constexpr int STAGES = 8;
    using K = MqKern<D, BSZ, STAGES>;
    auto kern = paged_mq_kernel<D, BSZ, STAGES>;
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(done_mask.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
        if (e != cudaSuccess) return e;
        done_mask.fetch_or(bit);
    }
    kern<<<grid, NTHREADS, K::SMEM, st>>>(mk, mv, p);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_mq_bs(int bs, const CUtensorMap& mk, const CUtensorMap& mv, const MqParams& p, dim3 grid,
                         cudaStream_t st) {
    switch (bs) {
        case 8: return launch_mq<D, 8>(mk, mv, p, grid, st);
        case 16: return launch_mq<D, 16>(mk, mv, p, grid, st);
        case 32: return launch_mq<D, 32>(mk, mv, p, grid, st);
        default: return launch_mq<D, 64>(mk, mv, p, grid, st);
    }
}

struct MqPlan {
    int ctx_cap, part_tokens, num_parts, row_tiles, wpr;
    bool tc;            // the tcgen05 kernel (128-row tiles)
};

// KV partitions: fixed (partition_tokens > 0, rounded up to whole blocks), or
// chosen (0): the fewest partitions of at most 2560 tokens that give about two
// waves of CTAs, counting each sequence's row tiles.
bool plan_mq(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks,
             int max_query_len, int max_context_len, int partition_tokens, MqPlan* pl) {
    if (num_seqs <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || !block_size_built(block_size) ||
        max_blocks <= 0 || max_query_len <= 0 || partition_tokens < 0)
        return false;
    const int64_t cap_tbl = (int64_t)max_blocks * block_size;
    if (cap_tbl > INT32_MAX) return false;
    int cap = (int)cap_tbl;
    if (max_context_len > 0) cap = std::min(cap, max_context_len);
    if (max_query_len > cap) return false;
    const int group = num_q_heads / num_kv_heads;
    pl->ctx_cap = cap;
    // few rows (speculative verify, decode): fewer row groups, the KV range split among their warps
    const int64_t rows = (int64_t)max_query_len * group;
    pl->wpr = rows <= MQ_ROWS_PER_WARP ? 4 : (rows <= 2 * MQ_ROWS_PER_WARP ? 2 : 1);
    // From 32 query rows per KV head on (prefill chunks, and speculative verify
    // on grouped-query heads) the tcgen05 kernel wins even with most of its 128
    // rows idle (measured, 70B-shaped verify of 5 tokens = 40 rows: 1.7x the
    // mma.sync kernel); below that, the mma.sync kernel splits the KV range over
    // its warps (head_dim 128 only on tcgen05).
    pl->tc = head_dim == 128 && rows >= 32;
    const int tile_rows = pl->tc ? tc::ROWS : mq_rows_per_tile(pl->wpr);
    pl->row_tiles = (int)((rows + tile_rows - 1) / tile_rows);
    int pt = partition_tokens;
    if (pt == 0) {
        // the tcgen05 kernel gets its parallelism from row tiles; splitting the KV
        // range only adds CTA start-ups and the merge (measured: one partition per
        // sequence is 27-42 % faster on 512-token chunks than 2560-token ones)
        const int kMaxAutoPartition = pl->tc ? (1 << 30) : 2560;
        int sms = 148, dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t target = 2ll * (pl->tc ? 1 : 2) * sms;       // ~two waves (1 or 2 CTAs per SM)
        pt = std::max(256, ((cap + block_size - 1) / block_size) * block_size);
        for (int nparts = 1; nparts <= 65535; ++nparts) {
            const int cand = (int)(((int64_t)(cap + nparts - 1) / nparts + block_size - 1) / block_size * block_size);
            if (cand < 256) break;
            pt = cand;
            if (cand > kMaxAutoPartition) continue;
            const int64_t est = (int64_t)num_seqs * num_kv_heads * pl->row_tiles * std::max<int64_t>(1, (nparts + 1) / 2);
            if (est >= target) break;
        }
    }
    pt = ((pt + block_size - 1) / block_size) * block_size;
    const int parts = std::max(1, (cap + pt - 1) / pt);
    if (parts > 65535 || (int64_t)num_seqs * pl->row_tiles > 65535) return false;
    pl->part_tokens = pt;
    pl->num_parts = parts;
    return true;
}

size_t mq_ws_bytes(int num_tokens, int num_q_heads, int head_dim, const MqPlan& pl) {
    if (pl.num_parts <= 1) return 0;
    const size_t rows = (size_t)num_tokens * num_q_heads * pl.num_parts;
    return (((rows * head_dim * 4) + 255) & ~size_t(255)) + rows * 2 * 4;
}

}  // namespace
}  // namespace attn
}  // namespace pkv

extern "C" {

size_t pkv_paged_attention_multi_query_workspace_bytes(int num_seqs, int num_tokens, int num_q_heads,
                                                       int num_kv_heads, int head_dim, int block_size,
                                                       int max_blocks_per_seq, int max_query_len, int max_context_len,
                                                       int partition_tokens) {
    pkv::attn::MqPlan pl;
    if (num_tokens < 0 || head_dim <= 0 ||
        !pkv::attn::plan_mq(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                            max_query_len, max_context_len, partition_tokens, &pl))
        return (size_t)-1;
    return pkv::attn::mq_ws_bytes(num_tokens, num_q_heads, head_dim, pl);
}

pkv_status pkv_paged_attention_multi_query(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                           const void* v_cache, pkv_dtype kv_dtype, const int32_t* block_tables,
                                           const int32_t* context_lens, const int32_t* query_start, float scale,
                                           int num_seqs, int num_tokens, int num_q_heads, int num_kv_heads,
                                           int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                                           int max_query_len, int max_context_len, int partition_tokens,
                                           void* workspace, size_t workspace_bytes, void* stream) {
    using namespace pkv;
    using namespace pkv::attn;
    if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_query_len < 0 || max_context_len < 0 || partition_tokens < 0 ||
        !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if (out_dtype != PKV_F32 && out_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    if (kv_dtype != PKV_BF16 && kv_dtype != PKV_F32 && kv_dtype != PKV_FP8_E4M3) return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    if (kv_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (!block_size_built(block_size)) return PKV_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
        return PKV_ERR_INVALID_ARG;
    auto al = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; };
    if (!al(out) || !al(q) || !al(k_cache) || !al(v_cache)) return PKV_ERR_INVALID_ARG;
    MqPlan pl;
    if (!plan_mq(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, max_query_len,
                 max_context_len, partition_tokens, &pl))
        return PKV_ERR_INVALID_ARG;
    const size_t need = mq_ws_bytes(num_tokens, num_q_heads, head_dim, pl);
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    CUtensorMap mk, mv, mqm;
    const int box_rows = pl.tc ? std::min(block_size, tc::TOK) : 0;   // 0: the decode pieces
    if (!make_cache_map(&mk, k_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, true, box_rows) ||
        !make_cache_map(&mv, v_cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_dim, true, box_rows))
        return PKV_ERR_CUDA;
    if (pl.tc && !make_q_map(&mqm, q, num_tokens, num_q_heads, head_dim, group)) return PKV_ERR_CUDA;
    MqParams p{};
    p.out = out;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.err = err;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out_f32 = out_dtype == PKV_F32;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.max_blocks = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.ctx_cap = pl.ctx_cap;
    p.max_query_len = max_query_len;
    p.block_size = block_size;
    p.part_blocks = pl.part_tokens / block_size;
    p.num_parts = pl.num_parts;
    p.row_tiles = pl.row_tiles;
    p.wpr = pl.wpr;
    p.causal = 1;
    p.slot = -1;
    p.withhold = -1;
    p.wait_ns = kDefaultWaitNs;
    if (pl.tc) take_wait_hook(1, &p.withhold, &p.wait_ns);
    if (need > 0) {
        const size_t rows = (size_t)num_tokens * num_q_heads * pl.num_parts;
        p.ws_o = static_cast<float*>(workspace);
        p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + (((rows * head_dim * 4) + 255) & ~size_t(255)));
    }
    if (pl.num_parts > 1 && num_tokens > 65535) return PKV_ERR_UNSUPPORTED;   // merge grid
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid(num_kv_heads, pl.num_parts, num_seqs * pl.row_tiles);
    cudaError_t e = pl.tc ? launch_mq_tc_bs(block_size, mqm, mk, mv, p, grid, st)
                    : head_dim == 128 ? launch_mq_bs<128>(block_size, mk, mv, p, grid, st)
                                      : launch_mq_bs<64>(block_size, mk, mv, p, grid, st);
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    if (pl.num_parts > 1) {
        dim3 g2(num_q_heads, num_tokens);
        if (head_dim == 128) merge_mq_kernel<128><<<g2, 128, 0, st>>>(p);
        else merge_mq_kernel<64><<<g2, 64, 0, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Shared-prefix decode (a cascade): a batch whose sequences all map the same
// first `prefix` cache tokens (parallel sampling after a copy-on-write fork,
// "为什么PagedAttention能让大模型推理吞吐量提升数倍", Memory Sharing) reads those
// blocks once. The batch's B decode queries attend to the prefix as B query
// tokens of one sequence with the causal mask off (the tcgen05 kernel: every
// KV head's prefix tiles are loaded once for all B x G rows; the prefix is cut
// into partitions so the call fills the GPU, each writing a normalised partial
// (o / l, m, l)); then each sequence's query attends to its own tail (the decode
// kernel, tokens prefix .. ctx - 1 through the table entries past the prefix's
// blocks, longest tail first), and merges the prefix's partials into its result
// by the exact log-sum-exp rule before writing the output. Not a step of the
// pages' method, which reads a shared block once per sequence that maps it.
// ---------------------------------------------------------------------------
namespace pkv {
namespace attn {
namespace {

struct CascadeWs {
    float* pre_o;    // [B, Hq, prefix partitions, D]
    float* pre_ml;   // [B, Hq, prefix partitions, 2]
    uint2* units;    // the tails' list: B entries and their count
    int32_t* ints;   // the prefix call's length [1] and query starts [2]
};

// Prefix partitions: at most one wave of the prefix call's CTAs (KV heads x row
// tiles x partitions; one CTA per SM), whole 128-token KV tiles, at most one per
// tile of prefix. Measured on the shared-prefix workload's shape (32 KV heads, a
// 1008-token prefix): 4 partitions (128 CTAs) 69 us a call, 8 (256 CTAs, two
// rounds) 76 us, 1 (32 CTAs) 78 us.
int cascade_prefix_parts(int num_seqs, int group, int num_kv_heads, int prefix) {
    const int row_tiles = (int)(((int64_t)num_seqs * group + tc::ROWS - 1) / tc::ROWS);
    const int want = std::max(1, num_sms() / std::max(1, num_kv_heads * row_tiles));
    return std::max(1, std::min(want, (prefix + tc::TOK - 1) / tc::TOK));
}

int cascade_prefix_part_tokens(int prefix, int parts) {
    const int pt = (prefix + parts - 1) / parts;
    return (pt + tc::TOK - 1) / tc::TOK * tc::TOK;             // whole KV tiles (a multiple of every block size)
}

// The workspace's regions in order, each 256-byte aligned.
size_t cascade_region(int i, int num_seqs, int num_q_heads, int head_dim, int pre_parts) {
    const size_t rows_p = (size_t)num_seqs * num_q_heads * pre_parts;
    const size_t sz[4] = {rows_p * head_dim * 4, rows_p * 2 * 4, (size_t)num_seqs * sizeof(uint2) + sizeof(int), 3 * 4};
    size_t off = 0;
    for (int k = 0; k < i; ++k) off += (sz[k] + 255) & ~size_t(255);
    return off;
}

size_t cascade_ws_bytes(int num_seqs, int num_q_heads, int head_dim, int pre_parts) {
    return cascade_region(4, num_seqs, num_q_heads, head_dim, pre_parts);
}

CascadeWs cascade_ws(void* workspace, int num_seqs, int num_q_heads, int head_dim, int pre_parts) {
    uint8_t* b = static_cast<uint8_t*>(workspace);
    auto at = [&](int i) { return b + cascade_region(i, num_seqs, num_q_heads, head_dim, pre_parts); };
    CascadeWs w;
    w.pre_o = reinterpret_cast<float*>(at(0));
    w.pre_ml = reinterpret_cast<float*>(at(1));
    w.units = reinterpret_cast<uint2*>(at(2));
    w.ints = reinterpret_cast<int32_t*>(at(3));
    return w;
}

// The plan of the call (one CTA of kPlanThreads): sequence s's tail is ctx_s -
// prefix tokens (at least 1: its own new token; a shorter context is flagged
// and read as prefix + 1, one past the cap as the cap), listed longest first
// (list_units; in sequence order when a tail of tail_cap tokens spans more
// blocks than the list's size bins), and the prefix call's descriptors: one
// sequence of `prefix` tokens with B queries.
__global__ void __launch_bounds__(kPlanThreads) cascade_plan_kernel(const int32_t* context_lens, CascadeWs ws,
                                                                     int num_seqs, int prefix, int cap, int block_size,
                                                                     int* err) {
    // the prefix call may start its CTAs now; they wait for this grid in-kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tail_cap = cap - prefix;
    auto tail = [&](int s, bool first) {
        int c = context_lens[s];
        if (c <= prefix || c > cap) {
            if (first) flag_error(err, PKV_ERR_DEVICE_BOUNDS);
            c = c <= prefix ? prefix + 1 : cap;
        }
        return c - prefix;
    };
    const int pb = (tail_cap + block_size - 1) / block_size;  // the tails' one partition, in blocks
    if (pb <= kPlanMaxBins) {
        list_units(tail, num_seqs, pb, block_size, ws.units, reinterpret_cast<int*>(ws.units + num_seqs));
    } else {
        for (int s = threadIdx.x; s < num_seqs; s += kPlanThreads)
            ws.units[s] = make_uint2((unsigned)s << 16, (unsigned)tail(s, true));
        if (threadIdx.x == 0) *reinterpret_cast<int*>(ws.units + num_seqs) = num_seqs;
    }
    if (threadIdx.x == 0) {
        ws.ints[0] = prefix;
        ws.ints[1] = 0;
        ws.ints[2] = num_seqs;
    }
}

}  // namespace
}  // namespace attn
}  // namespace pkv

extern "C" {

size_t pkv_paged_attention_shared_prefix_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                                        int head_dim, int prefix_tokens) {
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        head_dim <= 0 || prefix_tokens <= 0)
        return (size_t)-1;
    const int parts = pkv::attn::cascade_prefix_parts(num_seqs, num_q_heads / num_kv_heads, num_kv_heads,
                                                      prefix_tokens);
    return pkv::attn::cascade_ws_bytes(num_seqs, num_q_heads, head_dim, parts);
}

pkv_status pkv_paged_attention_decode_shared_prefix(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                                    const void* v_cache, const int32_t* block_tables,
                                                    const int32_t* context_lens, int prefix_tokens, float scale,
                                                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                    int block_size, int max_blocks_per_seq, int num_blocks,
                                                    int max_context_len, void* workspace, size_t workspace_bytes,
                                                    void* stream) {
    using namespace pkv;
    using namespace pkv::attn;
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || !std::isfinite(scale) || max_context_len <= 0)
        return PKV_ERR_INVALID_ARG;
    if (out_dtype != PKV_F32 && out_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    if (head_dim != 128 || !block_size_built(block_size)) return PKV_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return PKV_ERR_UNSUPPORTED;
    // the prefix call runs on the tcgen05 kernel: at least 32 query rows per KV head
    if ((int64_t)num_seqs * group < 32 || num_seqs > 65535) return PKV_ERR_UNSUPPORTED;
    if (prefix_tokens <= 0 || prefix_tokens % block_size != 0 || prefix_tokens >= max_context_len ||
        (int64_t)max_blocks_per_seq * block_size < max_context_len)
        return PKV_ERR_INVALID_ARG;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    auto al = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; };
    if (!al(out) || !al(q) || !al(k_cache) || !al(v_cache)) return PKV_ERR_INVALID_ARG;
    const int pre_parts = cascade_prefix_parts(num_seqs, group, num_kv_heads, prefix_tokens);
    const int pre_pt = cascade_prefix_part_tokens(prefix_tokens, pre_parts);
    const int npre = (prefix_tokens + pre_pt - 1) / pre_pt;       // the prefix's partitions (<= pre_parts)
    if (!workspace || workspace_bytes < cascade_ws_bytes(num_seqs, num_q_heads, head_dim, pre_parts) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const CascadeWs ws = cascade_ws(workspace, num_seqs, num_q_heads, head_dim, npre);
    const int tail_cap = max_context_len - prefix_tokens;
    cascade_plan_kernel<<<1, kPlanThreads, 0, st>>>(context_lens, ws, num_seqs, prefix_tokens, max_context_len,
                                                     block_size, err);
    if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;

    MqParams p{};
    p.out = nullptr;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.ws_o = ws.pre_o;
    p.ws_ml = ws.pre_ml;
    p.err = err;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.num_parts = npre;           // the prefix partials of each row
    p.withhold = -1;
    p.wait_ns = kDefaultWaitNs;

    // 1. the prefix, once: B queries of one sequence, no causal mask, one partial per partition (tcgen05)
    {
        CUtensorMap mk, mv, mqm;
        const int box_rows = std::min(block_size, tc::TOK);
        if (!make_cache_map(&mk, k_cache, PKV_BF16, num_blocks, block_size, num_kv_heads, head_dim, true, box_rows) ||
            !make_cache_map(&mv, v_cache, PKV_BF16, num_blocks, block_size, num_kv_heads, head_dim, true, box_rows) ||
            !make_q_map(&mqm, q, num_seqs, num_q_heads, head_dim, group))
            return PKV_ERR_CUDA;
        MqParams pp = p;
        pp.block_tables = block_tables;                         // row 0: its first prefix / bs entries
        pp.context_lens = ws.ints;
        pp.query_start = ws.ints + 1;
        pp.num_seqs = 1;
        pp.num_tokens = num_seqs;
        pp.max_blocks = max_blocks_per_seq;
        pp.ctx_cap = prefix_tokens;
        pp.max_query_len = num_seqs;
        pp.part_blocks = pre_pt / block_size;
        pp.row_tiles = (int)(((int64_t)num_seqs * group + tc::ROWS - 1) / tc::ROWS);
        pp.wpr = 1;
        pp.causal = 0;
        pp.slot = 0;
        dim3 grid(num_kv_heads, npre, pp.row_tiles);
        if (launch_mq_tc_bs(block_size, mqm, mk, mv, pp, grid, st, /*pdl=*/true) != cudaSuccess) return PKV_ERR_CUDA;
    }
    // 2. each sequence's tail: its query over tokens prefix .. ctx - 1 (the decode kernel, longest tail
    //    first), merged with the prefix's partials into the output
    return decode_tails_with_prefix(out, out_dtype, q, k_cache, v_cache, block_tables + prefix_tokens / block_size,
                                    ws.units, scale, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                    max_blocks_per_seq, num_blocks, tail_cap, ws.pre_o, ws.pre_ml, npre, st);
}

}  // extern "C"
