// Pieces shared by the paged decode attention kernels: parameters, output
// store, and the two consumer implementations (CUDA-core and tensor-core) that
// fold one 16-token block of K/V into a running online-softmax state.
#pragma once

#include <cmath>

#include "common.cuh"

namespace pkv {
namespace attn {

constexpr int TILE_ROWS = 16;   // tokens of one tensor-core tile
constexpr int NCW = 4;          // consumer warps per CTA

// Block sizes built (tokens per physical block). A ring stage always holds a
// fixed number of tokens: 16 for 4- and 2-byte caches, 32 for FP8 caches. A
// stage is filled with "pieces" of piece_rows(bs) tokens: several whole blocks
// when bs is smaller than a stage, one slice of a block when it is larger.
constexpr bool block_size_built(int bs) { return bs == 8 || bs == 16 || bs == 32 || bs == 64; }
constexpr int stage_tokens(int elt_bytes) { return elt_bytes == 1 ? 32 : 16; }
constexpr int piece_rows(int bs, int elt_bytes) { return bs < stage_tokens(elt_bytes) ? bs : stage_tokens(elt_bytes); }
constexpr int NTHREADS = 32 * (NCW + 1);
constexpr int kPlanMaxBins = 4096;   // longest-first schedule: partitions of at most this many blocks
// Partitions per context from which the decode grid works through the unit list
// in about one wave (paged_attention_kernel.cuh, launch_decode).
constexpr int kLoopParts = 8;
constexpr float kNegInf = -INFINITY;

struct Params {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;        // [B, Hq, C, D] partition outputs (normalised)
    float* ws_ml;       // [B, Hq, C, 2] partition (m, l), m in log2 units
    int* err;
    float scale_log2;   // scale * log2(e) (times the K scale for an fp8 cache)
    float out_scale;    // 1, or the V scale for an fp8 cache
    int out_f32;
    int num_q_heads, num_kv_heads, group;
    int max_blocks, num_blocks;
    int ctx_cap;        // clamp for context_lens
    int block_size;     // tokens per physical block
    int part_blocks;    // blocks per partition
    int num_parts;      // grid.y
    // persistent schedule
    int num_seqs;
    float* ws_part;                 // [2 * CTAs][group][D + 2]: per-piece (o / l, m, l)
    unsigned long long* counters;   // [B * Hkv]: (epoch << 24) | pieces arrived
    unsigned long long epoch;       // distinct per call
    int team_size;                  // CTAs per team (one KV head each), divides Hkv and the grid
    // longest-first schedule of the partitioned kernel (plan_units_kernel)
    uint2* units;                   // [B * C]: {seq << 16 | partition, clamped context length}; NULL: grid order
    int* unit_count;                // live units listed
    // pre_parts > 0 (the tails of the shared-prefix cascade, one partition per
    // sequence): each (sequence, query head) merges the prefix's normalised
    // partials (pre_o [B, Hq, pre_parts, D], pre_ml [B, Hq, pre_parts, 2]: m in
    // log2 units, l) with its own result before writing the output
    const float* pre_o;
    const float* pre_ml;
    int pre_parts;
    // bounded waits
    unsigned long long wait_ns;     // limit of every mbarrier wait (2 s unless the test hook shortened it)
    int withhold;                   // test hook: ring stage whose copies the first CTA never issues (-1: none)
};

__device__ __forceinline__ void consumers_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

__device__ __forceinline__ void store_out(const Params& p, int64_t idx, float v) {
    v *= p.out_scale;
    if (p.out_f32) static_cast<float*>(p.out)[idx] = v;
    else static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
}

template <typename TQ>
__device__ __forceinline__ float to_float(TQ x) {
    if constexpr (sizeof(TQ) == 4) return x;
    else return __bfloat162float(x);
}

// ---------------------------------------------------------------------------
// SIMT consumer: HPW query heads per warp, 8 lanes per token, 4 tokens per
// round, fp32 math. T = float or __nv_bfloat16.
// ---------------------------------------------------------------------------
template <typename T, int D, int HPW, typename TQ = T, int TOK = TILE_ROWS>
struct SimtConsumer {
    static constexpr int RB = D * (int)sizeof(T);          // row bytes
    static constexpr int NCH = RB / 16;                     // 16-byte chunks per row
    static constexpr int CPL = NCH / 8;                     // chunks per lane
    static constexpr int EPC = 16 / (int)sizeof(T);         // elements per chunk
    static constexpr int EPL = CPL * EPC;                   // elements per lane
    static constexpr int ROUNDS = TOK / 4;                 // 4 tokens per round (8 lanes each)
    static_assert(NCH % 8 == 0, "row must hold a multiple of 8 chunks");

    float q[HPW][EPL];
    float acc[HPW][EPL];
    float m[HPW], l[HPW];

    __device__ __forceinline__ static void unpack(const uint4& raw, float* f) {
        if constexpr (sizeof(T) == 1) {          // 16 e4m3 codes
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 a = f16x2_to_float2(e4m3x2_to_f16x2(w[i] & 0xffffu));
                const float2 b = f16x2_to_float2(e4m3x2_to_f16x2(w[i] >> 16));
                f[4 * i] = a.x; f[4 * i + 1] = a.y; f[4 * i + 2] = b.x; f[4 * i + 3] = b.y;
            }
        } else if constexpr (sizeof(T) == 4) {
            f[0] = __uint_as_float(raw.x); f[1] = __uint_as_float(raw.y);
            f[2] = __uint_as_float(raw.z); f[3] = __uint_as_float(raw.w);
        } else {
            f[0] = bf16lo(raw.x); f[1] = bf16hi(raw.x); f[2] = bf16lo(raw.y); f[3] = bf16hi(raw.y);
            f[4] = bf16lo(raw.z); f[5] = bf16hi(raw.z); f[6] = bf16lo(raw.w); f[7] = bf16hi(raw.w);
        }
    }

    // q_rows points at query head (first head of this warp) of this sequence.
    // Lane li holds dims (c * 8 + li) * EPC + e of each head, the dims it reads of K and V.
    __device__ __forceinline__ void init(const TQ* q_rows, float scale_log2, int lane) {
        const int li = lane & 7;
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
#pragma unroll
            for (int c = 0; c < CPL; ++c)
#pragma unroll
                for (int e = 0; e < EPC; ++e)
                    q[h][c * EPC + e] = to_float(q_rows[(int64_t)h * D + (c * 8 + li) * EPC + e]) * scale_log2;
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
// Tensor-core consumer (bf16, up to 8 * NT query heads per KV head: NT 8-wide
// MMA n-tiles of query heads share every K and V fragment).
// Stage layout: for K then V, D/64 half-tiles of [16 rows x 128 B], each
// written by TMA with the 128-byte swizzle (16-byte chunk c of row r lives at
// chunk c ^ (r & 7)), so ldmatrix reads are bank-conflict free.
// ---------------------------------------------------------------------------
template <int D, int NT = 1>
struct MmaConsumer {
    static constexpr int KS = D / 16;          // k-steps of S^T = K Q^T
    static constexpr int MT = D / 16;          // m-tiles of O^T
    static constexpr int HALF = TILE_ROWS * 128;   // bytes of one 64-wide half tile

    uint32_t qb[NT][KS][2];                    // Q^T as B fragments (N = 8 query heads per n-tile)
    float o[NT][MT][4];                        // O^T fragments: dims x heads
    float m0[NT], m1[NT], l0[NT], l1[NT];      // heads 8 nt + 2t, 8 nt + 2t + 1

    __device__ __forceinline__ void init(const __nv_bfloat16* q_rows, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = 8 * nt + g;
            const uint32_t* row = reinterpret_cast<const uint32_t*>(q_rows + (int64_t)h * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                if (h < group) {
                    qb[nt][ks][0] = row[(ks * 16 + 2 * t) / 2];
                    qb[nt][ks][1] = row[(ks * 16 + 2 * t + 8) / 2];
                } else {
                    qb[nt][ks][0] = qb[nt][ks][1] = 0u;
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
            m0[nt] = m1[nt] = kNegInf;
            l0[nt] = l1[nt] = 0.f;
        }
    }

    __device__ __forceinline__ void consume(uint32_t ks_base, uint32_t vs_base, uint8_t* vs_ptr, int nvalid,
                                            float scale_log2, int lane) {
        const int g = lane >> 2, t = lane & 3;
        // Rows past the context may hold anything (NaN included): zero them in V,
        // so that p = 0 times the row stays 0. K rows are masked by select.
        if (nvalid < TILE_ROWS) {
            for (int i = lane; i < (TILE_ROWS - nvalid) * (D / 8); i += 32) {
                const int r = nvalid + i / (D / 8), cc = i % (D / 8);
                const int half = cc >> 3, c = cc & 7;
                *reinterpret_cast<uint4*>(vs_ptr + half * HALF + r * 128 + ((c ^ (r & 7)) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int r = lane & 15;
            const int c = ((ks & 3) << 1) + (lane >> 4);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, ks_base + (ks >> 2) * HALF + r * 128 + ((c ^ (r & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
        uint32_t bh0[NT], bh1[NT], bl0[NT], bl1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            // s[0]: (token g, head 2t)  s[1]: (g, 2t+1)  s[2]: (g+8, 2t)  s[3]: (g+8, 2t+1)
            const float x0 = g < nvalid ? s[nt][0] * scale_log2 : kNegInf;
            const float x1 = g < nvalid ? s[nt][1] * scale_log2 : kNegInf;
            const float x2 = g + 8 < nvalid ? s[nt][2] * scale_log2 : kNegInf;
            const float x3 = g + 8 < nvalid ? s[nt][3] * scale_log2 : kNegInf;
            float b0 = fmaxf(x0, x2), b1 = fmaxf(x1, x3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, off));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, off));
            }
            const float n0 = fmaxf(m0[nt], b0), n1 = fmaxf(m1[nt], b1);
            const float al0 = fast_exp2(m0[nt] - n0), al1 = fast_exp2(m1[nt] - n1);
            m0[nt] = n0;
            m1[nt] = n1;
            const float p0 = fast_exp2(x0 - n0), p1 = fast_exp2(x1 - n1);
            const float p2 = fast_exp2(x2 - n0), p3 = fast_exp2(x3 - n1);
            l0[nt] = l0[nt] * al0 + (p0 + p2);
            l1[nt] = l1[nt] * al1 + (p1 + p3);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                o[nt][mt][0] *= al0; o[nt][mt][1] *= al1; o[nt][mt][2] *= al0; o[nt][mt][3] *= al1;
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
            bh0[nt] = __byte_perm(ya, yb, 0x5410);
            bh1[nt] = __byte_perm(ya, yb, 0x7632);
            bl0[nt] = __byte_perm(za, zb, 0x5410);
            bl1[nt] = __byte_perm(za, zb, 0x7632);
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int mi = lane >> 3;
            const int tok = (lane & 7) + ((mi >> 1) << 3);
            const int c = (((mt * 16) & 63) >> 3) + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(a0, a1, a2, a3,
                              vs_base + ((mt * 16) >> 6) * HALF + tok * 128 + ((c ^ (tok & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, bh0[nt], bh1[nt]);
                mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, bl0[nt], bl1[nt]);
            }
        }
    }

    __device__ __forceinline__ void finish(float* red_o, float* red_m, float* red_l, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float a = l0[nt], b = l1[nt];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, off);
                b += __shfl_xor_sync(0xffffffffu, b, off);
            }
            const int h0 = 8 * nt + 2 * t, h1 = h0 + 1;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                if (h0 < group) {
                    red_o[h0 * D + mt * 16 + g] = o[nt][mt][0];
                    red_o[h0 * D + mt * 16 + g + 8] = o[nt][mt][2];
                }
                if (h1 < group) {
                    red_o[h1 * D + mt * 16 + g] = o[nt][mt][1];
                    red_o[h1 * D + mt * 16 + g + 8] = o[nt][mt][3];
                }
            }
            if (g == 0) {
                if (h0 < group) { red_m[h0] = m0[nt]; red_l[h0] = a; }
                if (h1 < group) { red_m[h1] = m1[nt]; red_l[h1] = b; }
            }
        }
    }
};


// ---------------------------------------------------------------------------
// Tensor-core consumer for an FP8 (e4m3) cache, D = 128, up to 8 query heads.
// The K and V tiles are 16 rows x 128 bytes, TMA-written with the 128-byte
// swizzle. ldmatrix reads the codes as 16-bit pairs and cvt turns each pair
// into f16x2 exactly; the MMAs run in f16 (q is converted once; P split into
// f16 high + low parts).
//   S^T = K Q^T: thread (g, t) gets the codes of dims 4t..4t+3 of a 16-dim
//   chunk; they serve as the fragment's k slots 2t, 2t+1, 2t+8, 2t+9, and Q's
//   B fragment is built with the same dim order, so the dot products are
//   unchanged.
//   O^T += V^T P^T: ldmatrix.trans gives a thread two dims (2g, 2g+1) of two
//   tokens; a byte permute splits them into the even-dim row (fragment row g)
//   and the odd-dim row (fragment row g + 8), so each 16-dim chunk is one MMA
//   whose output rows are dims 2g and 2g + 1.
// ---------------------------------------------------------------------------
template <int NT, int NH = 1>      // 16-token tiles per stage (1 or 2); 8-wide query-head tiles (1 or 2)
struct MmaConsumerFp8 {
    static constexpr int D = 128;
    static constexpr int NCHUNK = D / 16;
    static constexpr int TOK = 16 * NT;

    uint32_t qb[NH][NCHUNK][2];
    float o[NH][NCHUNK][4];
    float m0[NH], m1[NH], l0[NH], l1[NH];

    __device__ __forceinline__ static uint32_t f16pair(float a, float b) {
        return pack_f16(fminf(fmaxf(a, -65504.f), 65504.f), fminf(fmaxf(b, -65504.f), 65504.f));
    }

    __device__ __forceinline__ void init(const __nv_bfloat16* q_rows, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) {
            const int h = 8 * nh + g;
#pragma unroll
            for (int ks = 0; ks < NCHUNK; ++ks) {
                if (h < group) {
                    const uint2 w = *reinterpret_cast<const uint2*>(q_rows + (int64_t)h * D + 16 * ks + 4 * t);
                    qb[nh][ks][0] = f16pair(bf16lo(w.x), bf16hi(w.x));
                    qb[nh][ks][1] = f16pair(bf16lo(w.y), bf16hi(w.y));
                } else {
                    qb[nh][ks][0] = qb[nh][ks][1] = 0u;
                }
            }
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c) o[nh][c][0] = o[nh][c][1] = o[nh][c][2] = o[nh][c][3] = 0.f;
            m0[nh] = m1[nh] = kNegInf;
            l0[nh] = l1[nh] = 0.f;
        }
    }

    // P^T of one 16-token tile as f16 B fragments (high and low parts).
    __device__ __forceinline__ static void p_fragments(float p0, float p1, float p2, float p3, int lane,
                                                       uint32_t& bh0, uint32_t& bh1, uint32_t& bl0, uint32_t& bl1) {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t h02 = pack_f16(p0, p2), h13 = pack_f16(p1, p3);
        const float2 f02 = f16x2_to_float2(h02), f13 = f16x2_to_float2(h13);
        const uint32_t e02 = pack_f16(p0 - f02.x, p2 - f02.y), e13 = pack_f16(p1 - f13.x, p3 - f13.y);
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
        bh0 = __byte_perm(ya, yb, 0x5410);
        bh1 = __byte_perm(ya, yb, 0x7632);
        bl0 = __byte_perm(za, zb, 0x5410);
        bl1 = __byte_perm(za, zb, 0x7632);
    }

    // One even/odd-dim MMA pair input from two ldmatrix.trans registers (tokens 0-7, 8-15 of a tile),
    // applied to every head tile.
    __device__ __forceinline__ void pv(int c, uint32_t rlo, uint32_t rhi, const uint32_t (&bh)[NH][2],
                                       const uint32_t (&bl)[NH][2]) {
        const uint32_t x = __byte_perm(rlo, 0u, 0x3120), y = __byte_perm(rhi, 0u, 0x3120);
        const uint32_t a0 = e4m3x2_to_f16x2(x & 0xffffu), a1 = e4m3x2_to_f16x2(x >> 16);
        const uint32_t a2 = e4m3x2_to_f16x2(y & 0xffffu), a3 = e4m3x2_to_f16x2(y >> 16);
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) {
            mma_f16_16816(o[nh][c], a0, a1, a2, a3, bh[nh][0], bh[nh][1]);
            mma_f16_16816(o[nh][c], a0, a1, a2, a3, bl[nh][0], bl[nh][1]);
        }
    }

    __device__ __forceinline__ void consume(uint32_t ks_base, uint32_t vs_base, uint8_t* vs_ptr, int nvalid,
                                            float scale_log2, int lane) {
        const int g = lane >> 2;
        if (nvalid < TOK) {         // rows past the context: zero V codes (0 * NaN would poison O)
            for (int i = lane; i < (TOK - nvalid) * 8; i += 32) {
                const int r = nvalid + i / 8, c = i % 8;
                *reinterpret_cast<uint4*>(vs_ptr + r * 128 + ((c ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        float s[NH][NT][4];
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) s[nh][tt][0] = s[nh][tt][1] = s[nh][tt][2] = s[nh][tt][3] = 0.f;
        const int mi = lane >> 3;
        const int row = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
        for (int kp = 0; kp < NCHUNK / 2; ++kp) {
            const int chunk = 2 * kp + (mi >> 1);
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                const int r = tt * 16 + row;
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4(r0, r1, r2, r3, ks_base + r * 128 + ((chunk ^ (r & 7)) << 4));
                const uint32_t k00 = e4m3x2_to_f16x2(r0 & 0xffffu), k01 = e4m3x2_to_f16x2(r1 & 0xffffu);
                const uint32_t k02 = e4m3x2_to_f16x2(r0 >> 16), k03 = e4m3x2_to_f16x2(r1 >> 16);
                const uint32_t k10 = e4m3x2_to_f16x2(r2 & 0xffffu), k11 = e4m3x2_to_f16x2(r3 & 0xffffu);
                const uint32_t k12 = e4m3x2_to_f16x2(r2 >> 16), k13 = e4m3x2_to_f16x2(r3 >> 16);
#pragma unroll
                for (int nh = 0; nh < NH; ++nh) {
                    mma_f16_16816(s[nh][tt], k00, k01, k02, k03, qb[nh][2 * kp][0], qb[nh][2 * kp][1]);
                    mma_f16_16816(s[nh][tt], k10, k11, k12, k13, qb[nh][2 * kp + 1][0], qb[nh][2 * kp + 1][1]);
                }
            }
        }
        uint32_t bh[NT][NH][2], bl[NT][NH][2];
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) {
            float x[NT][4];
            float b0 = kNegInf, b1 = kNegInf;
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                x[tt][0] = tt * 16 + g < nvalid ? s[nh][tt][0] * scale_log2 : kNegInf;
                x[tt][1] = tt * 16 + g < nvalid ? s[nh][tt][1] * scale_log2 : kNegInf;
                x[tt][2] = tt * 16 + g + 8 < nvalid ? s[nh][tt][2] * scale_log2 : kNegInf;
                x[tt][3] = tt * 16 + g + 8 < nvalid ? s[nh][tt][3] * scale_log2 : kNegInf;
                b0 = fmaxf(b0, fmaxf(x[tt][0], x[tt][2]));
                b1 = fmaxf(b1, fmaxf(x[tt][1], x[tt][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, off));
                b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, off));
            }
            const float n0 = fmaxf(m0[nh], b0), n1 = fmaxf(m1[nh], b1);
            const float al0 = fast_exp2(m0[nh] - n0), al1 = fast_exp2(m1[nh] - n1);
            m0[nh] = n0;
            m1[nh] = n1;
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                const float p0 = fast_exp2(x[tt][0] - n0), p1 = fast_exp2(x[tt][1] - n1);
                const float p2 = fast_exp2(x[tt][2] - n0), p3 = fast_exp2(x[tt][3] - n1);
                ps0 += p0 + p2;
                ps1 += p1 + p3;
                p_fragments(p0, p1, p2, p3, lane, bh[tt][nh][0], bh[tt][nh][1], bl[tt][nh][0], bl[tt][nh][1]);
            }
            l0[nh] = l0[nh] * al0 + ps0;
            l1[nh] = l1[nh] * al1 + ps1;
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c) {
                o[nh][c][0] *= al0; o[nh][c][1] *= al1; o[nh][c][2] *= al0; o[nh][c][3] *= al1;
            }
        }
        if constexpr (NT == 1) {
            const int tok = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
            for (int cp = 0; cp < NCHUNK / 2; ++cp) {
                const int chunk = 2 * cp + (mi >> 1);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, vs_base + tok * 128 + ((chunk ^ (tok & 7)) << 4));
                // r0: tokens 0-7 of chunk 2cp, r1: tokens 8-15 of it; r2, r3: chunk 2cp + 1
                pv(2 * cp, r0, r1, bh[0], bl[0]);
                pv(2 * cp + 1, r2, r3, bh[0], bl[0]);
            }
        } else {
            // one ldmatrix.x4.trans per chunk: tokens 0-7, 8-15 (tile 0) and 16-23, 24-31 (tile 1)
            const int tok = (mi >> 1) * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c) {
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, vs_base + tok * 128 + ((c ^ (tok & 7)) << 4));
                pv(c, r0, r1, bh[0], bl[0]);
                pv(c, r2, r3, bh[1], bl[1]);
            }
        }
    }

    __device__ __forceinline__ void finish(float* red_o, float* red_m, float* red_l, int group, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) {
            float a = l0[nh], b = l1[nh];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, off);
                b += __shfl_xor_sync(0xffffffffu, b, off);
            }
            const int h0 = 8 * nh + 2 * t, h1 = h0 + 1;
#pragma unroll
            for (int c = 0; c < NCHUNK; ++c) {
                const int de = 16 * c + 2 * g;            // fragment rows g / g + 8 are dims de / de + 1
                if (h0 < group) {
                    red_o[h0 * D + de] = o[nh][c][0];
                    red_o[h0 * D + de + 1] = o[nh][c][2];
                }
                if (h1 < group) {
                    red_o[h1 * D + de] = o[nh][c][1];
                    red_o[h1 * D + de + 1] = o[nh][c][3];
                }
            }
            if (g == 0) {
                if (h0 < group) { red_m[h0] = m0[nh]; red_l[h0] = a; }
                if (h1 < group) { red_m[h1] = m1[nh]; red_l[h1] = b; }
            }
        }
    }
};

// Partitioned schedule, one instantiation per block size (paged_attention_bs*.cu):
// picks the consumer path for the cache dtype, head size and group and launches
// the pipelined kernel over grid (Hkv, partitions, sequences).
template <int BSZ>
cudaError_t dispatch_partitioned(pkv_dtype kv_dtype, bool use_mma, int head_dim, int group, int num_kv_heads,
                                 const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                                 cudaStream_t st);

// Tensor map over a cache [nb, bs, hkv, d] (paged_attention.cu): box = piece_rows(bs)
// tokens of one head, whole rows (SIMT) or 128-byte swizzled box rows (tensor cores).
// box_rows > 0 overrides the piece height (a divisor of bs, at most 256).
bool make_cache_map(CUtensorMap* map, const void* base, pkv_dtype dt, int nb, int bs, int hkv, int d, bool mma,
                    int box_rows = 0);

// Persistent schedule (paged_attention_persistent.cu).
cudaError_t launch_persistent(bool bf16, bool use_mma, int head_dim, int group, const CUtensorMap& mk,
                              const CUtensorMap& mv, const Params& p, int grid, cudaStream_t st);
int persistent_ctas_per_sm();
int persistent_max_seqs();
// SMs of the current device (paged_attention.cu).
int num_sms();
// The tails of the shared-prefix cascade (paged_attention_mq.cu): one decode
// pass (bf16 cache, one partition per sequence) over the table rows past the
// prefix, in the longest-first order that `units` already lists (B entries and
// their count, from list_units), launched as a programmatic dependent of the
// call before it on the stream, which has written the prefix's partials; each
// (sequence, query head) merges them into its result and writes the output.
pkv_status decode_tails_with_prefix(void* out, pkv_dtype out_dtype, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* block_tables, const uint2* units,
                                    float scale, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int num_blocks, int ctx_cap,
                                    const float* pre_o, const float* pre_ml, int pre_parts, cudaStream_t st);

}  // namespace attn
}  // namespace pkv
