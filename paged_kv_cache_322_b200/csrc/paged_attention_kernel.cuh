// The pipelined paged decode kernel (partitioned schedule), templated on the
// cache element type, head size, consumer path, ring depth, KV heads per CTA
// and block size. Included by one translation unit per block size
// (paged_attention_bs*.cu), which instantiates dispatch_partitioned<BSZ>; the
// host side (tensor maps, schedule, argument checks, merge) is in
// paged_attention.cu. The design is described at the top of that file.
#pragma once

#include <atomic>
#include <type_traits>

#include "attention_common.cuh"

namespace pkv {
namespace attn {

// ---------------------------------------------------------------------------
// The pipelined kernel.
//   PATH 0: SIMT, block-split (each consumer warp takes whole blocks, HPW = group)
//   PATH 1: SIMT, head-split (every warp reads every block, HPW = group / NCW)
//   PATH 2: tensor cores, block-split (group <= HPW: 8, or 16 as two 8-wide head tiles)
// ---------------------------------------------------------------------------
template <typename T, int D, int PATH, int HPW, int STAGES, int KPC, int BSZ>
struct Kern {
    static constexpr bool kMma = PATH == 2;
    static constexpr int EB = (int)sizeof(T);
    static constexpr int BOX = 128 / EB;                               // elements per swizzled 128-byte box row
    static constexpr int NBOX = D * EB / 128;                          // boxes per row (tensor-core path)
    // A stage holds TOK tokens (16, or 32 for FP8 whose rows are half as long),
    // filled with BPS pieces of R rows: whole blocks when BSZ < TOK, else one
    // R-row slice of a block (a block then spans PPB pieces).
    static constexpr int TOK = stage_tokens(EB);
    static constexpr int R = piece_rows(BSZ, EB);
    static constexpr int BPS = TOK / R;                                // pieces per stage
    static constexpr int PPB = BSZ / R;                                // pieces per block
    static constexpr int PIECE = R * D * EB;                           // one piece, one head, K or V
    static constexpr int REGION = TOK * D * EB;                        // one head's K (or V) in a stage
    static_assert(BPS * R == TOK && PPB * R == BSZ, "block size must be a power of two >= 8");
    // KPC KV heads per CTA: their tiles are loaded back to back, so a token row's
    // neighbouring heads (adjacent in HBM) are read together; consumer warps split
    // by head (WPH warps per head). Stage layout: K [head][TOK rows], then V; on
    // the tensor-core path each head's rows are split in 128-byte box columns.
    static constexpr int WPH = NCW / KPC;
    static constexpr int STAGE_BYTES = 2 * KPC * REGION;
    // Byte offset of piece b (of BPS), box column h, inside one head's region.
    __device__ __forceinline__ static int piece_offset(int b, int h) {
        return kMma ? h * (TOK * 128) + b * (R * 128) : b * PIECE;
    }
    static_assert(PATH != 1 || KPC == 1, "head-split consumers serve one KV head");
    static constexpr int RING = STAGES * STAGE_BYTES;
    static constexpr int NSLOT = PATH == 1 ? 1 : NCW;                  // partial states to merge
    static constexpr int MAXG = PATH == 2 ? HPW : (PATH == 1 ? HPW * NCW : HPW);
    static_assert(PATH != 2 || HPW == 8 || HPW == 16, "tensor-core consumers take one or two 8-wide head tiles");
    static constexpr int RED = NSLOT * MAXG * (D + 2) * 4;
    static constexpr int BODY = RING > RED ? RING : RED;
    static constexpr int SMEM = 1024 /*align slack*/ + BODY + 2 * STAGES * 8;
    static_assert(RED <= BODY, "reduction scratch must fit");
    // Block-split consumers take tiles round-robin; with STAGES a multiple of NCW
    // every round of a stage goes to the same warp, so no warp can wait on a ring
    // phase two rounds ahead of the producer (the parity wait would pass early).
    static_assert(PATH == 1 || STAGES % WPH == 0, "ring depth must be a multiple of the warps per head");
};

// LOOP: the CTA works through the unit list (a grid of about one wave; see below);
// without it every CTA takes one unit (row) and the kernel has no loop at all.
template <typename T, int D, int PATH, int HPW, int STAGES, int KPC, int BSZ, bool LOOP>
__global__ void __launch_bounds__(NTHREADS, 3)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const Params p) {
    using K = Kern<T, D, PATH, HPW, STAGES, KPC, BSZ>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::BODY);
    uint64_t* empty = full + STAGES;
    __shared__ volatile int s_abort;

    const int kvh = blockIdx.x * KPC;                             // first KV head of this CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Barriers and tensor-map prefetch first: under the longest-first schedule
    // this overlaps the plan kernel, which the unit read below waits for.
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
    // Longest-first schedule: the plan kernel, this launch's programmatic
    // predecessor, listed the units, and row y of the grid takes listed row y.
    // With LOOP (contexts spanning many partitions, where most of the B x C
    // rows would find no unit: ~7000 such CTAs kept a long-context launch busy
    // ~6 us past its last unit) the grid is about one wave and row y also takes
    // listed rows y + gridDim.y, y + 2 gridDim.y, ... The ring's barriers carry
    // over from unit to unit: `base` counts the stages this CTA streamed before
    // the current unit, and every unit ends with a CTA barrier (the reduction
    // scratch aliases the ring), so a unit's first stages never meet an
    // unconsumed stage of the one before.
    int count = 1;
    if (p.units) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        count = *p.unit_count;
    }
    uint32_t base = 0;
    for (int row = blockIdx.y;;) {
    int part, seq, ctx;
    if (p.units) {
        if (row >= count) return;                                 // no unit left for this row (uniform)
        const uint2 u = p.units[row];
        seq = (int)(u.x >> 16);
        part = (int)(u.x & 0xffffu);
        ctx = (int)u.y;                                           // clamped (and flagged) by the plan kernel
    } else {
        part = blockIdx.y;
        seq = blockIdx.z;
        ctx = p.context_lens[seq];
        if (ctx < 0 || ctx > p.ctx_cap) {
            if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
            ctx = ctx < 0 ? 0 : p.ctx_cap;
        }
    }
    const int nblk_seq = (ctx + BSZ - 1) / BSZ;
    const int nparts = (nblk_seq + p.part_blocks - 1) / p.part_blocks;
    if (part > 0 && part >= nparts) return;                       // beyond this sequence's context
    const int blk0 = part * p.part_blocks;
    const int nblk = max(0, min(p.part_blocks, nblk_seq - blk0));
    const int ntok = max(0, min(p.part_blocks * BSZ, ctx - blk0 * BSZ));   // tokens of this partition
    const int npiece = (ntok + K::R - 1) / K::R;
    const int nstage = (npiece + K::BPS - 1) / K::BPS;
    const int group = p.group;
    const int64_t qh0 = (int64_t)kvh * group;                     // first query head of this KV head

    __syncthreads();   // the barriers are initialised; the previous unit is done with the ring

    float* red_o = reinterpret_cast<float*>(smem);
    float* red_m = red_o + K::NSLOT * K::MAXG * D;
    float* red_l = red_m + K::NSLOT * K::MAXG;

    int issued = (int)base;                                       // ring stages claimed so far (producer lane 0)
    // test hook: the first CTA never issues this stage's copies (and never
    // arrives on its barrier), so its consumer's bounded wait runs out
    const int withheld = (blockIdx.x | blockIdx.y | blockIdx.z) == 0 ? p.withhold : -1;
    if (warp == 0) {
        // ---------------- producer ----------------
        const uint64_t pol = l2_policy_evict_first();
        const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks + blk0;
        bool ok = true;
        // 32 blocks' ids per coalesced load; each block gives PPB pieces, the
        // pieces past the partition's last token are not loaded.
        for (int q0 = 0; q0 < npiece && ok; q0 += 32 * K::PPB) {   // (stage g = base + local stage)
            const int j0 = q0 / K::PPB;
            int id = 0;
            if (j0 + lane < nblk) {
                id = __ldg(bt + j0 + lane);
                if (id < 0 || id >= p.num_blocks) {
                    flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                    id = p.num_blocks;                            // TMA fills an out-of-range tile with zeros
                }
            }
            const int qn = min(32 * K::PPB, npiece - q0);
            // One stage per iteration (BPS pieces; BPS divides 32 * PPB, so a stage
            // never straddles two id loads). Lane 0 claims the stage; then lane o
            // issues copy o of the stage's BPS x KPC x boxes x {K, V} copies, in
            // parallel instead of one thread issuing them all.
            constexpr int NB = K::kMma ? K::NBOX : 1;
            static_assert(K::BPS * KPC * NB * 2 <= 32, "one copy per lane");
            const int kv = lane & 1, hb = lane >> 1;
            const int h = hb % NB, hd = (hb / NB) % KPC, b = hb / (NB * KPC);
            for (int qs = 0; qs < qn; qs += K::BPS) {
                const int q = q0 + qs, si = (int)base + q / K::BPS, st = si % STAGES;
                const int nq = min(K::BPS, npiece - q);               // pieces in this stage
                if (lane == 0) {
                    if (!mbar_wait_bounded(&empty[st], ((si / STAGES) & 1) ^ 1, p.err, p.wait_ns)) {
                        ok = false;
                        s_abort = 1;
                    } else {
                        if (si != withheld) mbar_arrive_expect_tx(&full[st], nq * 2 * KPC * K::PIECE);
                        issued = si + 1;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;    // also orders the expect-tx first
                if (!ok) break;
                const int pq = qs + (b < nq ? b : 0);                // this lane's piece, chunk-relative
                const int pb = __shfl_sync(0xffffffffu, id, pq / K::PPB);
                if (b < nq && si != withheld) {
                    uint8_t* dst = smem + st * K::STAGE_BYTES + (kv ? KPC + hd : hd) * K::REGION + K::piece_offset(b, h);
                    tma_load_4d(dst, kv ? &tm_v : &tm_k, &full[st], h * K::BOX, kvh + hd, (pq % K::PPB) * K::R, pb, pol);
                }
            }
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 1;
        const int hd = cw / K::WPH, sub = cw - hd * K::WPH;               // this warp's KV head, and its turn
        using TQ = std::conditional_t<sizeof(T) == 1, __nv_bfloat16, T>;   // an fp8 cache takes bf16 queries
        const TQ* qbase = static_cast<const TQ*>(p.q) + ((int64_t)seq * p.num_q_heads + qh0 + hd * group) * D;
        const int kofs = hd * K::REGION, vofs = (KPC + hd) * K::REGION;
        if constexpr (PATH == 2) {
            using Cons = std::conditional_t<sizeof(T) == 1, MmaConsumerFp8<K::TOK / TILE_ROWS, HPW / 8>,
                                            MmaConsumer<D, HPW / 8>>;
            Cons c;
            c.init(reinterpret_cast<const __nv_bfloat16*>(qbase), group, lane);
            for (int j = sub; j < nstage; j += K::WPH) {
                const int g = (int)base + j, st = g % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (g / STAGES) & 1, p.err, p.wait_ns);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {   // warp-uniform exit
                    s_abort = 1;
                    break;
                }
                uint8_t* stage = smem + st * K::STAGE_BYTES;
                const int nvalid = min(K::TOK, ntok - j * K::TOK);
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
                const int g = (int)base + j, st = g % STAGES;
                const bool got = mbar_wait_bounded(&full[st], (g / STAGES) & 1, p.err, p.wait_ns);
                if (__any_sync(0xffffffffu, !got || s_abort != 0)) {
                    s_abort = 1;
                    break;
                }
                const uint8_t* stage = smem + st * K::STAGE_BYTES;
                c.consume(stage + kofs, stage + vofs, min(K::TOK, ntok - j * K::TOK), lane);
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
    if (s_abort) {
        // A wait gave up (here or in a consumer). Every copy this CTA issued lands
        // before it exits: the producer may have issued all of them and left its
        // loop before a consumer gave up. (Bounded; stages already consumed pass at once.)
        if (warp == 0 && lane == 0)
            for (int j = max((int)base, issued - STAGES); j < issued; ++j)
                if (j != withheld) mbar_wait_bounded(&full[j % STAGES], (j / STAGES) & 1, p.err, p.wait_ns);
        return;
    }

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
        const int64_t qh = (int64_t)seq * p.num_q_heads + qh0 + hd * group + h;
        if (nparts <= 1 && p.pre_parts > 0) {
            // the shared prefix's partials and this tail: out = sum w_i o_i / sum w_i
            const float* pm = p.pre_ml + qh * p.pre_parts * 2;
            const float* po = p.pre_o + qh * p.pre_parts * D + d;
            float Mx = M;
            for (int i = 0; i < p.pre_parts; ++i) Mx = fmaxf(Mx, pm[2 * i]);
            float Lx = 0.f, Ox = 0.f;
            if (Mx != kNegInf) {
                if (M != kNegInf) {
                    const float sc = fast_exp2(M - Mx);
                    Lx = L * sc;
                    Ox = O * sc;
                }
                for (int i = 0; i < p.pre_parts; ++i) {
                    const float mi = pm[2 * i];
                    if (mi == kNegInf) continue;
                    const float w = pm[2 * i + 1] * fast_exp2(mi - Mx);
                    Lx += w;
                    Ox += w * po[(int64_t)i * D];
                }
            }
            store_out(p, qh * D + d, Lx > 0.f ? Ox / Lx : 0.f);
        } else if (nparts <= 1) {
            store_out(p, qh * D + d, L > 0.f ? O / L : 0.f);
        } else {
            const float val = L > 0.f ? O / L : 0.f;
            p.ws_o[(qh * C + part) * D + d] = val;
            if (d == 0) {
                p.ws_ml[(qh * C + part) * 2 + 0] = M;
                p.ws_ml[(qh * C + part) * 2 + 1] = L;
            }
        }
    }
    if constexpr (!LOOP) {
        return;                                                   // one unit per CTA
    } else {
        base += (uint32_t)nstage;
        row += gridDim.y;
    }
    }
}

template <typename T, int D, int PATH, int HPW, int STAGES, int KPC, int BSZ, bool LOOP>
cudaError_t launch_decode_as(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                             cudaStream_t stream) {
    using K = Kern<T, D, PATH, HPW, STAGES, KPC, BSZ>;
    auto kern = paged_decode_kernel<T, D, PATH, HPW, STAGES, KPC, BSZ, LOOP>;
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
    if (p.units) {
        // LOOP with many partitions: about one wave of CTAs (three per SM) works through the unit list
        if (LOOP && p.num_parts >= kLoopParts)
            grid.y = std::min<unsigned>(grid.y, (unsigned)std::max(1, 3 * num_sms() / (int)grid.x));
        // a programmatic dependent of the plan kernel: launched while it runs, the
        // CTAs wait for its list in-kernel (griddepcontrol.wait)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = K::SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, mk, mv, p);
    }
    kern<<<grid, NTHREADS, K::SMEM, stream>>>(mk, mv, p);
    return cudaGetLastError();
}

// The unit-list loop is built for 16-token blocks (the shape of the long-context
// workload) and used when a context can span kLoopParts or more partitions, where
// the list can be much shorter than B x partitions; elsewhere every CTA takes one
// unit. Same-box A/B: long-context 512-token partitions 52.3 -> 48.3 us; with two
// partitions (70B shape, 32 sequences) one unit per CTA is faster (68.7 vs 74.8
// us: a fixed stride left some CTAs two long units, and claiming rows from a
// counter as units finish still cost 3 %); compiled into the one-unit kernel, the
// loop alone cost ~1 % on single-partition calls.
template <typename T, int D, int PATH, int HPW, int STAGES, int KPC, int BSZ>
cudaError_t launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t stream) {
    if constexpr (BSZ == 16) {
        // e4m3 caches take the loop build for every listed schedule: compiled with the
        // loop, its fragments fit the 128 registers (no spill; 48-52 bytes without),
        // and with a grid of one row per unit the loop runs once
        if (p.units && (p.num_parts >= kLoopParts || sizeof(T) == 1))
            return launch_decode_as<T, D, PATH, HPW, STAGES, KPC, BSZ, true>(mk, mv, p, grid, stream);
    }
    return launch_decode_as<T, D, PATH, HPW, STAGES, KPC, BSZ, false>(mk, mv, p, grid, stream);
}

// Ring depth: about 64 KB of stages per CTA (8 KB per stage for bf16 D=128),
// so three CTAs fit on an SM with ~190 KB of KV in flight.
template <typename T, int D, int KPC = 1>
constexpr int stages_for() {
    constexpr int sb = 2 * KPC * stage_tokens((int)sizeof(T)) * D * (int)sizeof(T);   // Kern::STAGE_BYTES
    constexpr int n = 65536 / sb;
    return n < 4 ? 4 : (n > 16 ? 16 : n);
}

template <typename T, int D, int BSZ, int KPC = 1>
cudaError_t dispatch_simt(int group, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                          cudaStream_t st) {
    switch (group) {
        case 1: return launch_decode<T, D, 0, 1, stages_for<T, D, KPC>(), KPC, BSZ>(mk, mv, p, grid, st);
        case 2: return launch_decode<T, D, 0, 2, stages_for<T, D, KPC>(), KPC, BSZ>(mk, mv, p, grid, st);
        case 4: return KPC == 1 ? launch_decode<T, D, 1, 1, stages_for<T, D>(), 1, BSZ>(mk, mv, p, grid, st)
                                : cudaErrorInvalidValue;
        case 8: return KPC == 1 ? launch_decode<T, D, 1, 2, stages_for<T, D>(), 1, BSZ>(mk, mv, p, grid, st)
                                : cudaErrorInvalidValue;
        case 16: return KPC == 1 ? launch_decode<T, D, 1, 4, stages_for<T, D>(), 1, BSZ>(mk, mv, p, grid, st)
                                 : cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

// Tensor-core consumers for groups up to HG (8: one 8-wide head tile, 16: two).
template <int BSZ, int HG>
cudaError_t dispatch_mma(pkv_dtype kv_dtype, int head_dim, int num_kv_heads, const CUtensorMap& mk,
                         const CUtensorMap& mv, const Params& p, dim3 grid, cudaStream_t st) {
    if (kv_dtype == PKV_FP8_E4M3) {
        // Two KV heads per CTA: each token's 256 contiguous bytes of K (and of V)
        // are fetched in one go instead of two 128-byte halves by different CTAs.
        return num_kv_heads % 2 == 0
                   ? launch_decode<uint8_t, 128, 2, HG, stages_for<uint8_t, 128, 2>(), 2, BSZ>(mk, mv, p, grid, st)
                   : launch_decode<uint8_t, 128, 2, HG, stages_for<uint8_t, 128>(), 1, BSZ>(mk, mv, p, grid, st);
    }
    // bf16: 8-token blocks make 1 KB copies per head, so two KV heads per CTA
    // (measured on B200, 70B-shaped GQA: +16% at block size 8, within 3% at
    // 16-64 where halving the CTA count costs long-context, small batches far more).
    if (HG == 8 && BSZ < 16 && head_dim == 128 && num_kv_heads % 2 == 0)
        return launch_decode<__nv_bfloat16, 128, 2, HG, stages_for<__nv_bfloat16, 128, 2>(), 2, BSZ>(mk, mv, p, grid,
                                                                                                   st);
    return head_dim == 128
               ? launch_decode<__nv_bfloat16, 128, 2, HG, stages_for<__nv_bfloat16, 128>(), 1, BSZ>(mk, mv, p, grid, st)
               : launch_decode<__nv_bfloat16, 64, 2, HG, stages_for<__nv_bfloat16, 64>(), 1, BSZ>(mk, mv, p, grid, st);
}

template <int BSZ>
cudaError_t dispatch_partitioned(pkv_dtype kv_dtype, bool use_mma, int head_dim, int group, int num_kv_heads,
                                 const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, dim3 grid,
                                 cudaStream_t st) {
    // e4m3 always runs on tensor cores (use_mma is set for it)
    if (use_mma || kv_dtype == PKV_FP8_E4M3)
        return group <= 8 ? dispatch_mma<BSZ, 8>(kv_dtype, head_dim, num_kv_heads, mk, mv, p, grid, st)
                          : dispatch_mma<BSZ, 16>(kv_dtype, head_dim, num_kv_heads, mk, mv, p, grid, st);
    if (kv_dtype == PKV_BF16)
        return head_dim == 128 ? dispatch_simt<__nv_bfloat16, 128, BSZ>(group, mk, mv, p, grid, st)
                               : dispatch_simt<__nv_bfloat16, 64, BSZ>(group, mk, mv, p, grid, st);
    return head_dim == 128 ? dispatch_simt<float, 128, BSZ>(group, mk, mv, p, grid, st)
                           : dispatch_simt<float, 64, BSZ>(group, mk, mv, p, grid, st);
}

}  // namespace attn
}  // namespace pkv
