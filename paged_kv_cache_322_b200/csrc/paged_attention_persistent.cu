// Persistent, evenly split schedule for paged decode attention.
//
// Same computation as the partitioned kernel in paged_attention.cu (softmax
// attention of each sequence's one query per head over its block-table-addressed
// K/V; "LLM 推理引擎内部原理" §2.4), scheduled differently:
//
//   * CTAs form teams of `team_size` (normally Hkv): member m of a team serves
//     KV heads m, m + team_size, ... Units are (sequence s, head row gg, block j)
//     with Hkv / team_size head rows per sequence; the batch is
//     U = (Hkv / team_size) * sum_s ceil(ctx_s / 16) units and team t owns the
//     contiguous range [t U / NT, (t+1) U / NT). Every CTA gets the same number
//     of tiles, so no CTA waits on a long sequence at the end, and the members of
//     a team read the different heads of the same physical blocks side by side
//     (a block of all heads is one contiguous span in HBM).
//   * Inside its range a CTA meets a few segments (the run of tiles of one
//     (s, g) item). One producer warp streams every tile of the range through
//     the TMA ring without stopping at segment boundaries, and fetches each
//     segment's query rows with a 1-D bulk copy into a small query ring.
//   * Consumer warps fold tiles into online-softmax states as in the partitioned
//     kernel. At a segment end they merge their states; a segment that is the
//     whole item writes the output, otherwise it writes a (o/l, m, l) piece to
//     the workspace and bumps the item's counter; the CTA that brings the count
//     to the number of pieces merges all pieces (log-sum-exp) and writes the
//     output. No second kernel, no spin-wait on another CTA.
//   * The host clears the counters on the stream before each launch (B * Hkv
//     words of the workspace), so a counter never starts from bytes an earlier
//     call left behind; each also carries an epoch that is new on every call.
#include <atomic>

#include "attention_common.cuh"

namespace pkv {
namespace attn {

constexpr int PBS = 16;     // the persistent schedule serves 16-token blocks only

constexpr int kPersistCtasPerSm = 2;
constexpr int kQStages = 4;
constexpr int kMaxSeqsPersistent = 2048;
constexpr unsigned long long kCountMask = (1ull << 24) - 1;

template <typename T, int D, int PATH, int HPW, int STAGES>
struct PKern {
    static constexpr bool kMma = PATH == 2;
    static constexpr int TILE = PBS * D * (int)sizeof(T);
    static constexpr int STAGE_BYTES = 2 * TILE;
    static constexpr int RING = STAGES * STAGE_BYTES;
    static constexpr int MAXG = PATH == 2 ? 8 : (PATH == 1 ? HPW * NCW : HPW);
    static constexpr int QBYTES = ((MAXG * D * (int)sizeof(T)) + 127) / 128 * 128;
    static constexpr int NSLOT = PATH == 1 ? 1 : NCW;
    static constexpr int RED = NSLOT * MAXG * (D + 2) * 4;
    static constexpr int OFF_Q = RING;
    static constexpr int OFF_RED = OFF_Q + kQStages * QBYTES;
    static constexpr int OFF_PREFIX = OFF_RED + RED;
    static constexpr int OFF_CTX = OFF_PREFIX + (kMaxSeqsPersistent + 1) * 4;
    static constexpr int OFF_BAR = (OFF_CTX + kMaxSeqsPersistent * 4 + 7) / 8 * 8;
    static constexpr int NBAR = 2 * STAGES + 2 * kQStages;
    static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8;
    // Same rule as the partitioned kernel: every round of a stage must go to the
    // same consumer warp, or a parity wait can pass on a phase two rounds stale.
    static_assert(PATH == 1 || STAGES % NCW == 0, "ring depth must be a multiple of the consumer warps");
};

struct Seg {
    int s, gg, g, j0, j1, nblk, ctx;
    long long t_begin;
};

// Walks the segments of a tile range. `prefix[s]` = tiles before sequence s.
struct Walker {
    long long t, t1;
    int s;
    __device__ __forceinline__ bool next(const int* prefix, const int* ctxs, int ts, int member, Seg& sg) {
        if (t >= t1) return false;
        while (prefix[s + 1] <= t) ++s;
        const int nblk = (ctxs[s] + PBS - 1) / PBS;
        const long long off = t - prefix[s];
        sg.s = s;
        sg.gg = (int)(off / nblk);
        sg.g = sg.gg * ts + member;
        sg.j0 = (int)(off - (long long)sg.gg * nblk);
        const long long rem = t1 - t;
        sg.j1 = (int)((long long)(nblk - sg.j0) < rem ? nblk : sg.j0 + rem);
        sg.nblk = nblk;
        sg.ctx = ctxs[s];
        sg.t_begin = t;
        t += sg.j1 - sg.j0;
        return true;
    }
};

__device__ __forceinline__ long long range_begin(long long c, long long T, long long n) { return c * T / n; }
// the CTA whose range holds tile t
__device__ __forceinline__ int cta_of(long long t, long long T, long long n) { return (int)(((t + 1) * n - 1) / T); }

// Adds one arrival to an item's counter for this call's epoch; returns the count.
__device__ unsigned epoch_arrive(unsigned long long* ctr, unsigned long long epoch, int* err) {
    unsigned long long old = atomicAdd(ctr, 0ull);
    for (int it = 0; it < (1 << 20); ++it) {
        const unsigned long long nw = ((old >> 24) == epoch) ? old + 1 : ((epoch << 24) | 1ull);
        const unsigned long long prev = atomicCAS(ctr, old, nw);
        if (prev == old) return (unsigned)(nw & kCountMask);
        old = prev;
    }
    flag_error(err, PKV_ERR_DEVICE_TIMEOUT);
    return 0;
}

template <typename T, int D, int PATH, int HPW, int STAGES>
__global__ void __launch_bounds__(NTHREADS, kPersistCtasPerSm)
paged_decode_persistent_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const Params p) {
    using K = PKern<T, D, PATH, HPW, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* qbuf = smem + K::OFF_Q;
    float* red_o = reinterpret_cast<float*>(smem + K::OFF_RED);
    float* red_m = red_o + K::NSLOT * K::MAXG * D;
    float* red_l = red_m + K::NSLOT * K::MAXG;
    int* prefix = reinterpret_cast<int*>(smem + K::OFF_PREFIX);
    int* ctxs = reinterpret_cast<int*>(smem + K::OFF_CTX);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* qfull = empty + STAGES;
    uint64_t* qempty = qfull + kQStages;
    __shared__ volatile int s_abort;
    __shared__ int s_last;
    __shared__ int s_warp_sum[NCW + 1];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.num_seqs, hkv = p.num_kv_heads, group = p.group, hq = p.num_q_heads;
    const int c = blockIdx.x;
    const int ts = p.team_size, team = c / ts, member = c % ts, upr = hkv / ts;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], PATH == 1 ? NCW : 1);
        }
        for (int i = 0; i < kQStages; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
        }
        s_abort = 0;
        fence_barrier_init();
    }

    // ---- schedule: clamp lengths, tiles per sequence, exclusive prefix sum ----
    {
        const int per = (B + NTHREADS - 1) / NTHREADS;
        const int s_lo = min(B, threadIdx.x * per), s_hi = min(B, s_lo + per);
        int sum = 0;
        for (int s = s_lo; s < s_hi; ++s) {
            int ctx = p.context_lens[s];
            if (ctx < 0 || ctx > p.ctx_cap) {
                flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                ctx = ctx < 0 ? 0 : p.ctx_cap;
            }
            ctxs[s] = ctx;
            sum += ((ctx + PBS - 1) / PBS) * upr;
            if (ctx == 0 && (s % gridDim.x) == c) {             // empty context: zero output
                for (int i = 0; i < hq * D; ++i) store_out(p, (int64_t)s * hq * D + i, 0.f);
            }
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) s_warp_sum[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w) base += s_warp_sum[w];
        int run = base + incl - sum;                             // exclusive prefix of this thread
        for (int s = s_lo; s < s_hi; ++s) {
            prefix[s] = run;
            run += ((ctxs[s] + PBS - 1) / PBS) * upr;
        }
        if (threadIdx.x == NTHREADS - 1) prefix[B] = run;
        __syncthreads();
    }
    const long long ntiles = prefix[B];                       // units
    const long long nteams = gridDim.x / ts;
    const long long n_eff = ntiles < nteams ? ntiles : nteams;
    if ((long long)team >= n_eff) return;                      // uniform: nothing to do
    const long long t0 = range_begin(team, ntiles, n_eff), t1 = range_begin(team + 1, ntiles, n_eff);

    if (warp == 0) {
        // ================= producer =================
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
        const uint64_t pol = l2_policy_evict_first();
        Walker wk{t0, t1, 0};
        Seg sg;
        long long i = 0;   // tile index within this CTA's range
        int k = 0;         // segment index
        const uint32_t qbytes = (uint32_t)(group * D * sizeof(T));
        while (wk.next(prefix, ctxs, ts, member, sg)) {
            if (lane == 0 && !s_abort) {
                const int qs = k % kQStages;
                if (!mbar_wait_bounded(&qempty[qs], ((k / kQStages) & 1) ^ 1, p.err, p.wait_ns)) {
                    s_abort = 1;
                } else {
                    mbar_arrive_expect_tx(&qfull[qs], qbytes);
                    bulk_load_1d(qbuf + qs * K::QBYTES,
                                 static_cast<const T*>(p.q) + ((int64_t)sg.s * hq + (int64_t)sg.g * group) * D, qbytes,
                                 &qfull[qs]);
                }
            }
            const int32_t* bt = p.block_tables + (int64_t)sg.s * p.max_blocks;
            for (int j0 = sg.j0; j0 < sg.j1; j0 += 32) {
                int id = 0;
                if (j0 + lane < sg.j1) {
                    id = __ldg(bt + j0 + lane);
                    if (id < 0 || id >= p.num_blocks) {
                        flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                        id = p.num_blocks;                      // read as zeros by TMA
                    }
                }
                const int jn = min(32, sg.j1 - j0);
                for (int jj = 0; jj < jn; ++jj, ++i) {
                    const int pb = __shfl_sync(0xffffffffu, id, jj);
                    if (lane == 0 && !s_abort) {
                        const int st = (int)(i % STAGES);
                        if (!mbar_wait_bounded(&empty[st], (uint32_t)((i / STAGES) & 1) ^ 1u, p.err, p.wait_ns)) {
                            s_abort = 1;
                        } else {
                            mbar_arrive_expect_tx(&full[st], K::STAGE_BYTES);
                            uint8_t* dst = ring + st * K::STAGE_BYTES;
                            if constexpr (K::kMma) {
#pragma unroll
                                for (int h = 0; h < D / 64; ++h) {
                                    tma_load_4d(dst + h * (PBS * 128), &tm_k, &full[st], h * 64, sg.g, 0, pb, pol);
                                    tma_load_4d(dst + K::TILE + h * (PBS * 128), &tm_v, &full[st], h * 64, sg.g, 0, pb,
                                                pol);
                                }
                            } else {
                                tma_load_4d(dst, &tm_k, &full[st], 0, sg.g, 0, pb, pol);
                                tma_load_4d(dst + K::TILE, &tm_v, &full[st], 0, sg.g, 0, pb, pol);
                            }
                        }
                    }
                }
            }
            ++k;
        }
        if (lane == 0 && s_abort) {
            // drain: the last STAGES tile loads and kQStages query loads may still be landing
            for (long long j = (i > STAGES ? i - STAGES : 0); j < i; ++j)
                mbar_wait_bounded(&full[j % STAGES], (uint32_t)((j / STAGES) & 1), p.err, 100000000ull);
            for (int j = (k > kQStages ? k - kQStages : 0); j < k; ++j)
                mbar_wait_bounded(&qfull[j % kQStages], (uint32_t)((j / kQStages) & 1), p.err, 100000000ull);
        }
    } else {
        // ================= consumers =================
        const int cw = warp - 1, ct = threadIdx.x - 32;
        Walker wk{t0, t1, 0};
        Seg sg;
        long long i = 0;
        int k = 0;
        while (wk.next(prefix, ctxs, ts, member, sg)) {
            const int qs = k % kQStages;
            const long long iend = i + (sg.j1 - sg.j0);
            bool ok = !s_abort && mbar_wait_bounded(&qfull[qs], (uint32_t)((k / kQStages) & 1), p.err, p.wait_ns);
            if (__any_sync(0xffffffffu, !ok)) { s_abort = 1; ok = false; }
            const T* qrows = reinterpret_cast<const T*>(qbuf + qs * K::QBYTES);
            const int slot = PATH == 1 ? 0 : cw;
            if constexpr (PATH == 2) {
                MmaConsumer<D> cons;
                cons.init(reinterpret_cast<const __nv_bfloat16*>(qrows), group, lane);
                const long long first = i + ((cw - (int)(i % NCW)) + NCW) % NCW;
                for (long long ii = first; ii < iend && ok; ii += NCW) {
                    const int st = (int)(ii % STAGES);
                    const bool got = !s_abort && mbar_wait_bounded(&full[st], (uint32_t)((ii / STAGES) & 1), p.err, p.wait_ns);
                    if (__any_sync(0xffffffffu, !got)) { s_abort = 1; ok = false; break; }
                    uint8_t* stage = ring + st * K::STAGE_BYTES;
                    const int j = sg.j0 + (int)(ii - i);
                    const int nvalid = min(PBS, sg.ctx - j * PBS);
                    cons.consume(smem_u32(stage), smem_u32(stage + K::TILE), stage + K::TILE, nvalid, p.scale_log2,
                                 lane);
                    if (nvalid < PBS) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[st]);
                }
                cons.finish(red_o + slot * K::MAXG * D, red_m + slot * K::MAXG, red_l + slot * K::MAXG, group, lane);
            } else {
                const int hbase = PATH == 1 ? cw * HPW : 0;
                SimtConsumer<T, D, HPW> cons;
                cons.init(qrows + (int64_t)hbase * D, p.scale_log2, lane);
                const long long first = PATH == 1 ? i : i + ((cw - (int)(i % NCW)) + NCW) % NCW;
                const int step = PATH == 1 ? 1 : NCW;
                for (long long ii = first; ii < iend && ok; ii += step) {
                    const int st = (int)(ii % STAGES);
                    const bool got = !s_abort && mbar_wait_bounded(&full[st], (uint32_t)((ii / STAGES) & 1), p.err, p.wait_ns);
                    if (__any_sync(0xffffffffu, !got)) { s_abort = 1; ok = false; break; }
                    const uint8_t* stage = ring + st * K::STAGE_BYTES;
                    const int j = sg.j0 + (int)(ii - i);
                    cons.consume(stage, stage + K::TILE, min(PBS, sg.ctx - j * PBS), lane);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[st]);
                }
                cons.finish(red_o + (slot * K::MAXG + hbase) * D, red_m + slot * K::MAXG + hbase,
                            red_l + slot * K::MAXG + hbase, lane);
            }
            consumers_barrier();                                  // (A) states in shared memory
            if (ct == 0) mbar_arrive(&qempty[qs]);               // every warp has its query in registers

            // ---- segment epilogue (all consumer threads) ----
            const bool whole = sg.j0 == 0 && sg.j1 == sg.nblk;
            const int64_t qh0 = (int64_t)sg.s * hq + (int64_t)sg.g * group;
            const long long item0 = prefix[sg.s] + (long long)sg.gg * sg.nblk;
            const int c_first = cta_of(item0, ntiles, n_eff), c_last = cta_of(item0 + sg.nblk - 1, ntiles, n_eff);
            const int my_slot = 2 * c + (sg.t_begin == t0 ? 0 : 1);
            const int pstride = group * (D + 2);
            float* piece = p.ws_part + (int64_t)my_slot * pstride;
            if (!s_abort) {
                for (int idx = ct; idx < group * D; idx += NCW * 32) {
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
                    if (whole) {
                        store_out(p, (qh0 + h) * D + d, val);
                    } else {
                        piece[h * D + d] = val;
                        if (d == 0) {
                            piece[group * D + 2 * h] = M;
                            piece[group * D + 2 * h + 1] = L;
                        }
                    }
                }
            }
            if (!whole) {
                __threadfence();
                consumers_barrier();                              // (B) piece written and fenced
                if (ct == 0) {
                    const unsigned pieces = (unsigned)(c_last - c_first + 1);
                    s_last = !s_abort &&
                             epoch_arrive(p.counters + (int64_t)sg.s * hkv + sg.g, p.epoch, p.err) == pieces;
                }
                consumers_barrier();                              // (C) s_last visible
                if (s_last) {
                    __threadfence();
                    const int npieces = c_last - c_first + 1;
                    float* wbuf = red_o;                          // the warp states are merged already
                    constexpr int kCap = K::NSLOT * K::MAXG * (D + 2);
                    if ((npieces + 1) * group * 2 <= kCap) {
                        // (m, l) of every piece once, then weights w = l 2^(m - M) per head
                        for (int idx = ct; idx < npieces * group; idx += NCW * 32) {
                            const int pc = idx / group, h = idx - pc * group;
                            const int tt = c_first + pc;
                            const int sl = 2 * (tt * ts + member) + (range_begin(tt, ntiles, n_eff) >= item0 ? 0 : 1);
                            const float* pp = p.ws_part + (int64_t)sl * pstride + group * D + 2 * h;
                            wbuf[2 * idx] = ld_cg(pp);
                            wbuf[2 * idx + 1] = ld_cg(pp + 1);
                        }
                        consumers_barrier();
                        float* lsum = wbuf + 2 * npieces * group;
                        if (ct < group) {
                            float M = kNegInf;
                            for (int pc = 0; pc < npieces; ++pc) M = fmaxf(M, wbuf[2 * (pc * group + ct)]);
                            float L = 0.f;
                            for (int pc = 0; pc < npieces; ++pc) {
                                const float mc = wbuf[2 * (pc * group + ct)];
                                const float w = (M == kNegInf || mc == kNegInf)
                                                    ? 0.f : wbuf[2 * (pc * group + ct) + 1] * fast_exp2(mc - M);
                                wbuf[2 * (pc * group + ct)] = w;
                                L += w;
                            }
                            lsum[ct] = L;
                        }
                        consumers_barrier();
                        for (int idx = ct; idx < group * D; idx += NCW * 32) {
                            const int h = idx / D, d = idx - h * D;
                            float O = 0.f;
                            int pc = 0;
                            for (; pc + 4 <= npieces; pc += 4) {            // independent loads in flight
                                float v[4], w[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int tt = c_first + pc + u;
                                    const int sl = 2 * (tt * ts + member) +
                                                   (range_begin(tt, ntiles, n_eff) >= item0 ? 0 : 1);
                                    v[u] = ld_cg(p.ws_part + (int64_t)sl * pstride + h * D + d);
                                    w[u] = wbuf[2 * ((pc + u) * group + h)];
                                }
#pragma unroll
                                for (int u = 0; u < 4; ++u) O += w[u] * v[u];
                            }
                            for (; pc < npieces; ++pc) {
                                const int tt = c_first + pc;
                                const int sl = 2 * (tt * ts + member) + (range_begin(tt, ntiles, n_eff) >= item0 ? 0 : 1);
                                O += wbuf[2 * (pc * group + h)] * ld_cg(p.ws_part + (int64_t)sl * pstride + h * D + d);
                            }
                            const float L = lsum[h];
                            store_out(p, (qh0 + h) * D + d, L > 0.f ? O / L : 0.f);
                        }
                    } else {
                        // too many pieces to stage: read (m, l) straight from the workspace
                        for (int idx = ct; idx < group * D; idx += NCW * 32) {
                            const int h = idx / D, d = idx - h * D;
                            float M = kNegInf;
                            for (int tt = c_first; tt <= c_last; ++tt) {
                                const int sl = 2 * (tt * ts + member) + (range_begin(tt, ntiles, n_eff) >= item0 ? 0 : 1);
                                M = fmaxf(M, ld_cg(p.ws_part + (int64_t)sl * pstride + group * D + 2 * h));
                            }
                            float L = 0.f, O = 0.f;
                            if (M != kNegInf) {
                                for (int tt = c_first; tt <= c_last; ++tt) {
                                    const int sl =
                                        2 * (tt * ts + member) + (range_begin(tt, ntiles, n_eff) >= item0 ? 0 : 1);
                                    const float* pp = p.ws_part + (int64_t)sl * pstride;
                                    const float mc = ld_cg(pp + group * D + 2 * h);
                                    if (mc == kNegInf) continue;
                                    const float w = ld_cg(pp + group * D + 2 * h + 1) * fast_exp2(mc - M);
                                    L += w;
                                    O += w * ld_cg(pp + h * D + d);
                                }
                            }
                            store_out(p, (qh0 + h) * D + d, L > 0.f ? O / L : 0.f);
                        }
                    }
                    if (ct == 0) atomicExch(p.counters + (int64_t)sg.s * hkv + sg.g, p.epoch << 24);
                }
            }
            consumers_barrier();                                  // (D) shared states may be overwritten
            i = iend;
            ++k;
        }
    }
}

template <typename T, int D, int PATH, int HPW, int STAGES>
cudaError_t launch_persistent_t(const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, int grid,
                                cudaStream_t stream) {
    using K = PKern<T, D, PATH, HPW, STAGES>;
    auto kern = paged_decode_persistent_kernel<T, D, PATH, HPW, STAGES>;
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

template <typename T, int D>
constexpr int persistent_stages() {
    constexpr int sb = 2 * PBS * D * (int)sizeof(T);
    constexpr int n = 65536 / sb;
    return n < 4 ? 4 : (n > 16 ? 16 : n);
}

template <typename T, int D>
cudaError_t persistent_simt(int group, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, int grid,
                            cudaStream_t st) {
    constexpr int S = persistent_stages<T, D>();
    switch (group) {
        case 1: return launch_persistent_t<T, D, 0, 1, S>(mk, mv, p, grid, st);
        case 2: return launch_persistent_t<T, D, 0, 2, S>(mk, mv, p, grid, st);
        case 4: return launch_persistent_t<T, D, 1, 1, S>(mk, mv, p, grid, st);
        case 8: return launch_persistent_t<T, D, 1, 2, S>(mk, mv, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_persistent(bool bf16, bool use_mma, int head_dim, int group, const CUtensorMap& mk,
                              const CUtensorMap& mv, const Params& p, int grid, cudaStream_t st) {
    if (use_mma) {
        return head_dim == 128
                   ? launch_persistent_t<__nv_bfloat16, 128, 2, 8, persistent_stages<__nv_bfloat16, 128>()>(mk, mv, p,
                                                                                                         grid, st)
                   : launch_persistent_t<__nv_bfloat16, 64, 2, 8, persistent_stages<__nv_bfloat16, 64>()>(mk, mv, p,
                                                                                                       grid, st);
    }
    if (bf16)
        return head_dim == 128 ? persistent_simt<__nv_bfloat16, 128>(group, mk, mv, p, grid, st)
                               : persistent_simt<__nv_bfloat16, 64>(group, mk, mv, p, grid, st);
    return head_dim == 128 ? persistent_simt<float, 128>(group, mk, mv, p, grid, st)
                           : persistent_simt<float, 64>(group, mk, mv, p, grid, st);
}

int persistent_ctas_per_sm() { return kPersistCtasPerSm; }
int persistent_max_seqs() { return kMaxSeqsPersistent; }

}  // namespace attn
}  // namespace pkv
