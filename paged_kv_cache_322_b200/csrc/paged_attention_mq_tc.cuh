// Multi-query paged attention on the 5th-generation tensor cores (tcgen05) for
// prefill-sized query tiles: bf16 caches, head_dim 128, 128 query rows per CTA.
// Included by paged_attention_mq.cu, which routes a call here from 32 query rows
// (query tokens x group) per KV head on; shorter tiles are padded with idle rows.
//
//   S  = Q K^T   M = 128 query rows, N = 128 KV tokens, K = 128 dims  (TMEM, fp32)
//   O += P V     M = 128 rows, N = 128 dims, K = 128 tokens            (TMEM, fp32)
//
// Roles (352 threads): warp 0 loads Q once and streams K tiles, warp 10 streams
// V tiles (TMA, 128-byte swizzle, three-stage K and V rings); warp 1 owns the TMEM allocation and one of its threads
// issues every tcgen05.mma; warps 2-9 run the softmax, two threads per query row
// (its TMEM lane). Each of the two runs an online softmax of its own over one
// half of every tile's tokens (0-63 or 64-127) with its own O accumulator, so
// the two never wait for each other inside the loop; they combine their (m, l)
// and O once, at the end (exchanging the row maximum every tile instead cost
// each tile's softmax ~640 cycles of waiting, clock64 stamps). The S accumulator
// is double-buffered, so S of tile t+1 is computed while the softmax of tile t
// runs. P stays in TMEM, written over its own S buffer, as two bf16 parts (high,
// and the rounding residue) that both multiply V (the A operand read from TMEM),
// so the probabilities keep ~16 bits, P is double-buffered with S, and shared
// memory holds only Q and three-stage K and V rings. The online
// softmax rescales O in TMEM only when a row's running maximum grows by more
// than 2^8 over the reference it uses (p <= 2^8 stays exact enough in bf16 and
// fp32), so most tiles skip the O round trip.
#pragma once

namespace pkv {
namespace attn {
namespace tc {

constexpr int ROWS = 128;          // query rows per CTA (UMMA M)
constexpr int TOK = 128;           // KV tokens per tile
constexpr int D = 128;
constexpr int THREADS = 352;      // warps 0 / 10 K / V loads, warp 1 MMA, warps 2-9 softmax (two per row)
constexpr int HALF = 128 * 128;    // one 64-element-wide half of a 128-row operand, bytes
constexpr int NST = 3;             // K ring and V ring depth
constexpr int Q_OFF = 0;
constexpr int K_OFF = 2 * HALF;                   // NST stages of K (2 halves each)
constexpr int V_OFF = K_OFF + NST * 2 * HALF;     // NST stages of V
constexpr int BAR_OFF = V_OFF + NST * 2 * HALF;
constexpr int NBAR = 23;
constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8 + 16;
constexpr int TMEM_COLS = 512;     // S/P 0 [0,128) S/P 1 [128,256) O of token half 0 [256,384), of half 1 [384,512)
constexpr int T_O = 256;           // O of token half h at T_O + 128 h
// P of tile t is written over S of tile t (high part in the buffer's first 64
// columns, low part in the next 64): the buffer is free once S is read, and
// S of tile t + 2 is issued after the PV product that reads P of tile t.
static_assert(SMEM <= 232448, "shared memory per CTA");

// Barrier indices. P-ready is one barrier per tile parity: S of tile t + 1 is
// issued before the MMA thread waits for P of tile t, so the softmax may finish
// tiles t and t + 1 before that wait; on a single barrier that would put the
// phase two ahead of the waiter, where a parity wait cannot tell it apart.
// Tile t + 2 cannot arrive before that wait (its S is issued after PV of t).
// The final (m, l) exchange of a row's two threads has one barrier per TMEM
// lane quarter (64 arrivals: the two warps that share those rows).
enum {
    B_Q = 0, B_KFULL = 1, B_KEMPTY = 4, B_VFULL = 7, B_VEMPTY = 10, B_SFULL = 13, B_FIN = 15,
    B_PREADY = 19, B_ODONE = 21, B_DRAIN = 22
};

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;                              // descriptor version of sm_100
    d |= 2ull << 61;                              // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, A K-major, B K- or MN-major.
constexpr uint32_t idesc_bf16(int m, int n, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// A operand from TMEM (lane = row, two bf16 K-elements per 32-bit column).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
          "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
          "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// tm_q: q as [T, Hq, D] with box (64, G, 128 / G); tm_k / tm_v: the caches with
// box (64, 1, R, 1), R = min(block_size, 128) rows (one whole block per piece).
template <int BSZ>
__global__ void __launch_bounds__(THREADS, 1)
paged_mq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const MqParams p) {
    constexpr int R = BSZ < TOK ? BSZ : TOK;                    // rows of one TMA piece (a whole block)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BAR_OFF + NBAR * 8);
    __shared__ volatile int s_abort;

    const int kvh = blockIdx.x, part = blockIdx.y;
    const int seq = blockIdx.z / p.row_tiles, tile = blockIdx.z - seq * p.row_tiles;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    // launched as a programmatic dependent (the shared-prefix cascade), the CTAs
    // wait here for the grid that wrote the call's lengths; a no-op otherwise
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int q0, n, c;
    mq_sequence(p, seq, q0, n, c);
    const int row_begin = tile * ROWS;
    if (row_begin >= n * G) return;                             // no live rows (uniform over the CTA)
    const int last_tok = min(n - 1, (row_begin + ROWS - 1) / G);
    const int kv_end = p.causal ? c - n + last_tok + 1 : c;
    const int pt = p.part_blocks * BSZ;
    const int kv0 = part * pt;
    if (kv0 >= kv_end) return;
    const int ntok = min(pt, kv_end - kv0);
    const int ntiles = (ntok + TOK - 1) / TOK;
    const int blk0 = part * p.part_blocks;
    const bool direct = p.slot < 0 && (c + pt - 1) / pt <= 1;
    const int opart = p.slot >= 0 ? p.slot + part : part;        // the partial's index in the workspace

    if (threadIdx.x == 0) {
        mbar_init(&bar[B_Q], 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bar[B_KFULL + s], 1);
            mbar_init(&bar[B_KEMPTY + s], 1);
            mbar_init(&bar[B_VFULL + s], 1);
            mbar_init(&bar[B_VEMPTY + s], 1);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&bar[B_SFULL + s], 1);
        for (int q = 0; q < 4; ++q) mbar_init(&bar[B_FIN + q], 64);
        for (int s = 0; s < 2; ++s) mbar_init(&bar[B_PREADY + s], 256);
        mbar_init(&bar[B_ODONE], 1);
        mbar_init(&bar[B_DRAIN], 1);
        s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {                                            // TMEM: S0, S1, O, P high, P low
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 10) {
        // ---------------- producers: Q once, then the K stream (warp 0) and the V stream (warp 10) ----------------
        // One warp per stream: K of a tile is released as soon as S is computed,
        // V only after the PV product, so a V stage that frees late does not hold
        // back the next K tile (two half-warps of one warp could not do this:
        // their spin loops progressed in lockstep, clock64 stamps showed). Block
        // ids come 32 at a time, one batch ahead of use, and are checked when
        // used: loading and checking each tile's ids just before its copies put a
        // dependent global load (~2,700 cycles) on every tile's critical path.
        // Lane b issues piece b of a tile.
        const int kv = warp == 10;                              // stream: 0 K, 1 V
        bool ok = true;
        int issued = 0;                                         // tiles whose copies this stream issued
        // test hook: the first CTA never issues this tile's K copies (nor arrives
        // on their barrier), so the MMA thread's bounded wait for them runs out
        const int withheld = (blockIdx.x | blockIdx.y | blockIdx.z) == 0 ? p.withhold : -1;
        if (warp == 0 && lane == 0) {
            mbar_arrive_expect_tx(&bar[B_Q], 2 * HALF);
            for (int h = 0; h < 2; ++h)
                tma_load_3d(smem + Q_OFF + h * HALF, &tm_q, &bar[B_Q], h * 64, kvh * G, q0 + row_begin / G);
        }
        const uint64_t pol = l2_policy_evict_normal();
        const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks + blk0;
        constexpr int PPT = TOK / R;                            // pieces (blocks) per tile, divides 32
        static_assert(PPT <= 32 && 32 % PPT == 0, "a tile's block ids sit in one batch of 32");
        const int nblk = (ntok + BSZ - 1) / BSZ;                // blocks of this CTA's KV range
        auto load_batch = [&](int b) { return 32 * b + lane < nblk ? __ldg(bt + 32 * b + lane) : 0; };
        int batch = 0;
        int ids = load_batch(0), ids_next = load_batch(1);
        uint8_t* const ring = smem + (kv ? V_OFF : K_OFF);
        const CUtensorMap* map = kv ? &tm_v : &tm_k;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % NST;
            const int np = (min(TOK, ntok - t * TOK) + R - 1) / R;
            const int j0 = t * PPT;                             // first block of the tile
            if (j0 / 32 != batch) {
                batch = j0 / 32;
                ids = ids_next;
                ids_next = load_batch(batch + 1);
            }
            int id = __shfl_sync(0xffffffffu, ids, (j0 & 31) + (lane < PPT ? lane : 0));
            if (lane < np && (id < 0 || id >= p.num_blocks)) {
                flag_error(p.err, PKV_ERR_DEVICE_BOUNDS);
                id = p.num_blocks;                              // zero-filled tile
            }
            uint64_t* full = &bar[(kv ? B_VFULL : B_KFULL) + s];
            const bool skip = kv == 0 && t == withheld;
            if (lane == 0) {
                ok = mbar_wait_bounded(&bar[(kv ? B_VEMPTY : B_KEMPTY) + s], ((t / NST) & 1) ^ 1, p.err, p.wait_ns);
                if (ok) {
                    if (!skip) mbar_arrive_expect_tx(full, np * 2 * R * 128);
                    issued = t + 1;
                } else {
                    s_abort = 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;    // also orders the expect-tx before the copies
            if (!ok) break;
            if (lane < np && !skip) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(ring + s * 2 * HALF + h * HALF + lane * R * 128, map, full, h * 64, kvh, 0, id, pol);
            }
        }
        if (lane == 0) {
            // every copy this stream issued has landed before the CTA moves on (on
            // the normal path the MMA thread waited for each of them already; after
            // an abort some may still be in flight)
            for (int t = max(0, issued - NST); t < issued; ++t)
                if (kv != 0 || t != withheld)
                    mbar_wait_bounded(&bar[(kv ? B_VFULL : B_KFULL) + t % NST], (t / NST) & 1, p.err, p.wait_ns);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread) ----------------
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(ROWS, TOK, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(ROWS, D, true);
            // Descriptors of Q, and of K and V at ring stage 0, built once: a
            // descriptor's start-address field holds (address >> 4), so moving it by
            // d bytes adds d >> 4 (shared addresses stay below 256 KB, no carry).
            // Building two descriptors per MMA in the loop made one thread's MMA
            // issue about as slow as the MMAs themselves (clock64 stamps: ~90 cycles
            // per tcgen05.mma, 24 per tile).
            const uint64_t qd = desc_sw128(smem_u32(smem + Q_OFF), 16, 1024);
            const uint64_t kd = desc_sw128(smem_u32(smem + K_OFF), 16, 1024);
            const uint64_t vd = desc_sw128(smem_u32(smem + V_OFF), HALF, 1024);
            bool ok = mbar_wait_bounded(&bar[B_Q], 0, p.err, p.wait_ns);
            // PV of tile u: O_h += P_hi V + P_lo V over token half h (64 tokens, 4 k-steps of 16)
            auto pv = [&](int u) -> bool {
                if (!mbar_wait_bounded(&bar[B_PREADY + (u & 1)], (u >> 1) & 1, p.err, p.wait_ns)) return false;
                if (!mbar_wait_bounded(&bar[B_VFULL + u % NST], (u / NST) & 1, p.err, p.wait_ns)) return false;
                fence_after();
                const uint64_t vs = vd + (uint64_t)(((u % NST) * 2 * HALF) >> 4);
                const uint32_t pa = tmem + (u & 1) * 128;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int part_lo = 0; part_lo < 2; ++part_lo)
#pragma unroll
                        for (int k = 0; k < TOK / 32; ++k)
                            // A = P: tokens 64 hf + 16 k .. in columns 32 hf + 8 k .. (+64: the low part);
                            // B = V: MN-major (dims contiguous), those tokens' rows; dim halves HALF apart
                            mma_ts(tmem + T_O + hf * 128, pa + part_lo * 64 + hf * 32 + k * 8,
                                   vs + (uint64_t)(((hf * 64 + k * 16) * 128) >> 4), IDESC_PV,
                                   (u > 0 || part_lo > 0 || k > 0) ? 1u : 0u);
                commit(&bar[B_ODONE]);
                commit(&bar[B_VEMPTY + u % NST]);
                return true;
            };
            for (int t = 0; t < ntiles && ok; ++t) {
                const int sb = t & 1, ks = t % NST;
                // S of tile t goes into the buffer of tile t - 2, whose P the PV product
                // issued in the previous iteration reads first (MMAs run in issue order)
                ok = mbar_wait_bounded(&bar[B_KFULL + ks], (t / NST) & 1, p.err, p.wait_ns);
                if (!ok) break;
                fence_after();
                const uint64_t ksd = kd + (uint64_t)((ks * 2 * HALF) >> 4);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint64_t off = (uint64_t)(((k >> 2) * HALF + (k & 3) * 32) >> 4);
                    mma_ss(tmem + sb * 128, qd + off, ksd + off, IDESC_S, k > 0 ? 1u : 0u);
                }
                commit(&bar[B_SFULL + sb]);
                commit(&bar[B_KEMPTY + ks]);
                if (t >= 1) ok = pv(t - 1);
            }
            if (ok && ntiles > 0) ok = pv(ntiles - 1);
            if (!ok) s_abort = 1;
            // every MMA issued has finished before TMEM is released
            commit(&bar[B_DRAIN]);
            mbar_wait_bounded(&bar[B_DRAIN], 0, p.err, p.wait_ns);
        }
    } else {
        // ---------------- softmax: two threads per query row ----------------
        // Warps 2-9: warp w reads TMEM lanes 32 (w % 4) .. (its rows) and column
        // half h = (w - 2) / 4 of every 128-wide S buffer (tokens 64 h .. 64 h + 63
        // of the tile), so two warps per SM sub-partition hide each other's
        // latencies. Each thread's (m, l) and O_h cover its half's tokens only.
        const int quarter = warp & 3;                           // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;                       // columns [64 half, 64 half + 64)
        const int lr = quarter * 32 + lane;                     // row of the tile = TMEM lane
        const int r = row_begin + lr;
        const int qi = r / G, hh = r - qi * G;
        const int pos = qi < n ? (p.causal ? c - n + qi : c - 1) : -1;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        constexpr int HC = TOK / 2;                             // columns per thread
        float m_ref = kNegInf, l = 0.f;                         // this half's running reference and sum
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t & 1;
            const bool got = mbar_wait_bounded(&bar[B_SFULL + s], (t >> 1) & 1, p.err, p.wait_ns);
            if (__any_sync(0xffffffffu, !got || s_abort != 0)) {
                ok = false;
                s_abort = 1;
                break;
            }
            fence_after();
            float x[HC];
#pragma unroll
            for (int ch = 0; ch < HC / 32; ++ch) tmem_ld32(lane_base + s * 128 + half * HC + ch * 32, x + ch * 32);
            tmem_wait_ld();
            // masks: past the partition's range, or after the row's position (causal)
            const int tok0 = kv0 + t * TOK + half * HC;
            const int lim = min(pos, kv0 + ntok - 1) - tok0;    // this half's columns 0..lim are visible
            // the maximum as four independent chains joined by a tree (one serial
            // chain over the 64 values was the softmax's critical path)
            float e4[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
            if (lim >= HC - 1) {
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    x[j] *= p.scale_log2;
                    e4[j & 3] = fmaxf(e4[j & 3], x[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    x[j] = j <= lim ? x[j] * p.scale_log2 : kNegInf;
                    e4[j & 3] = fmaxf(e4[j & 3], x[j]);
                }
            }
            const float mt = fmaxf(fmaxf(e4[0], e4[1]), fmaxf(e4[2], e4[3]));
            const float m_new = fmaxf(m_ref, mt);
            const bool grow = m_new > m_ref + 8.f;              // also true when m_ref is -inf and the row sees a token
            // V rows past the range (the unwritten tail of the last block, or a stage
            // row no piece filled) may hold anything, NaN included: P is 0 there, but
            // 0 * NaN would not be, so those rows are zeroed (this thread: its half of
            // the dims) before the PV product.
            const int tok_here = min(TOK, ntok - t * TOK);
            if (lr >= tok_here) {
                const bool vin = mbar_wait_bounded(&bar[B_VFULL + t % NST], (t / NST) & 1, p.err, p.wait_ns);
                if (vin) {
                    uint8_t* vrow = smem + V_OFF + (t % NST) * 2 * HALF + half * HALF + lr * 128;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) *reinterpret_cast<uint4*>(vrow + (cc << 4)) = make_uint4(0u, 0u, 0u, 0u);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
            }
            // P = 2^(x - ref) as bf16 high + low parts
            const float ref_new = grow ? m_new : m_ref;
            const float ref = ref_new == kNegInf ? 0.f : ref_new;
            uint32_t ph[HC / 2], pl[HC / 2];
            float ps4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < HC / 2; ++e) {
                const float p0 = fast_exp2(x[2 * e] - ref), p1 = fast_exp2(x[2 * e + 1] - ref);
                ps4[e & 3] += p0 + p1;
                ph[e] = pack_bf16(p0, p1);
                pl[e] = pack_bf16(p0 - bf16lo(ph[e]), p1 - bf16hi(ph[e]));
            }
            // O_h must be rescaled only when this half's maximum grew past its
            // reference; then the PV product of tile t - 1 has to be complete first.
            // S of this tile being complete already implies PV of tile t - 2 is (one
            // commit covers every earlier MMA), and PV of tile t needs this thread's
            // P, so O-done is at most one phase behind and its parity wait is exact.
            if (t > 0 && __any_sync(0xffffffffu, grow && m_ref != kNegInf)) {
                const bool done = mbar_wait_bounded(&bar[B_ODONE], (t - 1) & 1, p.err, p.wait_ns);
                if (__any_sync(0xffffffffu, !done || s_abort != 0)) {
                    ok = false;
                    s_abort = 1;
                    break;
                }
                fence_after();
                const float alpha = (grow && m_ref != kNegInf) ? fast_exp2(m_ref - m_new) : 1.f;
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    float o[32];
                    tmem_ld32(lane_base + T_O + half * 128 + ch * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(lane_base + T_O + half * 128 + ch * 32, o);
                }
            }
            if (grow) {
                l = m_ref == kNegInf ? 0.f : l * fast_exp2(m_ref - m_new);
                m_ref = m_new;
            }
            l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
            // this half's tokens: P high columns [32 half, +32), P low columns 64 + [32 half, +32)
            tmem_st32u(lane_base + s * 128 + half * 32, ph);
            tmem_st32u(lane_base + s * 128 + 64 + half * 32, pl);
            tmem_wait_st();
            fence_before();
            mbar_arrive(&bar[B_PREADY + s]);
        }
        // the last PV, then the two halves' (m, l) combined, then this thread's 64
        // dims of the row's output (or of the partition's partial) from O_0 and O_1
        if (ok && ntiles > 0) {
            // O-done may be two phases behind here, where a parity wait cannot tell
            // them apart: wait for the single-use drain barrier the MMA thread
            // commits after its last MMA instead
            const bool done = mbar_wait_bounded(&bar[B_DRAIN], 0, p.err, p.wait_ns);
            ok = !__any_sync(0xffffffffu, !done || s_abort != 0);
        }
        float m_oth = kNegInf, l_oth = 0.f;
        if (ok) {
            // every MMA is complete, so the S columns are free: (m, l) of half h in
            // columns 2 h, 2 h + 1 of this row's lane
            uint32_t v2[2] = {__float_as_uint(m_ref), __float_as_uint(l)};
            asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(lane_base + 2 * half),
                         "r"(v2[0]), "r"(v2[1])
                         : "memory");
            tmem_wait_st();
            fence_before();
            mbar_arrive(&bar[B_FIN + quarter]);
            const bool fin = mbar_wait_bounded(&bar[B_FIN + quarter], 0, p.err, p.wait_ns);
            ok = !__any_sync(0xffffffffu, !fin || s_abort != 0);
            if (ok) {
                fence_after();
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                             : "=r"(v2[0]), "=r"(v2[1])
                             : "r"(lane_base + 2 * (half ^ 1)));
                tmem_wait_ld();
                m_oth = __uint_as_float(v2[0]);
                l_oth = __uint_as_float(v2[1]);
            }
        }
        if (ok) {
            const float M = fmaxf(m_ref, m_oth);
            const float w_me = m_ref == kNegInf ? 0.f : fast_exp2(m_ref - M);
            const float w_oth = m_oth == kNegInf ? 0.f : fast_exp2(m_oth - M);
            const float L = l * w_me + l_oth * w_oth;
            const float inv = L > 0.f ? 1.f / L : 0.f;
            const float w0 = (half == 0 ? w_me : w_oth) * inv, w1 = (half == 0 ? w_oth : w_me) * inv;
            const bool live = qi < n;
            const int64_t qh = (int64_t)(q0 + (live ? qi : 0)) * p.num_q_heads + kvh * G + hh;
#pragma unroll
            for (int ch = 0; ch < HC / 32; ++ch) {
                float o[32], o1[32];
                const int d0 = half * HC + ch * 32;
                tmem_ld32(lane_base + T_O + d0, o);
                tmem_ld32(lane_base + T_O + 128 + d0, o1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = o[i] * w0 + o1[i] * w1;
                if (live) {
                    // the thread's 32 dims are contiguous: 16-byte stores
                    if (direct && !p.out_f32) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + qh * D + d0);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(pack_bf16(o[8 * v4], o[8 * v4 + 1]), pack_bf16(o[8 * v4 + 2], o[8 * v4 + 3]),
                                                 pack_bf16(o[8 * v4 + 4], o[8 * v4 + 5]),
                                                 pack_bf16(o[8 * v4 + 6], o[8 * v4 + 7]));
                    } else {
                        float* dst = direct ? static_cast<float*>(p.out) + qh * D + d0
                                            : p.ws_o + (qh * p.num_parts + opart) * D + d0;
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            reinterpret_cast<float4*>(dst)[v4] =
                                make_float4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
                    }
                }
            }
            if (live && !direct && half == 0) {
                p.ws_ml[(qh * p.num_parts + opart) * 2 + 0] = M;
                p.ws_ml[(qh * p.num_parts + opart) * 2 + 1] = L;
            }
        }
    }
    fence_before();
    __syncthreads();
    if (warp == 1) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

}  // namespace tc
}  // namespace attn
}  // namespace pkv
