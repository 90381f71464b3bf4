// Longest-first unit list of the partitioned decode kernel, built by one CTA
// of kPlanThreads threads (plan_units_kernel in paged_attention.cu; the
// shared-prefix cascade's plan kernel in paged_attention_mq.cu).
//
// A grid sized for the longest context leaves most rows without work when
// lengths are mixed, and CTAs taken in grid order start long partitions late:
// measured with per-CTA timestamps, a 7B-shaped batch streamed ~7.5 TB/s while
// all 444 CTA slots were busy, then spent its last 35 of 210 us finishing late
// long sequences, and the long-context grid had 5528 empty CTAs among 872 with
// work. The list holds the live (sequence, partition) units: every full
// partition first, then each sequence's last partition by decreasing size (a
// sequence of length 0 last: its CTA writes the zero output). Row y of the
// partition grid takes unit y; rows past the list exit at the end of dispatch.
#pragma once

#include "attention_common.cuh"

namespace pkv {
namespace attn {

constexpr int kPlanThreads = 256;

// Exclusive scan of one value per thread over the CTA; *total gets the sum.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = lane < kPlanThreads / 32 ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += t;
        }
        if (lane < kPlanThreads / 32) s_warp[lane] = wi - w;
        if (lane == 31) s_warp[kPlanThreads / 32] = wi;
    }
    __syncthreads();
    const int r = s_warp[wid] + incl - v;
    *total = s_warp[kPlanThreads / 32];
    __syncthreads();                                            // s_warp is reused by the next scan
    return r;
}

// units[] gets {seq << 16 | partition, length} for every live unit and
// *unit_count their number. len(s, first) is sequence s's length, clamped to
// the call's cap; `first` is true on the one call per sequence that may flag a
// length outside the cap (the second pass re-reads lengths only when the batch
// has more sequences than threads).
template <class Len>
__device__ void list_units(Len len, int B, int pb, int bsz, uint2* units, int* unit_count) {
    __shared__ int hist[kPlanMaxBins];                          // tails per size (blocks), then their offsets
    __shared__ int s_warp[kPlanThreads / 32 + 1];
    __shared__ int s_first[kPlanThreads];                       // a pass's first full unit per sequence
    __shared__ int s_ctx[kPlanThreads];
    const int tid = threadIdx.x;
    for (int b = tid; b < pb; b += kPlanThreads) hist[b] = 0;
    __syncthreads();
    // full partitions, listed sequence-major; the tails counted by size
    int nfull = 0;
    int ctx_keep = 0;                                           // this thread's length when B fits one pass
    for (int s0 = 0; s0 < B; s0 += kPlanThreads) {
        const int sq = s0 + tid;
        int full = 0, ctx = 0;
        if (sq < B) {
            ctx = len(sq, true);
            const int nb = (ctx + bsz - 1) / bsz;
            full = nb / pb;
            if (nb % pb != 0 || nb == 0) atomicAdd(&hist[nb % pb], 1);
        }
        ctx_keep = ctx;
        int chunk = 0;
        const int off = cta_exclusive_scan(full, s_warp, &chunk);
        s_first[tid] = off;
        s_ctx[tid] = ctx;
        __syncthreads();
        // the pass's full units, spread over the threads: unit u belongs to the
        // last sequence whose first unit is <= u (binary search)
        for (int u = tid; u < chunk; u += kPlanThreads) {
            int lo = 0, hi = kPlanThreads - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_first[mid] <= u) lo = mid; else hi = mid - 1;
            }
            units[nfull + u] = make_uint2(((unsigned)(s0 + lo) << 16) | (unsigned)(u - s_first[lo]), (unsigned)s_ctx[lo]);
        }
        nfull += chunk;
        __syncthreads();                                        // s_first / s_ctx are reused by the next pass
    }
    // tail offsets in decreasing size: offset(size b) = tails longer than b
    int ntail = 0;
    for (int b0 = 0; b0 < pb; b0 += kPlanThreads) {
        const int b = pb - 1 - (b0 + tid);                        // sizes from the largest down
        const int h = b >= 0 ? hist[b] : 0;
        int chunk = 0;
        const int off = ntail + cta_exclusive_scan(h, s_warp, &chunk);
        if (b >= 0) hist[b] = nfull + off;
        ntail += chunk;
        __syncthreads();
    }
    // the tails, each at the next free place of its size
    for (int s0 = 0; s0 < B; s0 += kPlanThreads) {
        const int sq = s0 + tid;
        if (sq < B) {
            const int ctx = B > kPlanThreads ? len(sq, false) : ctx_keep;
            const int nb = (ctx + bsz - 1) / bsz;
            if (nb % pb != 0 || nb == 0) {
                const int at = atomicAdd(&hist[nb % pb], 1);
                units[at] = make_uint2(((unsigned)sq << 16) | (unsigned)(nb / pb), (unsigned)ctx);
            }
        }
    }
    if (tid == 0) *unit_count = nfull + ntail;
}

}  // namespace attn
}  // namespace pkv
