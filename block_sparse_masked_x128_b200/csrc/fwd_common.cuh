// fwd_common.cuh -- the forward kernel's view of the unit schedule as the block mask lays it
// out, the warp-collective entry reader, and the TMA producer role (kept apart from the
// tensor-core and softmax roles in attn_fwd.cu, and written against a configuration class so
// another tiling can reuse it).
//
// A unit is the pair of query blocks (2p, 2p+1) of one (b, h) with the merged list of kv
// blocks either of them reads; each entry is a kv block index (bits 0-15) with the
// live/full flags of the two query tiles (kLive0, kFull0, kLive1, kFull1).  The producer
// loads both Q tiles of a unit, then K_j and V_j of every entry into a ring of shared-memory
// stages; a configuration class C supplies the tile size, the ring depth and the barrier
// slots (kBarQFull / kBarQEmpty at 0 / 1, C::kBarSlotFull and C::kBarSlotEmpty per stage,
// C::kBarUFull and C::kBarUEmpty per slot of the unit ring).
#pragma once

#include "fa_internal.h"
#include "fa_trace.cuh"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kProducerSleepNs = 256;         // the producer's pause between polls
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;         // log2 of the largest P allowed
constexpr int kBarQFull = 0;
constexpr int kBarQEmpty = 1;

struct Unit {
    int b, h, pair, E;
    int nl0, nl1;  // live tiles of query tile 0 and 1
    const int32_t* entries;
};

// Units are ranked per (b, h) by descending cost.  Interleaved order (the r-th longest unit of
// every (b, h), then the (r+1)-th ...) hands the longest units of the whole job out first;
// head-major order keeps the CTAs in flight on one or two (b, h) at a time, so their K and V
// stay in L2 when all heads' K and V together would not fit.
// With the global ranking (sched_gorder), unit rank r of every stored (b, h) is handed out
// for all the (b, h) that share that mask row (the broadcast copies) before rank r + 1; for a
// fully broadcast mask that is the interleaved order.
__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
    const int BH = p.B * p.H;
    int b, h;
    size_t sidx;
    Unit un;
    if (!p.head_major && p.sched_gorder) {
        const int mult = BH / (p.maskB * p.maskH);   // (b, h) per stored mask row
        const int rank = u / mult, k = u - rank * mult;
        const int g = __ldg(p.sched_gorder + rank);
        sidx = (size_t)(g / p.NP);
        un.pair = g - (int)sidx * p.NP;
        const int mb = (int)sidx / p.maskH, mh = (int)sidx - mb * p.maskH;
        if (p.maskB == 1 && p.maskH == 1) {
            b = k / p.H;
            h = k - b * p.H;
        } else if (p.maskB == 1) {
            b = k;
            h = mh;
        } else if (p.maskH == 1) {
            b = mb;
            h = k;
        } else {
            b = mb;
            h = mh;
        }
    } else {
        int r, bh;
        if (p.head_major) {
            bh = u / p.NP;
            r = u - bh * p.NP;
        } else {
            r = u / BH;
            bh = u - r * BH;
        }
        b = bh / p.H;
        h = bh - b * p.H;
        const int mb = (p.maskB == 1) ? 0 : b, mh = (p.maskH == 1) ? 0 : h;
        sidx = (size_t)mb * p.maskH + mh;
        un.pair = __ldg(p.sched_order + sidx * p.NP + r);
    }
    un.b = b;
    un.h = h;
    FA_DCHECK_INDEX(un.pair, p.NP, p.status);
    const int2 c = __ldg(reinterpret_cast<const int2*>(p.sched_count) + sidx * p.NP + un.pair);
    un.E = c.x;
    FA_DCHECK_INDEX(un.E, p.KVB + 1, p.status);
    un.nl0 = c.y & 0xFFFF;
    un.nl1 = (int)((unsigned)c.y >> 16);
    un.entries = p.sched_entries + (sidx * p.NP + un.pair) * (size_t)p.KVB;
    return un;
}

// Warp-collective reader of a unit's entry list: lane l caches entry base + l.
// Indices passed to get() must not decrease.
struct EntryReader {
    const int32_t* ptr;
    int E, base, val;
    __device__ __forceinline__ void init(const int32_t* p, int n) {
        ptr = p;
        E = n;
        base = -64;
        val = 0;
    }
    __device__ __forceinline__ int get(int e) {
        const int nb = e & ~31;
        if (nb != base) {
            base = nb;
            const int idx = nb + (int)(threadIdx.x & 31);
            val = idx < E ? __ldg(ptr + idx) : 0;
        }
        return __shfl_sync(kFullMask, val, e & 31);
    }
};

// Units are handed out at run time, longest first: the TMA warp of each CTA takes the next
// index from a global counter (atomicAdd on sched_ctr[0]) when it is ready for another unit
// and publishes it to the MMA and softmax warps through a two-slot ring in shared memory
// (C::kBarUFull / C::kBarUEmpty per slot; -1 ends the sequence).  A CTA that finishes early
// simply takes more units, so the per-CTA work evens out whatever the units really cost.
constexpr int kUnitRing = 2;

// Consumer side: the next unit of this CTA, -1 when there is none; ok turns false when the
// bounded wait gave up.  Called by every lane of a warp.
template <class C, class Params>
__device__ __forceinline__ int take_unit(const Params& p, uint32_t bars, const volatile int* ring,
                                         uint32_t& u_iter, volatile int* abort_flag, bool& ok) {
    const int slot = (int)(u_iter % kUnitRing);
    const uint32_t par = (u_iter / kUnitRing) & 1u;
    if (!mbar_wait_bounded(bars + 8u * (uint32_t)(C::kBarUFull + slot), par, abort_flag, p.status,
                           kWaitLimitNs)) {
        ok = false;
        return -1;
    }
    const int u = ring[slot];
    mbar_arrive_warp(bars + 8u * (uint32_t)(C::kBarUEmpty + slot));
    ++u_iter;
    return u;
}

// Wait without regard to the abort flag (used to drain in-flight copies on the way out).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) break;
    }
    __syncwarp();
}

// ------------------------------------------------------------------ producer (warp 0)

template <class C>
__device__ void producer_role(const FwdParams& p, const CUtensorMap* tmq, const CUtensorMap* tmk,
                              const CUtensorMap* tmv, uint32_t sbase, uint32_t bars,
                              volatile int* ring, volatile int* abort_flag) {
    const uint32_t sQ = sbase, sKV = sbase + 2 * C::kTileBytes;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    // The producer runs ahead of the MMA and softmax warps and mostly waits for a free stage;
    // it sleeps between polls, so it takes fewer issue slots from the softmax warps that share
    // its SM sub-partition (measured: +0.5 % at 8k and 32k, for 64 to 1024 ns alike).
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded_sleepy(bar(i), par, abort_flag, p.status, kWaitLimitNs, kProducerSleepNs);
    };
    const uint32_t leader = elect_one_lane();
    if (leader) {
        tma_prefetch_desc(tmq);
        tma_prefetch_desc(tmk);
        tma_prefetch_desc(tmv);
    }
    __syncwarp();
    const int leader_lane = __ffs(__ballot_sync(kFullMask, leader != 0)) - 1;
    // Done taking units: the last CTA to get here resets the counters for the next launch
    // (every CTA gets here, also after a timeout, because every wait is bounded).
    auto finish = [&]() {
        if (leader) {
            __threadfence();
            if (atomicAdd(p.sched_ctr + 1, 1) == (int)gridDim.x - 1) {
                p.sched_ctr[0] = 0;
                p.sched_ctr[1] = 0;
                __threadfence();
            }
        }
        __syncwarp();
    };
    uint32_t kv_pos = 0, q_iter = 0, u_iter = 0;
    bool ok = true;
    const bool stall = p.stall_loads != 0;
    FA_TRACE_DECL
    for (;;) {
        int u = -1;
        if (leader) {
            const int v = atomicAdd(p.sched_ctr, 1);
            u = v < p.n_units ? v : -1;
        }
        u = __shfl_sync(kFullMask, u, leader_lane);
        {   // publish it to the MMA and softmax warps
            const int slot = (int)(u_iter % kUnitRing);
            if (!wait(C::kBarUEmpty + slot, ((u_iter / kUnitRing) & 1u) ^ 1u)) { ok = false; break; }
            if (leader) {
                ring[slot] = u;
                mbar_arrive(bar(C::kBarUFull + slot));
            }
            __syncwarp();
            ++u_iter;
        }
        if (u < 0) break;
        const Unit un = decode_unit(p, u);
        if (un.E == 0) continue;
        FA_TRACE_EV(0, 40);
        if (!wait(kBarQEmpty, (q_iter & 1u) ^ 1u)) { ok = false; break; }
        const int q0 = 2 * un.pair;
        const int nq = (q0 + 1 < p.QB) ? 2 : 1;
        mbar_arrive_expect_tx_if(leader, bar(kBarQFull), (uint32_t)(nq * C::kTileBytes));
        for (int t = 0; t < nq; ++t)
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_4d_if(leader, sQ + t * C::kTileBytes + c * 16384, tmq, bar(kBarQFull),
                               c * 64, (q0 + t) * kBlock, un.h, un.b);
        ++q_iter;
        if (stall) {  // test hook: let Q land, then never load K or V
            drain_wait(bar(kBarQFull), (q_iter - 1) & 1u);
            finish();
            return;
        }
        EntryReader er;
        er.init(un.entries, un.E);
        for (int e = 0; e < un.E && ok; ++e) {
            int j = er.get(e) & 0xFFFF;
            FA_DCHECK_INDEX(j, p.KVB, p.status);
            // K_j and V_j: rows j*128.. of batch b, or with paged K/V the page the table gives
            // for (b, j) (a page outside the pools is recorded and reads as zeros).
            int kv_row = j * kBlock, kv_batch = un.b;
            if (p.page_table) {
                int page = 0;
                if (leader) page = __ldg(p.page_table + (size_t)un.b * p.page_stride + j);
                page = __shfl_sync(kFullMask, page, leader_lane);
                if (leader && (page < 0 || page >= p.n_pages)) atomicExch(p.status, 2);
                kv_row = 0;
                kv_batch = page;
            }
            for (int which = 0; which < 2; ++which) {
                const int s = (int)(kv_pos % C::kStages);
                const uint32_t ph = (kv_pos / C::kStages) & 1u;
                FA_TRACE_EV(0, 30 + which);
                if (!wait(C::kBarSlotEmpty + s, ph ^ 1u)) { ok = false; break; }
                FA_TRACE_EV(0, 32 + which);
                mbar_arrive_expect_tx_if(leader, bar(C::kBarSlotFull + s), (uint32_t)C::kTileBytes);
                const CUtensorMap* tm = which ? tmv : tmk;
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_4d_if(leader, sKV + s * C::kTileBytes + c * 16384, tm,
                                   bar(C::kBarSlotFull + s), c * 64, kv_row, un.h, kv_batch);
                ++kv_pos;
            }
        }
    }
    if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        const uint32_t n = kv_pos < (uint32_t)C::kStages ? kv_pos : (uint32_t)C::kStages;
        for (uint32_t k = 0; k < n; ++k) {
            const uint32_t pos = kv_pos - 1 - k;
            drain_wait(bar(C::kBarSlotFull + (int)(pos % C::kStages)), (pos / C::kStages) & 1u);
        }
        if (q_iter > 0) drain_wait(bar(kBarQFull), (q_iter - 1) & 1u);
    }
    finish();
}

// A query row with no live key: O = 0 and lse = -inf (nothing for rows past Q_LEN).
template <int D, bool BF16>
__device__ __forceinline__ void store_row_zero(const FwdParams& p, const Unit& un, int q) {
    if (q >= p.Q_LEN) return;
    uint16_t* o = reinterpret_cast<uint16_t*>(p.out) + un.b * p.out_stride[0] +
                  un.h * p.out_stride[1] + (int64_t)q * p.out_stride[2];
#pragma unroll
    for (int d = 0; d < D; d += 8) *reinterpret_cast<uint4*>(o + d) = make_uint4(0, 0, 0, 0);
    if (p.lse) p.lse[((int64_t)un.b * p.H + un.h) * p.Q_LEN + q] = -INFINITY;
}

}  // namespace
}  // namespace fa
