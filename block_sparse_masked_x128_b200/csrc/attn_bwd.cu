// attn_bwd.cu -- block-sparse attention backward for sm_100a.
//
// What it computes: the gradients dQ, dK, dV of the forward's
//   O = softmax(mask(score_mod(scale * Q K^T))) V
// for an upstream gradient dO, over the same block mask.  The pages name the deterministic
// FlexAttention backward ("PyTorch 2.13 brings custom AI attention to Mac", "What Else
// Shipped in PyTorch 2.13?") and the dQ write order of the block mask
// ("tensorplay.nn.attention.create_block_mask", Parameters compute_dq_write_order and
// dq_kv_order); the arithmetic is the derivative of the forward's definition:
//   P = exp(s' - lse)          dV = P^T dO                dP = dO V^T
//   Delta_i = sum_d dO[i,d] O[i,d]                        dS = P * (dP - Delta) * score_mod'(s)
//   dQ = scale * dS K          dK = scale * dS^T Q
// with lse the forward's log-sum-exp, so P is recomputed exactly as the forward formed it.
//
// Three kernels, all deterministic (no atomics, no order that depends on timing):
//   bwd_preprocess_kernel   -Delta per query row and -lse in log2 units, into a caller-provided
//                           workspace padded to whole 128-row blocks (-inf / 0 in the padding,
//                           so padded rows get P = 0);
//   dK/dV kernel            one unit per kv block j (kv-major lists of the mask): K_j, V_j stay
//                           in shared memory while the query blocks i of the unit stream
//                           through a ring of stages (Q_i, dO_i, lse_i, Delta_i);
//                             S^T = K_j Q_i^T and dP^T = V_j dO_i^T     (SS MMAs into TMEM)
//                             P^T, dS^T in registers, written back to TMEM as 16-bit pairs
//                             dV += P^T dO_i and dK += dS^T Q_i          (TS MMAs, A from TMEM)
//   dQ kernel               one unit per query block i: Q_i, dO_i stay, K_j, V_j stream in the
//                           mask's dQ write order (descending or ascending j);
//                             S = Q_i K_j^T, dP = dO_i V_j^T, dS in its own columns,
//                             dQ += dS K_j.
// Each CTA owns its unit's accumulators in TMEM, so every sum runs in a fixed order.
//
// Organisation of both main kernels (one persistent CTA per SM, 12 warps, units handed out
// at run time longest first, as in the forward):
//   warp 0      TMA producer;   warp 1 MMA issuer (one elected lane);   warp 2 TMEM allocation;
//   warps 4-11  element-wise math, one TMEM lane (row) per thread, in two groups (warps 4-7,
//               8-11) that split each tile's columns; in the epilogue they write the two
//               accumulators (dV / dK) or the two halves of dQ.
// TMEM (512 columns), three layouts (BCfg): the dK/dV pass at D = 64 and the dQ pass keep P
// and dS in columns of their own after the accumulators, so the next entry's S and dP are
// computed while the math warps work (at D = 64 the dQ pass also holds Q_i and dO_i as MMA A
// operands); the dK/dV pass at D = 128, whose accumulators take 256 columns, works in
// half-steps of 64 queries with two 128-column buffers of S^T / dP^T, P and dS written over
// the columns just read.  All waits are bounded.
#include <cfloat>

#include <cuda_fp16.h>

#include "fa_internal.h"
#include "fa_trace.cuh"
#include "sm100_ptx.cuh"
#include "fwd_common.cuh"

#ifdef FA_TRACE
// The backward's own trace buffer (the tracer's device pointer is per translation unit).
extern "C" int fa_debug_set_trace_buffer_bwd(void* device_ptr) {
    return (int)cudaMemcpyToSymbol(g_fa_trace, &device_ptr, sizeof(device_ptr));
}
#endif

namespace fa {
namespace {

constexpr int kThreadsBwd = 384;
constexpr int kRegsAtLaunchBwd = 168;
constexpr int kRegsIssueBwd = 104;
constexpr int kRegsMathBwd = 200;
static_assert(128 * kRegsIssueBwd + 256 * kRegsMathBwd <= kThreadsBwd * kRegsAtLaunchBwd,
              "register split exceeds the launched pool");

enum : int {
    kBbFixFull = 0,     // the unit's fixed tiles landed (dK/dV: K_j, V_j; dQ: Q_i, dO_i)
    kBbFixEmpty = 1,    // the MMA warp is done with them
    kBbSFull = 2,       // S and dP of the current entry are in TMEM
    kBbPReady = 3,      // the math warps wrote the 16-bit operands of the accumulating MMAs
    kBbAccFull = 4,     // the unit's accumulators are complete
    kBbAccFree = 5,     // the epilogue has read them
    kBbDrain = 6,
    kBbLoaded = 7,      // all eight math warps hold S and dP in registers
    kBbAccDone = 8,     // the accumulating MMAs of the last entry are done (P, dS columns free)
    kBbUnitFull = 9,    // + unit-ring slot (2)
    kBbUnitEmpty = 11,  // + unit-ring slot (2)
    kBbSlot = 13        // + stage (full), then + stage (empty)
};

// KV: the dK/dV kernel (its stages also carry 128 lse and 128 Delta values).
template <int D, bool KV>
struct BCfg {
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kVecBytes = KV ? 1024 : 0;
    static constexpr int kStageBytes = 2 * kTileBytes + kVecBytes;   // multiple of 1024
    static constexpr int kStages = (D == 64) ? 5 : 2;
    static constexpr int kChunks = D / 64;
    static constexpr int kBarUFull = kBbUnitFull;
    static constexpr int kBarUEmpty = kBbUnitEmpty;
    static constexpr int kBarSlotFull = kBbSlot;
    static constexpr int kBarSlotEmpty = kBbSlot + kStages;
    // Half-step barriers of the dK/dV pass at D = 128 (S / dP full, P / dS ready), per buffer.
    static constexpr int kBarSFullH = kBbSlot + 2 * kStages;
    static constexpr int kBarPReadyH = kBarSFullH + 2;
    static constexpr int kNumBars = kBarPReadyH + 2;
    static constexpr int kStageOff = 2 * kTileBytes;
    static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;   // + alignment slack
    static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256, kColAcc1 = 256 + D;
    // Where TMEM has room (the dK/dV pass at D = 64, the dQ pass at both head sizes) the 16-bit
    // P and dS get columns of their own after the accumulators, so the next entry's S and dP can
    // be computed while the math warps still work on the current entry; otherwise (the dK/dV
    // pass at D = 128 fills all 512 columns) each math group writes its 16-bit P and dS over the
    // first 32 columns of its own 64 S and dP columns (group g: 64g.., 128 + 64g..), and the
    // MMAs and the element-wise pass alternate.
    static constexpr bool kSep = KV ? (D == 64) : true;
    // The dK/dV pass at D = 128 works in half-steps of 64 queries: S^T and dP^T of a half are
    // 64 columns each, in two buffers (columns 0-127 and 128-255), so the MMAs of half k + 1 run
    // while the math warps work on half k; the 16-bit P and dS of a half are written over the
    // first 16 of each group's 32 S and dP columns in the half's buffer.
    static constexpr bool kHalves = KV && D == 128;
    // The dQ pass at D = 64 keeps its fixed tiles (Q_i, dO_i: the A operands of S and dP) in
    // TMEM, copied there once per unit, so those MMAs read only B (K_j, V_j) from shared memory
    // and the fixed tiles' shared memory is free for the next unit as soon as the copy is done.
    static constexpr bool kTmemA = !KV && D == 64;
    static constexpr uint32_t kColA0 = 384, kColA1 = 384 + D / 2;
    static constexpr uint32_t kAccEnd = KV ? 256 + 2 * D : 256 + D;
    static constexpr uint32_t kColP = kSep ? kAccEnd : kColS;
    static constexpr uint32_t kColDS = kSep ? (KV ? kAccEnd + 64 : kAccEnd) : kColDP;
    static_assert(!kSep || kColDS + 64 <= 512, "TMEM budget");
    static_assert(!kTmemA || (kColA0 >= kColDS + 64 && kColA1 + D / 2 <= 512), "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct BUnit {
    int b, h, idx, E;
    const int32_t* entries;
};

__device__ __forceinline__ BUnit decode_bunit(const BwdParams& p, int u) {
    const int BH = p.B * p.H;
    int r, bh;
    if (p.head_major) {
        bh = u / p.units_per_bh;
        r = u - bh * p.units_per_bh;
    } else {
        r = u / BH;
        bh = u - r * BH;
    }
    BUnit un;
    un.b = bh / p.H;
    un.h = bh - un.b * p.H;
    const int mb = (p.maskB == 1) ? 0 : un.b, mh = (p.maskH == 1) ? 0 : un.h;
    const size_t base = ((size_t)mb * p.maskH + mh) * p.units_per_bh;
    un.idx = __ldg(p.order + base + r);
    FA_DCHECK_INDEX(un.idx, p.units_per_bh, p.status);
    un.E = __ldg(p.count + base + un.idx);
    FA_DCHECK_INDEX(un.E, p.entries_stride + 1, p.status);
    un.entries = p.entries + (base + un.idx) * (size_t)p.entries_stride;
    return un;
}

__device__ __forceinline__ float alibi_slope_log2(const BwdParams& p, int h) {
    float slope;
    if (p.alibi_slopes) {
        slope = __ldg(p.alibi_slopes + h);
    } else {
        const int num = 8 * (h + 1);
        slope = (num % p.H == 0) ? ldexpf(1.0f, -(num / p.H)) : exp2f(-(float)num / (float)p.H);
    }
    return slope * kLog2e;
}

// ------------------------------------------------------------------ producer (warp 0)

// KV = true: fixed tiles K_j, V_j; stages Q_i, dO_i, lse_i, Delta_i.
// KV = false: fixed tiles Q_i, dO_i; stages K_j, V_j.
template <int D, bool KV>
__device__ void bwd_producer(const BwdParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, const CUtensorMap* tdo, uint32_t sbase,
                             uint32_t bars, volatile int* ring, volatile int* abort_flag) {
    using C = BCfg<D, KV>;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    // Off the critical path (it runs ahead of the MMA warp): sleep between polls.
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded_sleepy(bar(i), par, abort_flag, p.status, kWaitLimitNs, kProducerSleepNs);
    };
    const CUtensorMap* fix0 = KV ? tk : tq;
    const CUtensorMap* fix1 = KV ? tv : tdo;
    const CUtensorMap* st0 = KV ? tq : tk;
    const CUtensorMap* st1 = KV ? tdo : tv;
    const uint32_t leader = elect_one_lane();
    if (leader) {
        tma_prefetch_desc(tq);
        tma_prefetch_desc(tk);
        tma_prefetch_desc(tv);
        tma_prefetch_desc(tdo);
    }
    __syncwarp();
    const int leader_lane = __ffs(__ballot_sync(kFullMask, leader != 0)) - 1;
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
    uint32_t pos = 0, fix_iter = 0, u_iter = 0;
    bool ok = true;
    FA_TRACE_DECL
    for (;;) {
        int u = -1;
        if (leader) {
            const int v = atomicAdd(p.sched_ctr, 1);
            u = v < p.n_units ? v : -1;
        }
        u = __shfl_sync(kFullMask, u, leader_lane);
        {
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
        const BUnit un = decode_bunit(p, u);
        if (un.E == 0) continue;
        FA_TRACE_EV(KV ? 0 : 12, 32);
        if (!wait(kBbFixEmpty, (fix_iter & 1u) ^ 1u)) { ok = false; break; }
        FA_TRACE_EV(KV ? 0 : 12, 33);
        mbar_arrive_expect_tx_if(leader, bar(kBbFixFull), (uint32_t)(2 * C::kTileBytes));
        for (int c = 0; c < C::kChunks; ++c) {
            tma_load_4d_if(leader, sbase + c * 16384, fix0, bar(kBbFixFull), c * 64, un.idx * kBlock,
                           un.h, un.b);
            tma_load_4d_if(leader, sbase + C::kTileBytes + c * 16384, fix1, bar(kBbFixFull), c * 64,
                           un.idx * kBlock, un.h, un.b);
        }
        ++fix_iter;
        if (p.stall_loads) {   // test hook: let the fixed tiles land, then load nothing more
            drain_wait(bar(kBbFixFull), (fix_iter - 1) & 1u);
            finish();
            return;
        }
        EntryReader er;
        er.init(un.entries, un.E);
        const size_t vec_row = ((size_t)un.b * p.H + un.h) * (size_t)p.q_pad;
        for (int e = 0; e < un.E; ++e) {
            int t = er.get(e) & 0xFFFF;
            FA_DCHECK_INDEX(t, p.entries_stride, p.status);
            const int s = (int)(pos % C::kStages);
            FA_TRACE_EV(KV ? 0 : 12, 30);
            if (!wait(C::kBarSlotEmpty + s, ((pos / C::kStages) & 1u) ^ 1u)) { ok = false; break; }
            FA_TRACE_EV(KV ? 0 : 12, 31);
            const uint32_t dst = sbase + C::kStageOff + (uint32_t)s * C::kStageBytes;
            mbar_arrive_expect_tx_if(leader, bar(C::kBarSlotFull + s),
                                     (uint32_t)(2 * C::kTileBytes + C::kVecBytes));
            for (int c = 0; c < C::kChunks; ++c) {
                tma_load_4d_if(leader, dst + c * 16384, st0, bar(C::kBarSlotFull + s), c * 64,
                               t * kBlock, un.h, un.b);
                tma_load_4d_if(leader, dst + C::kTileBytes + c * 16384, st1, bar(C::kBarSlotFull + s),
                               c * 64, t * kBlock, un.h, un.b);
            }
            if constexpr (KV) {
                if (leader) {
                    bulk_load(dst + 2 * C::kTileBytes, p.neg_lse_log2 + vec_row + (size_t)t * kBlock, 512,
                              bar(C::kBarSlotFull + s));
                    bulk_load(dst + 2 * C::kTileBytes + 512, p.neg_delta + vec_row + (size_t)t * kBlock, 512,
                              bar(C::kBarSlotFull + s));
                }
                __syncwarp();
            }
            ++pos;
        }
        if (!ok) break;
    }
    if (!ok) {
        const uint32_t n = pos < (uint32_t)C::kStages ? pos : (uint32_t)C::kStages;
        for (uint32_t k = 0; k < n; ++k) {
            const uint32_t q = pos - 1 - k;
            drain_wait(bar(C::kBarSlotFull + (int)(q % C::kStages)), (q / C::kStages) & 1u);
        }
        if (fix_iter > 0) drain_wait(bar(kBbFixFull), (fix_iter - 1) & 1u);
    }
    finish();
}

// ------------------------------------------------------------------ MMA issuer (warp 1)

template <int D, bool BF16, bool KV>
__device__ void bwd_mma(const BwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                        const volatile int* ring, volatile int* abort_flag) {
    using C = BCfg<D, KV>;
    const uint32_t leader = elect_one_lane();
    constexpr uint32_t kIdescSS = make_idesc_f16(BF16, 128, 128, false);
    constexpr uint32_t kIdescAcc = make_idesc_f16(BF16, 128, D, true);
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    // D[128 x 128] = A B^T with A, B both 128 x D tiles, K-major, 128-byte swizzle.
    auto issue_ss = [&](uint32_t dcol, uint32_t a, uint32_t b) {
        const uint64_t ad = make_sdesc_sw128(a, 16, 1024);
        const uint64_t bd = make_sdesc_sw128(b, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss_if(leader, tmem + dcol, ad + off, bd + off, kIdescSS, kk > 0 ? 1u : 0u);
        }
    };
    // D[128 x D] (+)= A[128 x 128] B[128 x D]: A 16-bit pairs in TMEM, B MN-major in smem.
    // The K step kk covers columns 16kk .. 16kk+15 of the 128 x 128 tile, 8 columns of 16-bit
    // pairs: contiguous with separate P / dS columns, else in the two groups' own column blocks.
    auto issue_ts = [&](uint32_t dcol, uint32_t acol, uint32_t b, bool accumulate) {
        const uint64_t bd = make_sdesc_sw128(b, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk) {
            const uint32_t aoff = C::kSep ? (uint32_t)(kk * 8) : (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8);
            mma_ts_if(leader, tmem + dcol, tmem + acol + aoff, bd + (uint64_t)((kk * 2048) >> 4),
                      kIdescAcc, (kk > 0 || accumulate) ? 1u : 0u);
        }
    };
    // D[128 x 128] = A B^T with A (128 x D, 16-bit pairs) in TMEM at acol, B K-major in smem.
    auto issue_ts_a = [&](uint32_t dcol, uint32_t acol, uint32_t b) {
        const uint64_t bd = make_sdesc_sw128(b, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ts_if(leader, tmem + dcol, tmem + acol + 8u * (uint32_t)kk, bd + off, kIdescSS, kk > 0 ? 1u : 0u);
        }
    };
    uint32_t pos = 0, fix_iter = 0, acc_iter = 0, pr_iter = 0, ld_iter = 0, u_iter = 0;
    bool ok = true;
    const uint32_t sFix0 = sbase, sFix1 = sbase + C::kTileBytes;
    FA_TRACE_DECL
    auto stage0 = [&](uint32_t ps) { return sbase + C::kStageOff + (ps % C::kStages) * C::kStageBytes; };
    // S (or S^T) and dP (or dP^T) of the entry at ring position ps.
    auto issue_s_dp = [&](uint32_t ps) -> bool {
        const int s = (int)(ps % C::kStages);
        if (!wait(C::kBarSlotFull + s, (ps / C::kStages) & 1u)) return false;
        tc_fence_after();
        const uint32_t st0 = stage0(ps), st1 = st0 + C::kTileBytes;
        if constexpr (C::kTmemA) {
            issue_ts_a(C::kColS, C::kColA0, st0);    // S = Q_i K_j^T, Q_i from TMEM
            issue_ts_a(C::kColDP, C::kColA1, st1);   // dP = dO_i V_j^T, dO_i from TMEM
        } else {
            issue_ss(C::kColS, sFix0, st0);    // dK/dV pass: S^T = K_j Q_i^T;  dQ pass: S = Q_i K_j^T
            issue_ss(C::kColDP, sFix1, st1);   // dK/dV pass: dP^T = V_j dO_i^T; dQ pass: dP = dO_i V_j^T
        }
        tc_commit_if(leader, bar(kBbSFull));
        return true;
    };
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) break;
        const BUnit un = decode_bunit(p, u);
        if (un.E == 0) continue;
        FA_TRACE_EV(KV ? 1 : 13, 20);
        if (!wait(kBbFixFull, fix_iter & 1u)) { ok = false; break; }
        FA_TRACE_EV(KV ? 1 : 13, 21);
        ++fix_iter;
        tc_fence_after();
        if constexpr (C::kTmemA) {
            // Q_i and dO_i into TMEM (after the last unit's MMAs, which read the old copy, in
            // issue order); their shared memory is released once the copies have completed.
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                tc_cp_128x256b_if(leader, tmem + C::kColA0 + 8u * (uint32_t)kk, make_sdesc_sw128(sFix0, 16, 1024) + off);
                tc_cp_128x256b_if(leader, tmem + C::kColA1 + 8u * (uint32_t)kk, make_sdesc_sw128(sFix1, 16, 1024) + off);
            }
            tc_commit_if(leader, bar(kBbFixEmpty));
        }
        if constexpr (C::kSep) {
            if (!issue_s_dp(pos)) { ok = false; break; }
        }
        for (int e = 0; e < un.E; ++e) {
            const uint32_t ps = pos;
            if constexpr (C::kSep) {
                // The next entry's S and dP as soon as the math warps hold this entry's.
                if (e + 1 < un.E) {
                    FA_TRACE_EV(KV ? 1 : 13, 22);
                    if (!wait(kBbLoaded, ld_iter & 1u)) { ok = false; break; }
                    FA_TRACE_EV(KV ? 1 : 13, 23);
                    ++ld_iter;
                    if (!issue_s_dp(ps + 1)) { ok = false; break; }
                } else {
                    if (!wait(kBbLoaded, ld_iter & 1u)) { ok = false; break; }
                    ++ld_iter;
                }
            } else {
                if (!issue_s_dp(ps)) { ok = false; break; }
            }
            FA_TRACE_EV(KV ? 1 : 13, 24);
            if (!wait(kBbPReady, pr_iter & 1u)) { ok = false; break; }
            FA_TRACE_EV(KV ? 1 : 13, 25);
            ++pr_iter;
            if (e == 0 && !wait(kBbAccFree, (acc_iter & 1u) ^ 1u)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st0 = stage0(ps), st1 = st0 + C::kTileBytes;
            if constexpr (KV) {
                issue_ts(C::kColAcc0, C::kColP, st1, e > 0);    // dV += P^T dO_i
                issue_ts(C::kColAcc1, C::kColDS, st0, e > 0);   // dK += dS^T Q_i
            } else {
                issue_ts(C::kColAcc0, C::kColDS, st0, e > 0);   // dQ += dS K_j
            }
            tc_commit_if(leader, bar(C::kBarSlotEmpty + (int)(ps % C::kStages)));
            if constexpr (C::kSep) tc_commit_if(leader, bar(kBbAccDone));
            ++pos;
        }
        if (!ok) break;
        tc_commit_if(leader, bar(kBbAccFull));
        if constexpr (!C::kTmemA) tc_commit_if(leader, bar(kBbFixEmpty));
        ++acc_iter;
    }
    if (!ok) {
        tc_commit_if(leader, bar(kBbDrain));
        drain_wait(bar(kBbDrain), 0u);
    }
}

// ------------------------------------------------------------------ element-wise math (warps 4-11)

// Score in log2 units after score_mod; t returns tanh of the soft-cap (for its derivative).
template <int SCORE>
__device__ __forceinline__ float score_log2(const BwdParams& p, float raw, float bias_log2, float& t) {
    float x;
    if constexpr ((SCORE & FA_SCORE_SOFTCAP) != 0) {
        t = tanh_approx(raw * p.inv_softcap_scale);
        x = p.softcap_log2 * t;
    } else {
        t = 0.f;
        x = raw * p.scale_log2;
    }
    if constexpr ((SCORE & FA_SCORE_ALIBI) != 0) x += bias_log2;
    return x;
}

constexpr int kVarDocumentB = 4;

// Writes a zero row of `cols` 16-bit values starting at column c0 (rows without live tiles).
__device__ __forceinline__ void store_zero_cols(uint16_t* row, int cols) {
    for (int d = 0; d < cols; d += 8) *reinterpret_cast<uint4*>(row + d) = make_uint4(0, 0, 0, 0);
}

// Per-row constants of the element-wise pass.
struct PairConsts {
    float2 sc2, inv2, cap2, step2;
    int lo, hi;             // live columns [lo, hi] of the row on a partial tile
    int row_doc;
    const int* doc_cols;    // document id of column 0 of the 32 (partial tiles with documents)
};

// P and dS of 32 columns of one row (16 pairs) from S and dP read out of TMEM, as 16-bit pairs:
//   x = score_mod(s) in log2 units,  P = 2^(x + nl),  dS = P (dP + nd) (1 - tanh^2 under a cap),
// with nl = -lse log2(e) and nd = -Delta of the pair's columns (nlv(i) / ndv(i)).  PART: the
// tile is partial, so columns outside [lo, hi] (and of another document) get P = 0.
template <bool BF16, int SCORE, bool DOC, bool PART, typename NL, typename ND>
__device__ __forceinline__ void bwd_pairs(const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                          const PairConsts& k, float2& pos2, NL nlv, ND ndv,
                                          uint32_t (&pk)[16], uint32_t (&dk)[16]) {
    constexpr bool kSoftcap = (SCORE & FA_SCORE_SOFTCAP) != 0;
    constexpr bool kAlibi = (SCORE & FA_SCORE_ALIBI) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int c = 2 * i;
        const float2 raw = make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
        const float2 dp = make_float2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1]));
        const float2 nl = nlv(i);
        float2 ex, th;
        if constexpr (kSoftcap) {
            const float2 a = __fmul2_rn(raw, k.inv2);
            th = make_float2(tanh_approx(a.x), tanh_approx(a.y));
            if constexpr (kAlibi) ex = __fadd2_rn(__ffma2_rn(k.cap2, th, pos2), nl);
            else ex = __ffma2_rn(k.cap2, th, nl);
        } else {
            if constexpr (kAlibi) ex = __fadd2_rn(__ffma2_rn(raw, k.sc2, pos2), nl);
            else ex = __ffma2_rn(raw, k.sc2, nl);
        }
        if constexpr (kAlibi) pos2 = __fadd2_rn(pos2, k.step2);
        float2 pr = make_float2(ex2_approx(ex.x), ex2_approx(ex.y));
        if constexpr (PART) {
            bool l0 = c >= k.lo && c <= k.hi, l1 = c + 1 >= k.lo && c + 1 <= k.hi;
            if constexpr (DOC) {
                l0 = l0 && (__ldg(k.doc_cols + c) == k.row_doc);
                l1 = l1 && (__ldg(k.doc_cols + c + 1) == k.row_doc);
            }
            pr = make_float2(l0 ? pr.x : 0.f, l1 ? pr.y : 0.f);
        }
        float2 ds = __fmul2_rn(pr, __fadd2_rn(dp, ndv(i)));
        if constexpr (kSoftcap) ds = __fmul2_rn(ds, __ffma2_rn(make_float2(-th.x, -th.y), th, make_float2(1.f, 1.f)));
        pk[i] = pack2<BF16>(pr.x, pr.y);
        dk[i] = pack2<BF16>(ds.x, ds.y);
    }
}

template <int D, bool BF16, int VAR, bool KV>
__device__ void bwd_math(const BwdParams& p, int g, uint32_t sbase, uint32_t bars, uint32_t tmem,
                         const volatile int* ring, volatile int* abort_flag) {
    using C = BCfg<D, KV>;
    constexpr int SCORE = VAR & (FA_SCORE_SOFTCAP | FA_SCORE_ALIBI);
    constexpr bool kDoc = (VAR & kVarDocumentB) != 0;
    constexpr bool kSoftcap = (SCORE & FA_SCORE_SOFTCAP) != 0;
    constexpr bool kAlibi = (SCORE & FA_SCORE_ALIBI) != 0;
    const int wq = (threadIdx.x >> 5) & 3;
    const int lane = threadIdx.x & 31;
    const int r = wq * 32 + lane;                       // row of the tile (TMEM lane)
    const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_bits + C::kColS + 64u * g;
    const uint32_t tDP = tmem + lane_bits + C::kColDP + 64u * g;
    // 16-bit pairs of P and dS: 32 columns per group, after the accumulators or over the
    // group's own S and dP columns.
    const uint32_t tP = tmem + lane_bits + C::kColP + (C::kSep ? 32u : 64u) * g;
    const uint32_t tDS = tmem + lane_bits + C::kColDS + (C::kSep ? 32u : 64u) * g;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    uint32_t pos = 0, sf_iter = 0, acc_iter = 0, u_iter = 0, ld_iter = 0, ad_iter = 0;
    bool ok = true;
    FA_TRACE_DECL
    const int tslot = (threadIdx.x >> 5) + (KV ? 0 : 12);   // trace slot: warp, by pass
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) return;
        const BUnit un = decode_bunit(p, u);
        const int row_pos = un.idx * kBlock + r;    // kv (dK/dV kernel) or q (dQ kernel)
        // The gradient this thread writes in the epilogue, and its columns.
        uint16_t* grow;
        int gcol0, gcols;
        float gmul;
        if constexpr (KV) {
            const bool dk = (g == 1);
            const int64_t* st = dk ? p.grad0_stride : p.grad1_stride;
            grow = reinterpret_cast<uint16_t*>(dk ? p.grad0 : p.grad1) + un.b * st[0] + un.h * st[1] +
                   (int64_t)row_pos * st[2];
            gcol0 = 0;
            gcols = D;
            gmul = dk ? p.scale : 1.0f;
        } else {
            grow = reinterpret_cast<uint16_t*>(p.grad0) + un.b * p.grad0_stride[0] +
                   un.h * p.grad0_stride[1] + (int64_t)row_pos * p.grad0_stride[2];
            gcol0 = g * (D / 2);
            gcols = D / 2;
            gmul = p.scale;
        }
        const bool row_in = row_pos < (KV ? p.KV_LEN : p.Q_LEN);
        if (un.E == 0) {
            if (row_in) store_zero_cols(grow + gcol0, gcols);
            continue;
        }
        const float slope_log2 = kAlibi ? alibi_slope_log2(p, un.h) : 0.f;
        const size_t vec_row = ((size_t)un.b * p.H + un.h) * (size_t)p.q_pad;
        // dQ kernel: this thread's query row has one lse and one Delta.
        float row_l = 0.f, row_d = 0.f;
        if constexpr (!KV) {
            row_l = __ldg(p.neg_lse_log2 + vec_row + row_pos);
            row_d = __ldg(p.neg_delta + vec_row + row_pos);
        }
        const int row_doc = (kDoc && row_pos < p.QB * kBlock) ? __ldg(p.doc_id + row_pos) : 0;
        const int kv_len = p.kv_lens ? min(p.KV_LEN, __ldg(p.kv_lens + (p.maskB == 1 ? 0 : un.b))) : p.KV_LEN;
        EntryReader er;
        er.init(un.entries, un.E);
        for (int e = 0; e < un.E; ++e) {
            const int code = er.get(e);
            int t = code & 0xFFFF;
            FA_DCHECK_INDEX(t, p.entries_stride, p.status);
            const bool full = (code & kFull0) != 0;
            const int s = (int)(pos % C::kStages);
            ++pos;
            FA_TRACE_EV(tslot, 2);
            if (!wait(kBbSFull, sf_iter & 1u)) { ok = false; break; }
            FA_TRACE_EV(tslot, 3);
            ++sf_iter;
            tc_fence_after();
            const int col0 = t * kBlock + 64 * g;        // first column position (q or kv)
            // Live columns [lo, hi] of this row on a partial tile (+ the document compare).
            int lo = 0, hi = 63;
            if (!full) {
                if constexpr (KV) {
                    // row = key kv, columns = queries q
                    const int kv = row_pos;
                    if (kv >= kv_len) hi = -1;
                    hi = min(hi, p.Q_LEN - 1 - col0);
                    if (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) lo = max(lo, kv - col0);
                    if (p.mask_kind & FA_MASK_SLIDING_WINDOW) hi = min(hi, kv + p.window - 1 - col0);
                } else {
                    // row = query q, columns = keys kv
                    const int q = row_pos;
                    if (q >= p.Q_LEN) hi = -1;
                    hi = min(hi, kv_len - 1 - col0);
                    if (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) hi = min(hi, q - col0);
                    if (p.mask_kind & FA_MASK_SLIDING_WINDOW) lo = max(lo, q - p.window + 1 - col0);
                }
            }
            const float* vl = nullptr;   // dK/dV pass: the stage's lse and Delta of the columns
            const float* vd = nullptr;
            if constexpr (KV) {
                const uint8_t* st = reinterpret_cast<const uint8_t*>(__cvta_shared_to_generic(
                    sbase + C::kStageOff + (uint32_t)s * C::kStageBytes + 2 * C::kTileBytes));
                vl = reinterpret_cast<const float*>(st) + 64 * g;
                vd = reinterpret_cast<const float*>(st + 512) + 64 * g;
            }
            // Column c's bias is slope * (kv - q): +1 per column in the dQ pass (kv grows),
            // -1 per column in the dK/dV pass (q grows).  Pairs of columns in packed f32x2.
            const float bias0 = KV ? slope_log2 * (float)(row_pos - col0) : slope_log2 * (float)(col0 - row_pos);
            const float dbias = KV ? -slope_log2 : slope_log2;
            float2 pos2 = make_float2(bias0, bias0 + dbias);
            PairConsts pc;
            pc.sc2 = make_float2(p.scale_log2, p.scale_log2);
            pc.inv2 = make_float2(p.inv_softcap_scale, p.inv_softcap_scale);
            pc.cap2 = make_float2(p.softcap_log2, p.softcap_log2);
            pc.step2 = make_float2(2.f * dbias, 2.f * dbias);
            pc.row_doc = row_doc;
            const float2 nrl2 = make_float2(row_l, row_l), nrd2 = make_float2(row_d, row_d);
            // P and dS of one 32-column half (h2) of this group's 64 columns, in 16-bit pairs.
            auto half = [&](int h2, const uint32_t (&sr)[32], const uint32_t (&dr)[32], uint32_t (&pk)[16],
                            uint32_t (&dk)[16]) {
                PairConsts k = pc;
                k.lo = lo - 32 * h2;
                k.hi = hi - 32 * h2;
                k.doc_cols = kDoc ? p.doc_id + col0 + 32 * h2 : nullptr;
                auto nl = [&](int i) -> float2 {
                    if constexpr (KV) return *reinterpret_cast<const float2*>(vl + 32 * h2 + 2 * i);
                    else return nrl2;
                };
                auto nd = [&](int i) -> float2 {
                    if constexpr (KV) return *reinterpret_cast<const float2*>(vd + 32 * h2 + 2 * i);
                    else return nrd2;
                };
                if (full) bwd_pairs<BF16, SCORE, kDoc, false>(sr, dr, k, pos2, nl, nd, pk, dk);
                else bwd_pairs<BF16, SCORE, kDoc, true>(sr, dr, k, pos2, nl, nd, pk, dk);
            };
            uint32_t pk0[16], dk0[16];
            if constexpr (C::kSep && !KV) {
                // dQ pass (dS only): both halves of S and dP into registers at once, so the MMA
                // warp computes the next entry's S and dP during all of this entry's math (at
                // D = 128 those MMAs take longer than the math).
                uint32_t sr0[32], dr0[32], sr1[32], dr1[32], dk1[16];
                tmem_ld_32x32b_x32(tS, sr0);
                tmem_ld_32x32b_x32(tDP, dr0);
                tmem_ld_32x32b_x32(tS + 32, sr1);
                tmem_ld_32x32b_x32(tDP + 32, dr1);
                tmem_ld_wait();
                reg_fence<32>(sr0);
                reg_fence<32>(dr0);
                reg_fence<32>(sr1);
                reg_fence<32>(dr1);
                tc_fence_before();
                mbar_arrive_warp(bar(kBbLoaded));
                FA_TRACE_EV(tslot, 4);
                half(0, sr0, dr0, pk0, dk0);
                half(1, sr1, dr1, pk0, dk1);
                FA_TRACE_EV(tslot, 5);
                if (!wait(kBbAccDone, (ad_iter & 1u) ^ 1u)) { ok = false; break; }
                FA_TRACE_EV(tslot, 6);
                ++ad_iter;
                tc_fence_after();
                tmem_st_32x32b_x16(tDS, dk0);
                tmem_st_32x32b_x16(tDS + 16, dk1);
            } else if constexpr (C::kSep) {
                // dK/dV pass: half 0, then half 1's loads; once both halves of S and dP are in
                // registers the MMA warp may compute the next entry's into them.  P and dS go to
                // their own columns after the last entry's accumulating MMAs have read those.
                {
                    uint32_t sr[32], dr[32];
                    tmem_ld_32x32b_x32(tS, sr);
                    tmem_ld_32x32b_x32(tDP, dr);
                    tmem_ld_wait();
                    reg_fence<32>(sr);
                    reg_fence<32>(dr);
                    half(0, sr, dr, pk0, dk0);
                }
                uint32_t sr[32], dr[32], pk1[16], dk1[16];
                tmem_ld_32x32b_x32(tS + 32, sr);
                tmem_ld_32x32b_x32(tDP + 32, dr);
                tmem_ld_wait();
                reg_fence<32>(sr);
                reg_fence<32>(dr);
                tc_fence_before();
                mbar_arrive_warp(bar(kBbLoaded));
                FA_TRACE_EV(tslot, 4);
                half(1, sr, dr, pk1, dk1);
                FA_TRACE_EV(tslot, 5);
                if (!wait(kBbAccDone, (ad_iter & 1u) ^ 1u)) { ok = false; break; }
                FA_TRACE_EV(tslot, 6);
                ++ad_iter;
                tc_fence_after();
                if constexpr (KV) {
                    tmem_st_32x32b_x16(tP, pk0);
                    tmem_st_32x32b_x16(tP + 16, pk1);
                }
                tmem_st_32x32b_x16(tDS, dk0);
                tmem_st_32x32b_x16(tDS + 16, dk1);
            } else {
                // Over the group's own columns, half by half: each half's P and dS land on S and
                // dP columns this group has already read.
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t sr[32], dr[32];
                    tmem_ld_32x32b_x32(tS + 32 * h2, sr);
                    tmem_ld_32x32b_x32(tDP + 32 * h2, dr);
                    tmem_ld_wait();
                    reg_fence<32>(sr);
                    reg_fence<32>(dr);
                    half(h2, sr, dr, pk0, dk0);
                    if constexpr (KV) tmem_st_32x32b_x16(tP + 16 * h2, pk0);
                    tmem_st_32x32b_x16(tDS + 16 * h2, dk0);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive_warp(bar(kBbPReady));
            FA_TRACE_EV(tslot, 7);
        }
        if (!ok) return;
        // Epilogue: this group's accumulator columns of the row, scaled, in the input dtype.
        FA_TRACE_EV(tslot, 8);
        if (!wait(kBbAccFull, acc_iter & 1u)) return;
        FA_TRACE_EV(tslot, 9);
        ++acc_iter;
        tc_fence_after();
        const uint32_t tAcc = tmem + lane_bits + (KV ? (g ? C::kColAcc1 : C::kColAcc0)
                                                     : C::kColAcc0 + (uint32_t)(g * (D / 2)));
#pragma unroll
        for (int c = 0; c < (KV ? D : D / 2) / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tAcc + 32 * c, o);
            tmem_ld_wait();
            reg_fence<32>(o);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * gmul, __uint_as_float(o[2 * i + 1]) * gmul);
            if (row_in) {
                uint4* dst = reinterpret_cast<uint4*>(grow + gcol0 + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        tc_fence_before();
        mbar_arrive_warp(bar(kBbAccFree));
        FA_TRACE_EV(tslot, 10);
    }
}

// ------------------------------------------------------------------ dK/dV pass in half-steps (D = 128)

template <int D, bool BF16>
__device__ void bwd_mma_halves(const BwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                               const volatile int* ring, volatile int* abort_flag) {
    using C = BCfg<D, true>;
    const uint32_t leader = elect_one_lane();
    constexpr uint32_t kIdescS = make_idesc_f16(BF16, 128, 64, false);   // N = 64 queries
    constexpr uint32_t kIdescAcc = make_idesc_f16(BF16, 128, D, true);
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    // D[128 x 64] = A[128 x D] B[64 x D]^T: B is 64 rows of a 128-row stage tile (its start
    // address moved by 64 rows = 8 KB, a whole number of 1 KB swizzle atoms).
    auto issue_ss64 = [&](uint32_t dcol, uint32_t a, uint32_t b) {
        const uint64_t ad = make_sdesc_sw128(a, 16, 1024);
        const uint64_t bd = make_sdesc_sw128(b, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss_if(leader, tmem + dcol, ad + off, bd + off, kIdescS, kk > 0 ? 1u : 0u);
        }
    };
    // D[128 x D] += A[128 x 64] B[64 x D]: A 16-bit pairs of the half (K step kk: group kk / 2,
    // its columns 8 (kk % 2) ..), B 64 rows of a stage tile, MN-major.
    auto issue_ts64 = [&](uint32_t dcol, uint32_t acol, uint32_t b, bool accumulate) {
        const uint64_t bd = make_sdesc_sw128(b, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t aoff = (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8);
            mma_ts_if(leader, tmem + dcol, tmem + acol + aoff, bd + (uint64_t)((kk * 2048) >> 4), kIdescAcc,
                      (kk > 0 || accumulate) ? 1u : 0u);
        }
    };
    auto stage0 = [&](uint32_t ps) { return sbase + C::kStageOff + (ps % C::kStages) * C::kStageBytes; };
    uint32_t pos = 0, hs = 0, fix_iter = 0, acc_iter = 0, u_iter = 0;
    uint32_t pr_iter[2] = {0u, 0u};
    bool ok = true;
    const uint32_t sFix0 = sbase, sFix1 = sbase + C::kTileBytes;
    // S^T and dP^T of half-step k of the unit (entry pos0 + k / 2, queries 64 (k % 2) ..) into
    // buffer (hs0 + k) % 2.
    auto issue_half = [&](uint32_t pos0, uint32_t hs0, int k) -> bool {
        const uint32_t ps = pos0 + (uint32_t)(k >> 1);
        const int h = k & 1;
        if (h == 0) {
            if (!wait(C::kBarSlotFull + (int)(ps % C::kStages), (ps / C::kStages) & 1u)) return false;
            tc_fence_after();
        }
        const uint32_t b = (hs0 + (uint32_t)k) & 1u;
        const uint32_t st0 = stage0(ps) + 8192u * (uint32_t)h, st1 = st0 + C::kTileBytes;
        issue_ss64(128u * b, sFix0, st0);         // S^T_h = K_j Q_h^T
        issue_ss64(128u * b + 64u, sFix1, st1);   // dP^T_h = V_j dO_h^T
        tc_commit_if(leader, bar(C::kBarSFullH + (int)b));
        return true;
    };
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) break;
        const BUnit un = decode_bunit(p, u);
        if (un.E == 0) continue;
        if (!wait(kBbFixFull, fix_iter & 1u)) { ok = false; break; }
        ++fix_iter;
        tc_fence_after();
        const uint32_t pos0 = pos, hs0 = hs;
        const int K2 = 2 * un.E;
        if (!issue_half(pos0, hs0, 0)) { ok = false; break; }
        for (int k = 0; k < K2; ++k) {
            // The next half's S^T and dP^T first: they overwrite the buffer of half k - 1, whose
            // accumulating MMAs were issued before (one thread's MMAs run in issue order).
            if (k + 1 < K2 && !issue_half(pos0, hs0, k + 1)) { ok = false; break; }
            const uint32_t b = (hs0 + (uint32_t)k) & 1u;
            if (!wait(C::kBarPReadyH + (int)b, pr_iter[b] & 1u)) { ok = false; break; }
            ++pr_iter[b];
            if (k == 0 && !wait(kBbAccFree, (acc_iter & 1u) ^ 1u)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ps = pos0 + (uint32_t)(k >> 1);
            const int h = k & 1;
            const uint32_t st0 = stage0(ps) + 8192u * (uint32_t)h, st1 = st0 + C::kTileBytes;
            issue_ts64(C::kColAcc0, 128u * b, st1, k > 0);         // dV += P^T_h dO_h
            issue_ts64(C::kColAcc1, 128u * b + 64u, st0, k > 0);   // dK += dS^T_h Q_h
            if (h == 1) tc_commit_if(leader, bar(C::kBarSlotEmpty + (int)(ps % C::kStages)));
        }
        if (!ok) break;
        pos += (uint32_t)un.E;
        hs += (uint32_t)K2;
        tc_commit_if(leader, bar(kBbAccFull));
        tc_commit_if(leader, bar(kBbFixEmpty));
        ++acc_iter;
    }
    if (!ok) {
        tc_commit_if(leader, bar(kBbDrain));
        drain_wait(bar(kBbDrain), 0u);
    }
}

template <int D, bool BF16, int VAR>
__device__ void bwd_math_halves(const BwdParams& p, int g, uint32_t sbase, uint32_t bars, uint32_t tmem,
                                const volatile int* ring, volatile int* abort_flag) {
    using C = BCfg<D, true>;
    constexpr int SCORE = VAR & (FA_SCORE_SOFTCAP | FA_SCORE_ALIBI);
    constexpr bool kDoc = (VAR & kVarDocumentB) != 0;
    constexpr bool kSoftcap = (SCORE & FA_SCORE_SOFTCAP) != 0;
    constexpr bool kAlibi = (SCORE & FA_SCORE_ALIBI) != 0;
    const int wq = (threadIdx.x >> 5) & 3;
    const int lane = threadIdx.x & 31;
    const int r = wq * 32 + lane;                       // key row of the tile (TMEM lane)
    const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    uint32_t pos = 0, hs = 0, acc_iter = 0, u_iter = 0;
    uint32_t sf_iter[2] = {0u, 0u};
    bool ok = true;
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) return;
        const BUnit un = decode_bunit(p, u);
        const int kv = un.idx * kBlock + r;
        // Group 0 writes dV, group 1 dK (scaled).
        const bool dk_row = (g == 1);
        const int64_t* gst = dk_row ? p.grad0_stride : p.grad1_stride;
        uint16_t* grow = reinterpret_cast<uint16_t*>(dk_row ? p.grad0 : p.grad1) + un.b * gst[0] +
                         un.h * gst[1] + (int64_t)kv * gst[2];
        const float gmul = dk_row ? p.scale : 1.0f;
        const bool row_in = kv < p.KV_LEN;
        if (un.E == 0) {
            if (row_in) store_zero_cols(grow, D);
            continue;
        }
        const float slope_log2 = kAlibi ? alibi_slope_log2(p, un.h) : 0.f;
        const int row_doc = (kDoc && kv < p.QB * kBlock) ? __ldg(p.doc_id + kv) : 0;
        const int kv_len = p.kv_lens ? min(p.KV_LEN, __ldg(p.kv_lens + (p.maskB == 1 ? 0 : un.b))) : p.KV_LEN;
        EntryReader er;
        er.init(un.entries, un.E);
        for (int e = 0; e < un.E && ok; ++e) {
            const int code = er.get(e);
            int t = code & 0xFFFF;
            FA_DCHECK_INDEX(t, p.entries_stride, p.status);
            const bool full = (code & kFull0) != 0;
            const int s = (int)(pos % C::kStages);
            ++pos;
            const uint8_t* stv = reinterpret_cast<const uint8_t*>(__cvta_shared_to_generic(
                sbase + C::kStageOff + (uint32_t)s * C::kStageBytes + 2 * C::kTileBytes));
            for (int h = 0; h < 2; ++h) {
                const uint32_t b = hs & 1u;
                ++hs;
                if (!wait(C::kBarSFullH + (int)b, sf_iter[b] & 1u)) { ok = false; break; }
                ++sf_iter[b];
                tc_fence_after();
                const uint32_t tS = tmem + lane_bits + 128u * b + 32u * g;
                const uint32_t tDP = tS + 64u;
                uint32_t sr[32], dr[32];
                tmem_ld_32x32b_x32(tS, sr);
                tmem_ld_32x32b_x32(tDP, dr);
                tmem_ld_wait();
                reg_fence<32>(sr);
                reg_fence<32>(dr);
                // Columns: queries q = col0 + c, c in [0, 32).
                const int col0 = t * kBlock + 64 * h + 32 * g;
                int lo = 0, hi = 31;
                if (!full) {
                    if (kv >= kv_len) hi = -1;
                    hi = min(hi, p.Q_LEN - 1 - col0);
                    if (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) lo = max(lo, kv - col0);
                    if (p.mask_kind & FA_MASK_SLIDING_WINDOW) hi = min(hi, kv + p.window - 1 - col0);
                }
                const float* vl = reinterpret_cast<const float*>(stv) + 64 * h + 32 * g;
                const float* vd = vl + kBlock;
                float2 pos2 = make_float2(slope_log2 * (float)(kv - col0), slope_log2 * (float)(kv - col0 - 1));
                PairConsts k;
                k.sc2 = make_float2(p.scale_log2, p.scale_log2);
                k.inv2 = make_float2(p.inv_softcap_scale, p.inv_softcap_scale);
                k.cap2 = make_float2(p.softcap_log2, p.softcap_log2);
                k.step2 = make_float2(-2.f * slope_log2, -2.f * slope_log2);
                k.lo = lo;
                k.hi = hi;
                k.row_doc = row_doc;
                k.doc_cols = kDoc ? p.doc_id + col0 : nullptr;
                auto nl = [&](int i) { return *reinterpret_cast<const float2*>(vl + 2 * i); };
                auto nd = [&](int i) { return *reinterpret_cast<const float2*>(vd + 2 * i); };
                uint32_t pk[16], dk[16];
                if (full) bwd_pairs<BF16, SCORE, kDoc, false>(sr, dr, k, pos2, nl, nd, pk, dk);
                else bwd_pairs<BF16, SCORE, kDoc, true>(sr, dr, k, pos2, nl, nd, pk, dk);
                // Over this group's own S and dP columns of the buffer, already read.
                tmem_st_32x32b_x16(tS, pk);
                tmem_st_32x32b_x16(tDP, dk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive_warp(bar(C::kBarPReadyH + (int)b));
            }
        }
        if (!ok) return;
        if (!wait(kBbAccFull, acc_iter & 1u)) return;
        ++acc_iter;
        tc_fence_after();
        const uint32_t tAcc = tmem + lane_bits + (dk_row ? C::kColAcc1 : C::kColAcc0);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tAcc + 32 * c, o);
            tmem_ld_wait();
            reg_fence<32>(o);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * gmul, __uint_as_float(o[2 * i + 1]) * gmul);
            if (row_in) {
                uint4* dst = reinterpret_cast<uint4*>(grow + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
        tc_fence_before();
        mbar_arrive_warp(bar(kBbAccFree));
    }
}

// ------------------------------------------------------------------ kernels

template <int D, bool BF16, int VAR, bool KV>
__global__ void __launch_bounds__(kThreadsBwd, 1)
attn_bwd_kernel(const __grid_constant__ BwdParams p, const __grid_constant__ CUtensorMap tq,
                const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tdo) {
    using C = BCfg<D, KV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + C::kBarOff;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + C::kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(bars + 8u * kBbFixFull, 1);
        mbar_init(bars + 8u * kBbFixEmpty, 1);
        mbar_init(bars + 8u * kBbSFull, 1);
        mbar_init(bars + 8u * kBbPReady, 8);     // one arrival per math warp
        mbar_init(bars + 8u * kBbAccFull, 1);
        mbar_init(bars + 8u * kBbAccFree, 8);
        mbar_init(bars + 8u * kBbDrain, 1);
        mbar_init(bars + 8u * kBbLoaded, 8);
        mbar_init(bars + 8u * kBbAccDone, 1);
        for (int r = 0; r < kUnitRing; ++r) {
            mbar_init(bars + 8u * (C::kBarUFull + r), 1);
            mbar_init(bars + 8u * (C::kBarUEmpty + r), 9);   // the MMA warp + 8 math warps
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bars + 8u * (C::kBarSlotFull + s), 1);
            mbar_init(bars + 8u * (C::kBarSlotEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars + 8u * (C::kBarSFullH + b), 1);
            mbar_init(bars + 8u * (C::kBarPReadyH + b), 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp < 4) {
        regs_dec<kRegsIssueBwd>();
        if (warp == 0) {
            bwd_producer<D, KV>(p, &tq, &tk, &tv, &tdo, sbase, bars, ring, abort_flag);
        } else if (warp == 1) {
            if constexpr (C::kHalves) bwd_mma_halves<D, BF16>(p, sbase, bars, tmem, ring, abort_flag);
            else bwd_mma<D, BF16, KV>(p, sbase, bars, tmem, ring, abort_flag);
        }
    } else {
        regs_inc<kRegsMathBwd>();
        if constexpr (C::kHalves) bwd_math_halves<D, BF16, VAR>(p, (warp - 4) >> 2, sbase, bars, tmem, ring, abort_flag);
        else bwd_math<D, BF16, VAR, KV>(p, (warp - 4) >> 2, sbase, bars, tmem, ring, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tmem, 512);
}

template <int D, bool BF16, int VAR, bool KV>
cudaError_t launch_bwd_t(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, const CUtensorMap& tdo, int grid, cudaStream_t stream) {
    auto kern = attn_bwd_kernel<D, BF16, VAR, KV>;
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    if (attr.numRegs < kRegsAtLaunchBwd) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg<D, KV>::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreadsBwd, BCfg<D, KV>::kSmemBytes, stream>>>(p, tq, tk, tv, tdo);
    return cudaGetLastError();
}

template <bool KV>
cudaError_t launch_bwd_any(const BwdParams& p, int D, bool bf16, int score_kind, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                           int grid, cudaStream_t stream) {
    const int var = score_kind | ((p.mask_kind & FA_MASK_DOCUMENT) ? kVarDocumentB : 0);
#define FA_BCASE(DD, BB, VV)                                                 \
    if (D == DD && bf16 == BB && var == VV)                                  \
        return launch_bwd_t<DD, BB, VV, KV>(p, tq, tk, tv, tdo, grid, stream);
#define FA_BCASES(DD, BB) FA_BCASE(DD, BB, 0) FA_BCASE(DD, BB, 1) FA_BCASE(DD, BB, 2) FA_BCASE(DD, BB, 3) \
    FA_BCASE(DD, BB, 4) FA_BCASE(DD, BB, 5) FA_BCASE(DD, BB, 6) FA_BCASE(DD, BB, 7)
    FA_BCASES(64, true)
    FA_BCASES(64, false)
    FA_BCASES(128, true)
    FA_BCASES(128, false)
#undef FA_BCASES
#undef FA_BCASE
    return cudaErrorInvalidValue;
}

// Delta = rowsum(dO * O) and lse * log2(e) per query row, padded to q_pad rows per (b, h).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(
    const uint16_t* __restrict__ out, int64_t os0, int64_t os1, int64_t os2,
    const uint16_t* __restrict__ dout, int64_t ds0, int64_t ds1, int64_t ds2,
    const float* __restrict__ lse, int B, int H, int Q_LEN, int q_pad, float* __restrict__ neg_lse_log2,
    float* __restrict__ neg_delta) {
    constexpr int kLanesPerRow = D / 8;          // one 16-byte vector per lane
    constexpr int kRowsPerWarp = 32 / kLanesPerRow;
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t row = gw * kRowsPerWarp + lane / kLanesPerRow;
    const int sub = lane % kLanesPerRow;
    const int64_t total = (int64_t)B * H * q_pad;
    float acc = 0.f;
    int64_t bh = 0, q = 0;
    if (row < total) {
        bh = row / q_pad;
        q = row - bh * q_pad;
        if (q < Q_LEN) {
            const int64_t b = bh / H, h = bh - b * H;
            const uint4 ov = *reinterpret_cast<const uint4*>(out + b * os0 + h * os1 + q * os2 + sub * 8);
            const uint4 dv = *reinterpret_cast<const uint4*>(dout + b * ds0 + h * ds1 + q * ds2 + sub * 8);
            const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t ob = (ow[i] >> (16 * k)) & 0xFFFFu, db = (dw[i] >> (16 * k)) & 0xFFFFu;
                    float o, d;
                    if constexpr (BF16) {
                        o = __uint_as_float(ob << 16);
                        d = __uint_as_float(db << 16);
                    } else {
                        o = __half2float(__ushort_as_half((unsigned short)ob));
                        d = __half2float(__ushort_as_half((unsigned short)db));
                    }
                    acc = fmaf(o, d, acc);
                }
            }
        }
    }
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(kFullMask, acc, o);
    if (row < total && sub == 0) {
        // Stored negated, so the main kernels add them (P = 2^(x + neg_lse_log2) and
        // dP + neg_delta) with no negation per element.
        neg_delta[row] = (q < Q_LEN) ? -acc : 0.f;
        const float l = (q < Q_LEN) ? lse[bh * Q_LEN + q] : -INFINITY;
        neg_lse_log2[row] = (l == -INFINITY) ? -INFINITY : -(l * kLog2e);
    }
}

}  // namespace

cudaError_t launch_bwd_preprocess(const void* out, const int64_t out_stride[3], const void* dout,
                                  const int64_t dout_stride[3], const float* lse, int B, int H,
                                  int Q_LEN, int q_pad, int D, bool bf16, float* neg_lse_log2,
                                  float* neg_delta, cudaStream_t stream) {
    const int64_t rows = (int64_t)B * H * q_pad;
    const int rows_per_warp = 32 / (D / 8);
    const int64_t warps = (rows + rows_per_warp - 1) / rows_per_warp;
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    const uint16_t* o = static_cast<const uint16_t*>(out);
    const uint16_t* d = static_cast<const uint16_t*>(dout);
#define FA_PRE(DD, BB)                                                                              \
    if (D == DD && bf16 == BB) {                                                                    \
        bwd_preprocess_kernel<DD, BB><<<(unsigned)blocks, 256, 0, stream>>>(                        \
            o, out_stride[0], out_stride[1], out_stride[2], d, dout_stride[0], dout_stride[1],      \
            dout_stride[2], lse, B, H, Q_LEN, q_pad, neg_lse_log2, neg_delta);                              \
        return cudaGetLastError();                                                                  \
    }
    FA_PRE(64, true)
    FA_PRE(64, false)
    FA_PRE(128, true)
    FA_PRE(128, false)
#undef FA_PRE
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_dkdv(const BwdParams& p, int D, bool bf16, int score_kind,
                                 const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const CUtensorMap& tdo, int grid, cudaStream_t stream) {
    return launch_bwd_any<true>(p, D, bf16, score_kind, tq, tk, tv, tdo, grid, stream);
}

cudaError_t launch_attn_bwd_dq(const BwdParams& p, int D, bool bf16, int score_kind,
                               const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tdo, int grid, cudaStream_t stream) {
    return launch_bwd_any<false>(p, D, bf16, score_kind, tq, tk, tv, tdo, grid, stream);
}

}  // namespace fa
