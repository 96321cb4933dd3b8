// attn_fwd.cu -- fused block-sparse attention forward for sm_100a.
//
// What it computes ("How to Use FlexAttention on Apple Silicon", "The two hooks" and
// "Bonus: a score_mod for soft-capping"):
//   O = softmax(mask(score_mod(scale * Q K^T))) V,  lse = log-sum-exp per query row,
// visiting only the tiles a block mask lists, evaluating the mask only on partial
// tiles and never writing the score matrix to memory.
//
// Organisation (one persistent CTA per SM, 12 warps):
//   warp 0      TMA producer (fwd_common.cuh): takes the next unit from the global counter,
//               publishes it to the other roles through a shared-memory ring, then loads
//               the unit's Q tiles and K_j, V_j of every listed kv block into a ring of
//               shared-memory stages (128-byte swizzle).
//   warp 1      MMA issuer (one elected lane): S_t = Q_t K_j^T into TMEM (SS MMA), and
//               O_t += P_t V_j with P_t read from TMEM (TS MMA); at D = 64 for tile 0 only,
//               at D = 128 for both tiles.
//   warp 2      TMEM allocation / release.
//   warp 3      at D = 64 the MMA issuer of tile 1; idle at D = 128 (completes the warpgroup).
//   warps 4-7   softmax for query tile 0 (one thread per query row = TMEM lane),
//   warps 8-11  softmax for query tile 1.
// A work unit is a pair of adjacent query blocks (2p, 2p+1) of one (b, h); both tiles
// share every K/V load of the merged kv-block list.  At D = 128 one MMA warp serves tile 0,
// then tile 1, for every entry; that fixed order keeps the two softmax groups about half a
// tile apart, so one group's exponentials run while the other waits for its next S.  At
// D = 64 each tile has its own MMA warp, whose stream waits only on that tile's softmax.
//
// TMEM (512 columns x 128 lanes, fp32):
//   D = 64:  S0 at 0, S1 at 128, P0 at 256, P1 at 320 (16-bit pairs), O0 at 384, O1 at 448;
//            the next S_t may be computed while P_t is still being written (S_free).
//   D = 128: S0 at 0, S1 at 128, O0 at 256, O1 at 384; P_t overwrites the first 64
//            columns of S_t, so P.V of an entry is issued before the next S_t.
//
// Softmax: running max in log2 units with a lazy rescale -- O and the row sum are
// rescaled only when the max grows by more than 8 (a factor 256), which keeps P <= 256
// and is exact because the final division uses the same stale max.  The score_mod kind
// and the presence of a document predicate are template parameters.  All waits are
// bounded; a wait that runs out sets the status word and every role unwinds.
#include <cfloat>

#include "fa_internal.h"
#include "fa_trace.cuh"
#include "sm100_ptx.cuh"
#include "fwd_common.cuh"

#ifdef FA_TRACE
extern "C" int fa_debug_set_trace_buffer(void* device_ptr) {
    return (int)cudaMemcpyToSymbol(g_fa_trace, &device_ptr, sizeof(device_ptr));
}
#endif

namespace fa {
namespace {

constexpr int kThreadsFwd = 384;
// Register budgets (setmaxnreg): the launch gives every thread 65536 / 384 rounded down to a
// multiple of 8 = 168; the TMA/MMA warpgroup drops to 104 (at 80 its issue loops spill) and
// the two softmax warpgroups rise to 200: exactly the launched pool.
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsProducer = 104;
constexpr int kRegsSoftmax = 200;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreadsFwd * kRegsAtLaunch,
              "register split exceeds the launched pool");

// Barrier slots (kBarQFull = 0 and kBarQEmpty = 1 come with the producer).
enum : int {
    kBarSFull = 2,    // + tile
    kBarPFull = 4,    // + tile
    kBarOFull = 6,    // + tile
    kBarOFree = 8,    // + tile
    kBarSFree = 10,   // + tile: softmax has S in registers (separate-P layout only)
    kBarPVDone = 12,  // + tile: the tile's last P.V has completed (separate-P layout only)
    kBarDrain = 14,     // + tile
    kBarUnitFull = 16,  // + unit-ring slot (2)
    kBarUnitEmpty = 18, // + unit-ring slot (2)
    kBarSlotBase = 20   // + stage, then slot-empty barriers follow
};

template <int D>
struct Cfg {
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kStages = (D == 64) ? 8 : 4;
    static constexpr int kChunks = D / 64;               // 128-byte-wide TMA boxes per row
    static constexpr int kBarUFull = kBarUnitFull;
    static constexpr int kBarUEmpty = kBarUnitEmpty;
    static constexpr int kBarSlotFull = kBarSlotBase;
    static constexpr int kBarSlotEmpty = kBarSlotFull + kStages;
    static constexpr int kNumBars = kBarSlotEmpty + kStages;
    static constexpr int kBarOff = (2 + kStages) * kTileBytes;
    // After the barriers: TMEM address, abort flag, the two unit-ring slots.
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 32 + 1024;  // + alignment slack
    // TMEM columns.  At D = 64 everything fits apart: S0 S1 (128 each), P0 P1 (64 each),
    // O0 O1 (64 each) = 512, so the next Q K^T can overwrite S while P is still being
    // computed.  At D = 128, P_t is written over the first 64 columns of S_t.
    static constexpr bool kSepP = (D == 64);
    // MMA warps: one per query tile with separate P (warps 1 and 3), else warp 1 for both.
    static constexpr int kMmaWarps = kSepP ? 2 : 1;
    // Pairs (of every 16) whose 2^x runs on the FMA pipe in full tiles, to take load off the
    // MUFU unit; worth it only when a score_mod already spends MUFU time (tanh), per
    // measurement (32k soft-cap + ALiBi, with 4 to 6 of 16 tanh pairs on the FMA pipe: 0 of 16
    // 874-877, 1 891-902, 2 886-887 TFLOP/s; 8k causal without a score_mod: 0 674, 1 655,
    // 2 665, 4 648).
    static constexpr int emu_pairs(int score) { return score != 0 ? 1 : 0; }
    __device__ static constexpr uint32_t colS(int t) { return (uint32_t)t * 128u; }
    __device__ static constexpr uint32_t colP(int t) {
        return kSepP ? 256u + (uint32_t)t * 64u : (uint32_t)t * 128u;
    }
    __device__ static constexpr uint32_t colO(int t) {
        return kSepP ? 384u + (uint32_t)t * 64u : 256u + (uint32_t)t * (uint32_t)D;
    }
};

// ------------------------------------------------------------------ MMA issuers (warps 1, 3)

// The tensor-core work of one query tile t, issued by the elected lane of the calling warp.
template <int D, bool BF16>
struct TileMma {
    using C = Cfg<D>;
    uint32_t leader, sQ, sKV, tmem;
    // S_t = Q_t K^T: M = 128 query rows, N = 128 keys, K = D in steps of 16.  Both
    // operands are K-major with 128-byte swizzle: 8-row atoms 1024 bytes apart (SBO),
    // a step of 16 elements is 32 bytes inside the atom, and columns 64.. live in the
    // next 16 KB box.
    __device__ __forceinline__ void qk(int t, int slot) const {
        constexpr uint32_t kIdescQK = make_idesc_f16(BF16, 128, 128, false);
        const uint32_t d = tmem + C::colS(t);
        const uint64_t qd = make_sdesc_sw128(sQ + t * C::kTileBytes, 16, 1024);
        const uint64_t kd = make_sdesc_sw128(sKV + slot * C::kTileBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            // Start-address field counts 16-byte units: add the byte offset >> 4.
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss_if(leader, d, qd + off, kd + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
    }
    // O_t += P_t V: M = 128, N = D, K = 128 keys in steps of 16.  P_t comes from TMEM
    // (8 columns of packed pairs per step).  V is MN-major (D contiguous): 16 keys are
    // two 8-row atoms (SBO = 1024 bytes), 64-column boxes 16 KB apart (LBO).
    __device__ __forceinline__ void pv(int t, int slot, bool accumulate) const {
        constexpr uint32_t kIdescPV = make_idesc_f16(BF16, 128, D, true);
        const uint32_t d = tmem + C::colO(t);
        const uint32_t pa = tmem + C::colP(t);
        const uint64_t vd = make_sdesc_sw128(sKV + slot * C::kTileBytes, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk) {
            mma_ts_if(leader, d, pa + (uint32_t)(kk * 8), vd + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                      (kk > 0 || accumulate) ? 1u : 0u);
        }
    }
};

// MMA issuer of one query tile t (the D = 64 layout, S and P apart in TMEM): warp 1 serves
// tile 0 and warp 3 tile 1, so each tile's stream waits only on its own softmax group and the
// issue work is split between two SM sub-partitions (686 -> 700 TFLOP/s at 8k causal).  Both
// warps commit to each stage-empty and Q-empty barrier.
template <int D, bool BF16>
__device__ void mma_role_tile(const FwdParams& p, int t, uint32_t sbase, uint32_t bars, uint32_t tmem,
                              const volatile int* ring, volatile int* abort_flag) {
    using C = Cfg<D>;
    static_assert(C::kSepP, "one MMA warp per tile needs S and P apart");
    TileMma<D, BF16> mma;
    mma.leader = elect_one_lane();
    mma.sQ = sbase;
    mma.sKV = sbase + 2 * C::kTileBytes;
    mma.tmem = tmem;
    const uint32_t leader = mma.leader;
    const int live = t ? kLive1 : kLive0;
    const int tslot = t ? 10 : 1;   // trace slot of this warp
    (void)tslot;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    uint32_t kv_pos = 0, q_iter = 0, pf_cnt = 0, of_cnt = 0, qk_cnt = 0;
    bool ok = true;
    FA_TRACE_DECL
    // S_t = Q_t K^T into TMEM once the softmax holds the previous S_t in registers.
    auto do_qk = [&](int slot) -> bool {
        if (!wait(kBarSFree + t, (qk_cnt & 1u) ^ 1u)) return false;
        tc_fence_after();
        ++qk_cnt;
        mma.qk(t, slot);
        tc_commit_if(leader, bar(kBarSFull + t));
        return true;
    };
    // Stage of ring position pos, and the wait for its TMA load; K of entry e sits at
    // kbase + 2e and V of entry e right after it.
    auto stage = [&](uint32_t pos) { return (int)(pos % C::kStages); };
    auto wait_pos = [&](uint32_t pos) {
        return wait(C::kBarSlotFull + stage(pos), (pos / C::kStages) & 1u);
    };
    uint32_t u_iter = 0;
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) break;
        const Unit un = decode_unit(p, u);
        if (un.E == 0) continue;
        const int nl = t ? un.nl1 : un.nl0;
        if (!wait(kBarQFull, q_iter & 1u)) { ok = false; break; }
        ++q_iter;
        tc_fence_after();
        const uint32_t kbase = kv_pos;
        kv_pos += 2u * (uint32_t)un.E;
        int ndone = 0;
        // O_t += P_t V once the softmax has published P_t.
        auto do_pv = [&](int slot) -> bool {
            FA_TRACE_EV(tslot, 16 + t);
            if (!wait(kBarPFull + t, pf_cnt & 1u)) return false;
            FA_TRACE_EV(tslot, 18 + t);
            ++pf_cnt;
            if (ndone == 0 && !wait(kBarOFree + t, (of_cnt & 1u) ^ 1u)) return false;
            tc_fence_after();
            mma.pv(t, slot, ndone > 0);
            tc_commit_if(leader, bar(kBarPVDone + t));
            if (ndone + 1 == nl) tc_commit_if(leader, bar(kBarOFull + t));
            ++ndone;
            return true;
        };
        EntryReader er;
        er.init(un.entries, un.E);
        int code = er.get(0);
        {   // S for entry 0
            if (!wait_pos(kbase)) { ok = false; break; }
            tc_fence_after();
            if (code & live) ok = do_qk(stage(kbase));
            if (!ok) break;
            tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(kbase)));
            if (un.E == 1) tc_commit_if(leader, bar(kBarQEmpty));
        }
        for (int e = 0; e < un.E; ++e) {
            const bool has_next = e + 1 < un.E;
            const int next = has_next ? er.get(e + 1) : 0;
            const uint32_t vpos = kbase + 2u * (uint32_t)e + 1u, kpos = vpos + 1u;
            FA_TRACE_EV(tslot, 22);
            if (!wait_pos(vpos)) { ok = false; break; }
            if (has_next && !wait_pos(kpos)) { ok = false; break; }
            FA_TRACE_EV(tslot, 23);
            tc_fence_after();
            // The next S first (it only needs the softmax to hold the current S), then P.V of
            // the current entry.
            if (next & live) ok = do_qk(stage(kpos));
            if (ok && (code & live)) ok = do_pv(stage(vpos));
            if (!ok) break;
            tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(vpos)));
            if (has_next) {
                tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(kpos)));
                if (e + 2 == un.E) tc_commit_if(leader, bar(kBarQEmpty));
            }
            code = next;
        }
        if (!ok) break;
        if (nl > 0) ++of_cnt;
    }
    if (!ok) {
        // Wait for every MMA this warp issued before the CTA can release TMEM.
        tc_commit_if(leader, bar(kBarDrain + t));
        drain_wait(bar(kBarDrain + t), 0u);
    }
}

// MMA issuer of both query tiles (the D = 128 layout, P over S), warp 1: tile 0 then tile 1 for
// every entry, P.V of the current entry before the next Q K^T (which overwrites P).  The fixed
// order keeps the two softmax groups half a period apart; with one warp per tile they drift
// into step (854 -> 718 TFLOP/s at 32k soft-cap, 718 -> 672 sliding window).
template <int D, bool BF16>
__device__ void mma_role_pair(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                              const volatile int* ring, volatile int* abort_flag) {
    using C = Cfg<D>;
    static_assert(!C::kSepP, "the paired issuer is for P over S");
    TileMma<D, BF16> mma;
    mma.leader = elect_one_lane();
    mma.sQ = sbase;
    mma.sKV = sbase + 2 * C::kTileBytes;
    mma.tmem = tmem;
    const uint32_t leader = mma.leader;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    uint32_t kv_pos = 0, q_iter = 0;
    uint32_t pf_cnt[2] = {0u, 0u}, of_cnt[2] = {0u, 0u};
    bool ok = true;
    FA_TRACE_DECL
    auto do_qk = [&](int t, int slot) {
        mma.qk(t, slot);
        tc_commit_if(leader, bar(kBarSFull + t));
    };
    auto stage = [&](uint32_t pos) { return (int)(pos % C::kStages); };
    auto wait_pos = [&](uint32_t pos) {
        return wait(C::kBarSlotFull + stage(pos), (pos / C::kStages) & 1u);
    };
    uint32_t u_iter = 0;
    for (;;) {
        const int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, ok);
        if (u < 0) break;
        const Unit un = decode_unit(p, u);
        if (un.E == 0) continue;
        const int nl[2] = {un.nl0, un.nl1};
        if (!wait(kBarQFull, q_iter & 1u)) { ok = false; break; }
        ++q_iter;
        tc_fence_after();
        const uint32_t kbase = kv_pos;
        kv_pos += 2u * (uint32_t)un.E;
        int ndone[2] = {0, 0};
        // O_t += P_t V once the softmax has published P_t.
        auto do_pv = [&](int t, int slot) -> bool {
            FA_TRACE_EV(1, 16 + t);
            if (!wait(kBarPFull + t, pf_cnt[t] & 1u)) return false;
            FA_TRACE_EV(1, 18 + t);
            ++pf_cnt[t];
            if (ndone[t] == 0 && !wait(kBarOFree + t, (of_cnt[t] & 1u) ^ 1u)) return false;
            tc_fence_after();
            mma.pv(t, slot, ndone[t] > 0);
            if (ndone[t] + 1 == nl[t]) tc_commit_if(leader, bar(kBarOFull + t));
            ++ndone[t];
            return true;
        };
        EntryReader er;
        er.init(un.entries, un.E);
        int code = er.get(0);
        {   // S for entry 0
            if (!wait_pos(kbase)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t)
                if (code & (t ? kLive1 : kLive0)) do_qk(t, stage(kbase));
            tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(kbase)));
            if (un.E == 1) tc_commit_if(leader, bar(kBarQEmpty));
        }
        for (int e = 0; e < un.E; ++e) {
            const bool has_next = e + 1 < un.E;
            const int next = has_next ? er.get(e + 1) : 0;
            const uint32_t vpos = kbase + 2u * (uint32_t)e + 1u, kpos = vpos + 1u;
            FA_TRACE_EV(1, 22);
            if (!wait_pos(vpos)) { ok = false; break; }
            if (has_next && !wait_pos(kpos)) { ok = false; break; }
            FA_TRACE_EV(1, 23);
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (ok && (code & (t ? kLive1 : kLive0))) ok = do_pv(t, stage(vpos));
                if (ok && (next & (t ? kLive1 : kLive0))) do_qk(t, stage(kpos));
            }
            if (!ok) break;
            tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(vpos)));
            if (has_next) {
                tc_commit_if(leader, bar(C::kBarSlotEmpty + stage(kpos)));
                if (e + 2 == un.E) tc_commit_if(leader, bar(kBarQEmpty));
            }
            code = next;
        }
        if (!ok) break;
#pragma unroll
        for (int t = 0; t < 2; ++t)
            if (nl[t] > 0) ++of_cnt[t];
    }
    if (!ok) {
        // Wait for every MMA already issued before the CTA can release TMEM.
        tc_commit_if(leader, bar(kBarDrain));
        drain_wait(bar(kBarDrain), 0u);
    }
}

// ------------------------------------------------------------------ softmax (warps 4-11)

// P = 2^(x - base) for one 128-wide row, packed to 16-bit pairs and stored to TMEM at tP
// in four 32-column chunks; returns the (two-lane) row sum.  EMU of every 16 pairs use
// the FMA-pipe exp2 (only for tiles without masked positions), the rest MUFU ex2.
// A warp issues in program order, so all 128 exponentials come first (overwriting x) and the
// sums, packing and TMEM stores after them: the MUFU unit then gets one instruction per
// issue opportunity instead of waiting at every chunk for the previous chunk's dependent work.
template <bool BF16, bool SCORE, int EMU>
__device__ __forceinline__ float2 softmax_p_row(float2 (&x)[64], float2 nb2, float2 k2, uint32_t tP) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float2 a = SCORE ? __fadd2_rn(x[i], nb2) : __ffma2_rn(x[i], k2, nb2);
        if (((i & 15) * EMU) % 16 < EMU) {
            x[i] = exp2_fma2(a);
        } else {
            x[i] = make_float2(ex2_approx(a.x), ex2_approx(a.y));
        }
    }
    float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};
#pragma unroll
    for (int chunk = 0; chunk < 4; ++chunk) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float2 pe = x[chunk * 16 + i];
            rs[i & 3] = __fadd2_rn(rs[i & 3], pe);
            pk[i] = pack2<BF16>(pe.x, pe.y);
        }
        tmem_st_32x32b_x16(tP + chunk * 16, pk);
    }
    return __fadd2_rn(__fadd2_rn(rs[0], rs[1]), __fadd2_rn(rs[2], rs[3]));
}

// VAR = score_mod bits (FA_SCORE_*) | kVarDocument when the mask has a document predicate
// | kVarFixedMax for the fixed-max soft-cap variant: all compile-time, so kernels without them
// carry none of their registers.
constexpr int kVarDocument = 4;
// Fixed max (bf16 with a soft-cap, every live score <= cap): P = 2^(x - cap log2 e) <= 1 with no
// row max and no rescale.  Without ALiBi every live score is >= -cap; with it the bias must not
// be positive (causal-type masks, the default positive slopes) and each query row keeps its
// own key, whose bias is 0.  Either way a row's sum is >= e^(-2 cap), a normal float32 and
// bfloat16 value for caps up to 32 (e^-60 at cap 30), and a key the fixed base drives below
// the float range weighs less than 2^-39 of that row's largest term.
constexpr int kVarFixedMax = 8;
// Largest |s / cap| for which the soft-cap's tanh is taken from its Taylor polynomial.
constexpr float kTanhPolyBound = 0.2f;
// Pairs (of every 16) whose tanh comes from the polynomial when the bound holds; the rest stay
// on the MUFU unit, which balances the two pipes (a polynomial pair costs the FMA pipe about as
// long as a tanh.approx pair costs the MUFU).  Measured at 32k soft-cap + ALiBi with one exp2
// pair on the FMA pipe: 0 of 16 855, 4 891, 5 900, 6 895 TFLOP/s; all 16 (and two exp2 pairs)
// 832.
constexpr int kTanhPolyPairs = 5;

template <int D, bool BF16, int VAR>
__device__ void softmax_role(const FwdParams& p, int t, uint32_t bars, uint32_t tmem,
                             const volatile int* ring, volatile int* abort_flag) {
    using C = Cfg<D>;
    constexpr int SCORE = VAR & (FA_SCORE_SOFTCAP | FA_SCORE_ALIBI);
    constexpr bool kDoc = (VAR & kVarDocument) != 0;
    constexpr bool kFixedMax = (VAR & kVarFixedMax) != 0;
    static_assert(!kFixedMax || (SCORE & FA_SCORE_SOFTCAP), "fixed max needs the soft-cap bound");
    const int wq = (threadIdx.x >> 5) & 3;  // TMEM lane quadrant this warp may access
    const int lane = threadIdx.x & 31;
    const int row = wq * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_bits + C::colS(t);
    const uint32_t tP = tmem + lane_bits + C::colP(t);
    const uint32_t tO = tmem + lane_bits + C::colO(t);
    const int live_bit = t ? kLive1 : kLive0;
    const int full_bit = t ? kFull1 : kFull0;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
    auto wait = [&](int i, uint32_t par) {
        return mbar_wait_bounded(bar(i), par, abort_flag, p.status, kWaitLimitNs);
    };
    constexpr bool has_softcap = (SCORE & FA_SCORE_SOFTCAP) != 0;
    constexpr bool has_alibi = (SCORE & FA_SCORE_ALIBI) != 0;

    uint32_t sf_cnt = 0, of_cnt = 0, pst_cnt = 0;
    const int tslot = 2 + (int)(threadIdx.x >> 5) - 4;  // one trace slot per softmax warp
    FA_TRACE_DECL
    (void)tslot;
    uint32_t u_iter = 0;
    bool taken = true;
    // The next unit is taken before this unit's epilogue waits for O, so the ring handshake
    // overlaps the last P.V instead of following it.
    int u = take_unit<C>(p, bars, ring, u_iter, abort_flag, taken);
    for (;;) {
        if (u < 0) return;
        const Unit un = decode_unit(p, u);
        const int qblk = 2 * un.pair + t;
        const int nl = t ? un.nl1 : un.nl0;
        if (qblk >= p.QB || nl == 0) {
            if (qblk < p.QB) store_row_zero<D, BF16>(p, un, qblk * kBlock + row);
            u = take_unit<C>(p, bars, ring, u_iter, abort_flag, taken);
            continue;
        }
        const int q = qblk * kBlock + row;
        const int kv_len = p.kv_lens ? min(p.KV_LEN, __ldg(p.kv_lens + (p.maskB == 1 ? 0 : un.b))) : p.KV_LEN;
        float slope_log2 = 0.f;
        if constexpr (has_alibi) {
            float slope;
            if (p.alibi_slopes) {
                slope = __ldg(p.alibi_slopes + un.h);
            } else {
                const int num = 8 * (un.h + 1);
                slope = (num % p.H == 0) ? ldexpf(1.0f, -(num / p.H))
                                         : exp2f(-(float)num / (float)p.H);
            }
            slope_log2 = slope * kLog2e;
        }
        float m = -INFINITY;  // running max, log2 units
        float l = 0.f;        // running row sum of P
        int done = 0;
        EntryReader er;
        er.init(un.entries, un.E);
        bool ok = true;
        for (int e = 0; e < un.E; ++e) {
            const int code = er.get(e);
            if (!(code & live_bit)) continue;
            int j = code & 0xFFFF;
            FA_DCHECK_INDEX(j, p.KVB, p.status);
            const bool full = (code & full_bit) != 0;
            FA_TRACE_EV(tslot, 1);
            if (!wait(kBarSFull + t, sf_cnt & 1u)) { ok = false; break; }
            FA_TRACE_EV(tslot, 2);
            ++sf_cnt;
            tc_fence_after();
            // S row of this thread: 128 fp32 scores held as 64 pairs.
            float2 x[64];
            {
                uint32_t sr[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + c * 32, sr[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c) reg_fence<32>(sr[c]);
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    x[i] = make_float2(__uint_as_float(sr[i >> 4][(2 * i) & 31]),
                                       __uint_as_float(sr[i >> 4][(2 * i + 1) & 31]));
            }
            if constexpr (C::kSepP) {
                // S is in registers: the next Q K^T may overwrite it.
                tc_fence_before();
                mbar_arrive_warp(bar(kBarSFree + t));
            }
            FA_TRACE_EV(tslot, 3);
            const int kv0 = j * kBlock;
            if constexpr (SCORE != 0) {
                // score_mod on every position of the tile, in log2 units; masked
                // positions are set to -inf afterwards (the mask decides liveness).
                const float2 inv2 = make_float2(p.inv_softcap_scale, p.inv_softcap_scale);
                const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
                const float2 sl2 = make_float2(slope_log2, slope_log2);
                const float2 two = make_float2(2.f, 2.f);
                float2 pos = make_float2((float)(kv0 - q), (float)(kv0 - q + 1));
                auto bias = [&](float2 y) {
                    if constexpr (has_alibi) {
                        y = __ffma2_rn(sl2, pos, y);
                        pos = __fadd2_rn(pos, two);
                    }
                    return y;
                };
                if constexpr (has_softcap) {
                    // cap tanh(s / cap).  If every |s / cap| of this warp's rows in the tile is
                    // at most kTanhPolyBound, kTanhPolyPairs of every 16 pairs take tanh from its
                    // odd Taylor polynomial through a^7 on the FMA pipe (the series alternates,
                    // so the error is below the first omitted term, 62/2835 a^9: under 6e-8 of
                    // tanh there) and the rest from the MUFU's tanh.approx; otherwise all of
                    // them from tanh.approx.  The cap (log2 units) is folded into the
                    // coefficients.
                    float am0 = 0.f, am1 = 0.f;
#pragma unroll
                    for (int i = 0; i < 64; i += 2) {
                        am0 = max3(am0, fabsf(x[i].x), fabsf(x[i].y));
                        am1 = max3(am1, fabsf(x[i + 1].x), fabsf(x[i + 1].y));
                    }
                    const bool poly = __all_sync(kFullMask, fmaxf(am0, am1) * fabsf(p.inv_softcap_scale) <=
                                                                kTanhPolyBound);
                    const float cap = p.softcap_log2;
                    if (poly) {
                        const float2 k1 = make_float2(cap, cap);
                        const float2 k3 = make_float2(cap * (-1.0f / 3.0f), cap * (-1.0f / 3.0f));
                        const float2 k5 = make_float2(cap * (2.0f / 15.0f), cap * (2.0f / 15.0f));
                        const float2 k7 = make_float2(cap * (-17.0f / 315.0f), cap * (-17.0f / 315.0f));
#pragma unroll
                        for (int i = 0; i < 64; ++i) {
                            const float2 a = __fmul2_rn(x[i], inv2);
                            if ((i & 15) < kTanhPolyPairs) {
                                const float2 a2 = __fmul2_rn(a, a);
                                float2 t = __ffma2_rn(k7, a2, k5);
                                t = __ffma2_rn(t, a2, k3);
                                t = __ffma2_rn(t, a2, k1);
                                x[i] = bias(__fmul2_rn(a, t));
                            } else {
                                x[i] = bias(__fmul2_rn(k1, make_float2(tanh_approx(a.x), tanh_approx(a.y))));
                            }
                        }
                    } else {
                        const float2 cap2 = make_float2(cap, cap);
#pragma unroll
                        for (int i = 0; i < 64; ++i) {
                            const float2 a = __fmul2_rn(x[i], inv2);
                            x[i] = bias(__fmul2_rn(cap2, make_float2(tanh_approx(a.x), tanh_approx(a.y))));
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = bias(__fmul2_rn(x[i], sc2));
                }
            }
            if (!full) {
                // Keys past the context (a ragged last kv tile, zero-filled by TMA, or this
                // batch's own length) are masked.
                int lo = 0, hi = min(kBlock - 1, kv_len - 1 - kv0);
                if (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) hi = min(hi, q - kv0);
                if (p.mask_kind & FA_MASK_SLIDING_WINDOW) lo = max(lo, q - p.window + 1 - kv0);
                if constexpr (kDoc) {
                    const int dq = __ldg(p.doc_id + q);
                    const int4* dk = reinterpret_cast<const int4*>(p.doc_id + kv0);
#pragma unroll
                    for (int c4 = 0; c4 < 32; ++c4) {
                        const int4 d4 = __ldg(dk + c4);
                        const int c = 4 * c4;
                        if (!(c + 0 >= lo && c + 0 <= hi && d4.x == dq)) x[2 * c4].x = -INFINITY;
                        if (!(c + 1 >= lo && c + 1 <= hi && d4.y == dq)) x[2 * c4].y = -INFINITY;
                        if (!(c + 2 >= lo && c + 2 <= hi && d4.z == dq)) x[2 * c4 + 1].x = -INFINITY;
                        if (!(c + 3 >= lo && c + 3 <= hi && d4.w == dq)) x[2 * c4 + 1].y = -INFINITY;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        if (2 * i < lo || 2 * i > hi) x[i].x = -INFINITY;
                        if (2 * i + 1 < lo || 2 * i + 1 > hi) x[i].y = -INFINITY;
                    }
                }
            }
            bool any_need = false;
            float alpha = 1.0f;
            if constexpr (kFixedMax) {
                m = p.softcap_log2;          // the bound of every live score
            } else {
                // Row max with three-input max: eight independent chains over eighths.
                float mc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mc[c] = fmaxf(x[8 * c].x, x[8 * c].y);
#pragma unroll
                for (int i = 1; i < 8; ++i)
#pragma unroll
                    for (int c = 0; c < 8; ++c) mc[c] = max3(mc[c], x[8 * c + i].x, x[8 * c + i].y);
#pragma unroll
                for (int c = 0; c < 4; ++c) mc[c] = fmaxf(mc[c], mc[c + 4]);
                float mt = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
                if constexpr (SCORE == 0) mt *= p.scale_log2;
                const float m_new = fmaxf(m, mt);
                FA_TRACE_EV(tslot, 4);
                const bool need = m_new > m + kRescaleThreshold;
                any_need = __any_sync(kFullMask, need);
                if (need) {
                    alpha = ex2_approx(m - m_new);  // m = -inf gives 0 (l and O are empty then)
                    m = m_new;
                }
            }
            const float base = (m == -INFINITY) ? 0.f : m;
            FA_TRACE_EV(tslot, 9);
            if constexpr (C::kSepP) {
                // The previous P.V of this tile must be done before P and O are touched.
                if (!wait(kBarPVDone + t, (pst_cnt & 1u) ^ 1u)) { ok = false; break; }
                tc_fence_after();
            }
            FA_TRACE_EV(tslot, 10);
            ++pst_cnt;
            // P = 2^(x - base) in 16-bit pairs, written to TMEM in four chunks.
            const float2 nb2 = make_float2(-base, -base);
            const float2 k2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 rs = full ? softmax_p_row<BF16, (SCORE != 0), C::emu_pairs(SCORE)>(x, nb2, k2, tP)
                                   : softmax_p_row<BF16, (SCORE != 0), 0>(x, nb2, k2, tP);
            l = fmaf(l, alpha, rs.x + rs.y);
            FA_TRACE_EV(tslot, 5);
            if (any_need && done > 0) {
                // Rescale O only now, after S has left the registers.
                const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tO + c * 32, o);
                    tmem_ld_wait();
                    reg_fence<32>(o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 v = __fmul2_rn(
                            make_float2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), al2);
                        o[2 * i] = __float_as_uint(v.x);
                        o[2 * i + 1] = __float_as_uint(v.y);
                    }
                    tmem_st_32x32b_x32(tO + c * 32, o);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive_warp(bar(kBarPFull + t));
            FA_TRACE_EV(tslot, 6);
            ++done;
        }
        if (!ok) return;
        u = take_unit<C>(p, bars, ring, u_iter, abort_flag, taken);
        // Epilogue: O / l in the output dtype, and the natural-log lse.
        FA_TRACE_EV(tslot, 7);
        if (!wait(kBarOFull + t, of_cnt & 1u)) return;
        ++of_cnt;
        tc_fence_after();
        const float inv = (l > 0.f) ? 1.0f / l : 0.f;
        const bool q_in = q < p.Q_LEN;   // rows past Q_LEN (a ragged last query tile) are not stored
        uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + un.b * p.out_stride[0] +
                         un.h * p.out_stride[1] + (int64_t)q * p.out_stride[2];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tO + c * 32, o);
            tmem_ld_wait();
            reg_fence<32>(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
            if (q_in) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
        if (p.lse && q_in)
            p.lse[((int64_t)un.b * p.H + un.h) * p.Q_LEN + q] =
                (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
        tc_fence_before();
        mbar_arrive_warp(bar(kBarOFree + t));
        FA_TRACE_EV(tslot, 8);
    }
}

// ------------------------------------------------------------------ kernel

template <int D, bool BF16, int VAR>
__global__ void __launch_bounds__(kThreadsFwd, 1)
attn_fwd_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tmq,
                const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
    using C = Cfg<D>;
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
        mbar_init(bars + 8u * kBarQFull, 1);
        mbar_init(bars + 8u * kBarQEmpty, C::kMmaWarps);   // one commit per MMA warp
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars + 8u * (kBarSFull + t), 1);
            mbar_init(bars + 8u * (kBarPFull + t), 4);   // one arrival per softmax warp
            mbar_init(bars + 8u * (kBarOFull + t), 1);
            mbar_init(bars + 8u * (kBarOFree + t), 4);
            mbar_init(bars + 8u * (kBarSFree + t), 4);
            mbar_init(bars + 8u * (kBarPVDone + t), 1);
        }
        mbar_init(bars + 8u * kBarDrain, 1);
        mbar_init(bars + 8u * (kBarDrain + 1), 1);
        for (int r = 0; r < kUnitRing; ++r) {
            mbar_init(bars + 8u * (C::kBarUFull + r), 1);    // the TMA warp publishes
            mbar_init(bars + 8u * (C::kBarUEmpty + r), C::kMmaWarps + 8);   // MMA + softmax warps
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bars + 8u * (C::kBarSlotFull + s), 1);
            mbar_init(bars + 8u * (C::kBarSlotEmpty + s), C::kMmaWarps);
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

    // Registers: the TMA/MMA warpgroup needs few, the softmax warpgroups hold a 128-wide
    // score row each (budgets above).  Each role runs inside the branch of its own budget.
    if (warp < 4) {
        regs_dec<kRegsProducer>();
        if (warp == 0) {
            producer_role<Cfg<D>>(p, &tmq, &tmk, &tmv, sbase, bars, ring, abort_flag);
        } else if (warp == 1 || (C::kMmaWarps == 2 && warp == 3)) {
            if constexpr (C::kMmaWarps == 2)
                mma_role_tile<D, BF16>(p, warp == 3 ? 1 : 0, sbase, bars, tmem, ring, abort_flag);
            else
                mma_role_pair<D, BF16>(p, sbase, bars, tmem, ring, abort_flag);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        softmax_role<D, BF16, VAR>(p, (warp - 4) >> 2, bars, tmem, ring, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tmem, 512);
}

template <int D, bool BF16, int VAR>
cudaError_t launch_t(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t stream) {
    auto kern = attn_fwd_kernel<D, BF16, VAR>;
    // setmaxnreg.inc waits for registers from the launched pool; refuse to launch a build
    // whose per-thread register count would make that pool smaller than the split needs.
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    if (attr.numRegs < kRegsAtLaunch) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreadsFwd, Cfg<D>::kSmemBytes, stream>>>(p, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const FwdParams& p, int D, bool bf16, int score_kind,
                            const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            int grid, cudaStream_t stream) {
    int var = score_kind | ((p.mask_kind & FA_MASK_DOCUMENT) ? kVarDocument : 0);
    // The fixed-max variant: bf16 (P keeps float32's exponent range) and a soft-cap of at most
    // 32 (so e^(-2 cap) stays a normal float), and with ALiBi a bias that cannot be positive
    // (a causal-type mask, the default positive slopes) and every query row's own key, whose
    // bias is 0, inside the context (no per-batch lengths, Q_LEN <= KV_LEN).  Without ALiBi
    // every live score is >= -cap, so any row with a live key keeps its sum that large.
    const bool causal_type = (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) != 0;
    if (bf16 && (score_kind & FA_SCORE_SOFTCAP) && p.softcap <= 32.0f &&
        (!(score_kind & FA_SCORE_ALIBI) ||
         (causal_type && !p.alibi_slopes && !p.kv_lens && p.Q_LEN <= p.KV_LEN)))
        var |= kVarFixedMax;
#define FA_CASE(DD, BB, VV)                                                 \
    if (D == DD && bf16 == BB && var == VV)                                 \
        return launch_t<DD, BB, VV>(p, tq, tk, tv, grid, stream);
#define FA_CASES(DD, BB) FA_CASE(DD, BB, 0) FA_CASE(DD, BB, 1) FA_CASE(DD, BB, 2) FA_CASE(DD, BB, 3) \
    FA_CASE(DD, BB, 4) FA_CASE(DD, BB, 5) FA_CASE(DD, BB, 6) FA_CASE(DD, BB, 7)
#define FA_FIXED(DD) FA_CASE(DD, true, 9) FA_CASE(DD, true, 11) FA_CASE(DD, true, 13) FA_CASE(DD, true, 15)
    FA_CASES(64, true)
    FA_CASES(64, false)
    FA_CASES(128, true)
    FA_CASES(128, false)
    FA_FIXED(64)
    FA_FIXED(128)
#undef FA_FIXED
#undef FA_CASES
#undef FA_CASE
    return cudaErrorInvalidValue;
}

}  // namespace fa
