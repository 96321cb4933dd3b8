// mask_builder.cu -- block-mask construction on the GPU.
//
// Follows "tensorplay.nn.attention.create_block_mask" (Parameters: BLOCK_SIZE,
// separate_full_blocks) and "How to Use FlexAttention on Apple Silicon" ("The two hooks":
// fully masked blocks are skipped; "Mask 1": build once, broadcast over B and H).
//
// Three steps, all integer work:
//   1. classify_compact_kernel: one CTA per (stored b/h, query block).  Each thread
//      classifies one kv block at a time as dead / partial / full.  The causal and
//      sliding-window predicates depend only on d = q - kv, which takes every integer
//      value between its extremes over a rectangular tile, so interval arithmetic on d
//      classifies those tiles exactly.  The document predicate is resolved from
//      per-block (min, max, uniform) statistics where they decide it; the remaining
//      tiles are evaluated element by element by the whole CTA.  Live tiles are then
//      compacted into ascending lists with warp ballots and popc prefix sums.
//   2. schedule_kernel: one CTA per work unit (a pair of adjacent query blocks) merges
//      the two tiles' partial and full lists into one list of kv blocks, nearest first
//      (descending), with per-tile live/full flags, so the forward kernel loads each K/V
//      tile once for both query tiles.  The unit's cost estimates its forward time in
//      quarter entries: an entry with both tiles live costs 4 (the two softmax groups run
//      side by side), an entry with one live tile 3 (one group runs alone, faster per tile
//      but not twice as fast), plus 2 for the unit's prologue and epilogue; with L live
//      tiles over n entries that is L + 2n + 2.
//   3. lpt_order_kernel: ranks the units of each stored (b, h) by descending cost (ties
//      by index) so the persistent forward kernel hands the longest units out first.
#include <climits>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kThreads = 128;
// The classifier: one thread per kv block of a query block's row (in chunks), and 16 warps to
// resolve the row's ambiguous tiles (a query block holding a document boundary can have dozens).
constexpr int kClsThreads = 512;

__global__ void __launch_bounds__(kThreads) doc_block_stats_kernel(const int32_t* __restrict__ doc,
                                                                  int len, int nblk, int bs,
                                                                  int32_t* __restrict__ stats) {
    const int blk = blockIdx.x;
    if (blk >= nblk) return;
    const int s0 = blk * bs;
    const int n = min(bs, len - s0);
    int mn = INT_MAX, mx = INT_MIN;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int d = doc[s0 + i];
        mn = min(mn, d);
        mx = max(mx, d);
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    __shared__ int smn[kThreads / 32], smx[kThreads / 32];
    if ((threadIdx.x & 31) == 0) {
        smn[threadIdx.x >> 5] = mn;
        smx[threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) {
            mn = min(mn, smn[w]);
            mx = max(mx, smx[w]);
        }
        stats[3 * blk + 0] = mn;
        stats[3 * blk + 1] = mx;
        stats[3 * blk + 2] = (mn == mx) ? 1 : 0;
    }
}

// Allowed range of d = q - kv from the interval predicates (causal, sliding window).
__device__ __forceinline__ void interval_bounds(const MaskSpec& m, long long& lo, long long& hi) {
    lo = LLONG_MIN / 4;
    hi = LLONG_MAX / 4;
    if (m.kind & FA_MASK_CAUSAL) lo = lo > 0 ? lo : 0;
    if (m.kind & FA_MASK_SLIDING_WINDOW) {
        lo = lo > 0 ? lo : 0;
        hi = hi < (long long)m.window - 1 ? hi : (long long)m.window - 1;
    }
}

__device__ int classify_fast(const MaskSpec& m, int i, int j) {
    const int qs = i * m.BQ, qe = min(qs + m.BQ, m.Q_LEN) - 1;
    const int ks = j * m.BKV, ke = min(ks + m.BKV, m.KV_LEN) - 1;
    // A tile wholly past the context (a batch shorter than KV_LEN under kv_lens) has no key.
    if (ks >= m.KV_LEN || qs >= m.Q_LEN) return kDead;
    const bool ragged = (qe - qs + 1 < m.BQ) || (ke - ks + 1 < m.BKV);
    long long lo, hi;
    interval_bounds(m, lo, hi);
    const long long dmin = (long long)qs - ke, dmax = (long long)qe - ks;
    if (dmax < lo || dmin > hi) return kDead;
    const bool interval_full = dmin >= lo && dmax <= hi;
    if (!(m.kind & FA_MASK_DOCUMENT)) return (interval_full && !ragged) ? kFull : kPartial;
    const int32_t* qst = m.doc_stats + 3 * i;
    const int32_t* kst = m.doc_stats_kv + 3 * j;
    if (qst[1] < kst[0] || kst[1] < qst[0]) return kDead;   // id ranges disjoint
    if (qst[2] && kst[2]) {                                  // both blocks hold one id
        if (qst[0] != kst[0]) return kDead;
        return (interval_full && !ragged) ? kFull : kPartial;
    }
    return kAmbiguous;
}

// Element-by-element classification of one tile by one warp, in 32 x 32 sub-blocks: lane l
// holds key k0 + cb + l (and its document id) and walks the sub-block's 32 query rows, whose
// document ids it gets from the lane that loaded them (one shuffle per row, no memory access
// in the inner loop).  The warp stops as soon as it has seen both an allowed and a masked pair
// (a partial tile); row blocks are visited first, last, then the rest, so a tile whose mask
// changes only at its last rows (a document boundary near a block edge) is decided early.
// Only dead and full tiles are read in full.
__device__ int resolve_tile_warp(const MaskSpec& m, int i, int j) {
    long long lo64, hi64;
    interval_bounds(m, lo64, hi64);
    // q - kv of in-range pairs fits in 32 bits (lengths are below 2^31): clamp the bounds.
    const int lo = (int)max(lo64, (long long)INT_MIN), hi = (int)min(hi64, (long long)INT_MAX);
    const int lane = threadIdx.x & 31;
    const int q0 = i * m.BQ, k0 = j * m.BKV;
    const bool has_doc = (m.kind & FA_MASK_DOCUMENT) != 0;
    const int nrb = (m.BQ + 31) / 32, ncb = (m.BKV + 31) / 32;
    // Document ids of this lane's rows and keys, fetched up front (independent loads) for
    // tiles of up to 128 x 128; larger blocks fetch them per sub-block.
    constexpr int kPre = 4;
    int pre_q[kPre], pre_k[kPre];
#pragma unroll
    for (int c = 0; c < kPre; ++c) {
        const int qr = q0 + 32 * c + lane, kv = k0 + 32 * c + lane;
        pre_q[c] = (has_doc && c < nrb && 32 * c + lane < m.BQ && qr < m.Q_LEN) ? m.doc[qr] : 0;
        pre_k[c] = (has_doc && c < ncb && 32 * c + lane < m.BKV && kv < m.KV_LEN) ? m.doc[kv] : 0;
    }
    bool any = false, all = true;
    for (int t = 0; t < nrb; ++t) {
        const int rbi = t == 0 ? 0 : (t == 1 ? nrb - 1 : t - 1);
        const int rb = 32 * rbi;
        const int qr = q0 + rb + lane;
        int my_dq = 0;
#pragma unroll
        for (int c = 0; c < kPre; ++c)
            if (rbi == c) my_dq = pre_q[c];
        if (rbi >= kPre) my_dq = (has_doc && rb + lane < m.BQ && qr < m.Q_LEN) ? m.doc[qr] : 0;
        const int nrows = min(32, m.BQ - rb);
        for (int cbi = 0; cbi < ncb; ++cbi) {
            const int cb = 32 * cbi;
            const bool in_tile = cb + lane < m.BKV;          // lanes past the tile's keys sit out
            const int kv = k0 + cb + lane;
            const bool k_ok = in_tile && kv < m.KV_LEN;
            int dk = 0;
#pragma unroll
            for (int c = 0; c < kPre; ++c)
                if (cbi == c) dk = pre_k[c];
            if (cbi >= kPre) dk = (has_doc && k_ok) ? m.doc[kv] : 0;
            bool sub_any = false, sub_all = true;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const int dq = __shfl_sync(0xffffffffu, my_dq, r);
                const int q = q0 + rb + r;
                const int d = q - kv;
                const bool live = k_ok && q < m.Q_LEN && d >= lo && d <= hi && (!has_doc || dk == dq);
                if (r < nrows) {
                    sub_any |= live;
                    sub_all &= live;
                }
            }
            if (in_tile) {
                any |= sub_any;
                all &= sub_all;
            }
            const bool a = __any_sync(0xffffffffu, any);
            const bool f = __all_sync(0xffffffffu, all);
            if (a && !f) return kPartial;
        }
    }
    const bool a = __any_sync(0xffffffffu, any);
    const bool f = __all_sync(0xffffffffu, all);
    return !a ? kDead : (f ? kFull : kPartial);
}

__global__ void __launch_bounds__(kClsThreads)
classify_compact_kernel(MaskSpec m, int separate_full, int32_t* __restrict__ kv_num,
                        int32_t* __restrict__ kv_idx, int32_t* __restrict__ full_num,
                        int32_t* __restrict__ full_idx) {
    const int i = blockIdx.x;
    const int bh = blockIdx.y;
    // Per-batch context length: keys past it count as masked (the block grid stays KVB wide).
    if (m.kv_lens) m.KV_LEN = max(0, min(m.KV_LEN, m.kv_lens[bh / m.maskH]));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_cls[kClsThreads];
    __shared__ int s_amb[kClsThreads];
    __shared__ int s_namb;
    __shared__ int s_wp[kClsThreads / 32], s_wf[kClsThreads / 32];

    const size_t row = (size_t)bh * m.QB + i;
    int32_t* my_kv = kv_idx + row * m.KVB;
    int32_t* my_full = full_idx + row * m.KVB;
    int np = 0, nf = 0;
    for (int jb = 0; jb < m.KVB; jb += kClsThreads) {
        const int j = jb + tid;
        int cls = (j < m.KVB) ? classify_fast(m, i, j) : kDead;
        if (tid == 0) s_namb = 0;
        __syncthreads();
        if (cls == kAmbiguous) s_amb[atomicAdd(&s_namb, 1)] = tid;
        s_cls[tid] = cls;
        __syncthreads();
        const int namb = s_namb;
        for (int a = warp; a < namb; a += kClsThreads / 32) {   // one warp per ambiguous tile
            const int t = s_amb[a];
            const int c = resolve_tile_warp(m, i, jb + t);
            if (lane == 0) s_cls[t] = c;
        }
        __syncthreads();
        cls = s_cls[tid];
        if (!separate_full && cls == kFull) cls = kPartial;
        const unsigned bp = __ballot_sync(0xffffffffu, cls == kPartial);
        const unsigned bf = __ballot_sync(0xffffffffu, cls == kFull);
        if (lane == 0) {
            s_wp[warp] = __popc(bp);
            s_wf[warp] = __popc(bf);
        }
        __syncthreads();
        int op = np, of = nf, tp = 0, tf = 0;
        for (int w = 0; w < kClsThreads / 32; ++w) {
            if (w < warp) {
                op += s_wp[w];
                of += s_wf[w];
            }
            tp += s_wp[w];
            tf += s_wf[w];
        }
        const unsigned lt = (1u << lane) - 1u;
        if (cls == kPartial) my_kv[op + __popc(bp & lt)] = j;
        if (cls == kFull) my_full[of + __popc(bf & lt)] = j;
        np += tp;
        nf += tf;
        __syncthreads();
    }
    for (int t = np + tid; t < m.KVB; t += kClsThreads) my_kv[t] = 0;
    for (int t = nf + tid; t < m.KVB; t += kClsThreads) my_full[t] = 0;
    if (tid == 0) {
        kv_num[row] = np;
        full_num[row] = nf;
    }
}

__global__ void __launch_bounds__(kThreads)
schedule_kernel(int QB, int KVB, int NP, const int32_t* __restrict__ kv_num,
                const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ full_num,
                const int32_t* __restrict__ full_idx, int32_t* __restrict__ sched_count,
                int32_t* __restrict__ sched_cost, int32_t* __restrict__ sched_entries) {
    extern __shared__ uint8_t s_code[];  // one byte of flags per kv block
    const int p = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_w[kThreads / 32], s_l0[kThreads / 32], s_l1[kThreads / 32];
    for (int j = tid; j < KVB; j += kThreads) s_code[j] = 0;
    __syncthreads();
    for (int t = 0; t < 2; ++t) {
        const int i = 2 * p + t;
        if (i >= QB) break;
        const size_t row = (size_t)bh * QB + i;
        const uint8_t live = (uint8_t)(t ? (kLive1 >> 16) : (kLive0 >> 16));
        const uint8_t full = (uint8_t)(t ? (kFull1 >> 16) : (kFull0 >> 16));
        const int n_p = kv_num[row], n_f = full_num[row];
        for (int n = tid; n < n_p; n += kThreads) {
            const int j = kv_idx[row * KVB + n];
            if (j >= 0 && j < KVB) s_code[j] |= live;
        }
        __syncthreads();
        for (int n = tid; n < n_f; n += kThreads) {
            const int j = full_idx[row * KVB + n];
            if (j >= 0 && j < KVB) s_code[j] |= (uint8_t)(live | full);
        }
        __syncthreads();
    }
    const size_t unit = (size_t)bh * NP + p;
    int32_t* out = sched_entries + unit * KVB;
    // Entries go out nearest first (descending kv block): the diagonal tiles come first, so
    // a row's running max is usually settled by its first tile (with ALiBi the bias grows
    // toward the diagonal, and ascending order would raise the max on every tile).
    int cnt = 0, l0 = 0, l1 = 0;
    for (int jb = 0; jb < KVB; jb += kThreads) {
        const int j = KVB - 1 - (jb + tid);
        const int c = (j >= 0) ? s_code[j] : 0;
        const unsigned b = __ballot_sync(0xffffffffu, c != 0);
        const unsigned b0 = __ballot_sync(0xffffffffu, (c & (kLive0 >> 16)) != 0);
        const unsigned b1 = __ballot_sync(0xffffffffu, (c & (kLive1 >> 16)) != 0);
        if (lane == 0) {
            s_w[warp] = __popc(b);
            s_l0[warp] = __popc(b0);
            s_l1[warp] = __popc(b1);
        }
        __syncthreads();
        int off = cnt, tot = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) off += s_w[w];
            tot += s_w[w];
            l0 += s_l0[w];
            l1 += s_l1[w];
        }
        if (c != 0) out[off + __popc(b & ((1u << lane) - 1u))] = j | (c << 16);
        cnt += tot;
        __syncthreads();
    }
    if (tid == 0) {
        sched_count[2 * unit] = cnt;
        sched_count[2 * unit + 1] = l0 | (l1 << 16);
        sched_cost[unit] = l0 + l1 + 2 * cnt + 2;
    }
}

__global__ void __launch_bounds__(1024) lpt_order_kernel(int NP, const int32_t* __restrict__ cost,
                                                        int32_t* __restrict__ order) {
    extern __shared__ int s_cost[];
    const int bh = blockIdx.x;
    for (int p = threadIdx.x; p < NP; p += blockDim.x) s_cost[p] = cost[(size_t)bh * NP + p];
    __syncthreads();
    for (int p = threadIdx.x; p < NP; p += blockDim.x) {
        const int c = s_cost[p];
        int rank = 0;
        for (int o = 0; o < NP; ++o) {
            const int co = s_cost[o];
            rank += (co > c) || (co == c && o < p);
        }
        order[(size_t)bh * NP + rank] = p;
    }
}

// ------------------------------------------------------------------ backward metadata

__device__ __forceinline__ bool sorted_contains(const int32_t* __restrict__ a, int n, int x) {
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = a[mid];
        if (v == x) return true;
        if (v < x) lo = mid + 1; else hi = mid - 1;
    }
    return false;
}

// Transposed lists (per kv block, the query blocks whose tile is partial / full, ascending)
// and the kv-major entries of the dK/dV kernel: query block i | kLive0 (| kFull0), ascending.
// One CTA per (stored b/h, kv block); each thread looks its query row's tile up in the row's
// sorted lists.
__global__ void __launch_bounds__(kThreads)
transpose_lists_kernel(int QB, int KVB, const int32_t* __restrict__ kv_num,
                       const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ full_num,
                       const int32_t* __restrict__ full_idx, int32_t* __restrict__ q_num,
                       int32_t* __restrict__ q_idx, int32_t* __restrict__ fq_num,
                       int32_t* __restrict__ fq_idx, int32_t* __restrict__ kv_count,
                       int32_t* __restrict__ kv_cost, int32_t* __restrict__ kv_entries) {
    const int j = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_wp[kThreads / 32], s_wf[kThreads / 32];
    const size_t col = (size_t)bh * KVB + j;
    int32_t* my_q = q_idx + col * QB;
    int32_t* my_fq = fq_idx + col * QB;
    int32_t* my_e = kv_entries ? kv_entries + col * QB : nullptr;
    int np = 0, nf = 0;
    for (int ib = 0; ib < QB; ib += kThreads) {
        const int i = ib + tid;
        int cls = kDead;
        if (i < QB) {
            const size_t row = (size_t)bh * QB + i;
            const int n_p = min(max(kv_num[row], 0), KVB), n_f = min(max(full_num[row], 0), KVB);
            if (sorted_contains(full_idx + row * KVB, n_f, j)) cls = kFull;
            else if (sorted_contains(kv_idx + row * KVB, n_p, j)) cls = kPartial;
        }
        const unsigned bp = __ballot_sync(0xffffffffu, cls == kPartial);
        const unsigned bf = __ballot_sync(0xffffffffu, cls == kFull);
        if (lane == 0) {
            s_wp[warp] = __popc(bp);
            s_wf[warp] = __popc(bf);
        }
        __syncthreads();
        int op = np, of = nf, tp = 0, tf = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) {
                op += s_wp[w];
                of += s_wf[w];
            }
            tp += s_wp[w];
            tf += s_wf[w];
        }
        const unsigned lt = (1u << lane) - 1u;
        if (cls == kPartial) my_q[op + __popc(bp & lt)] = i;
        if (cls == kFull) my_fq[of + __popc(bf & lt)] = i;
        // Merged entries in ascending i: the live tiles before this thread's come first.
        const unsigned bl = bp | bf;
        if (cls != kDead && kv_entries)
            my_e[op + of + __popc(bl & lt)] =
                i | kLive0 | (cls == kFull ? kFull0 : 0);
        np += tp;
        nf += tf;
        __syncthreads();
    }
    for (int t = np + tid; t < QB; t += kThreads) my_q[t] = 0;
    for (int t = nf + tid; t < QB; t += kThreads) my_fq[t] = 0;
    if (kv_entries)
        for (int t = np + nf + tid; t < QB; t += kThreads) my_e[t] = 0;
    if (tid == 0) {
        q_num[col] = np;
        fq_num[col] = nf;
        if (kv_count) {
            kv_count[col] = np + nf;
            kv_cost[col] = np + nf + 1;
        }
    }
}

// Per query block, the merged kv list (partial | full) of the dQ kernel: kv block j | kLive0
// (| kFull0), in descending j when `descending`, else ascending.  This is the order in which
// the block's dQ accumulates its kv contributions (the dQ write order), fixed per mask.
__global__ void __launch_bounds__(kThreads)
dq_entries_kernel(int QB, int KVB, int descending, const int32_t* __restrict__ kv_num,
                  const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ full_num,
                  const int32_t* __restrict__ full_idx, int32_t* __restrict__ dq_count,
                  int32_t* __restrict__ dq_cost, int32_t* __restrict__ dq_entries) {
    extern __shared__ uint8_t s_code[];
    const int i = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_w[kThreads / 32];
    const size_t row = (size_t)bh * QB + i;
    for (int j = tid; j < KVB; j += kThreads) s_code[j] = 0;
    __syncthreads();
    const int n_p = min(max(kv_num[row], 0), KVB), n_f = min(max(full_num[row], 0), KVB);
    for (int n = tid; n < n_p; n += kThreads) {
        const int j = kv_idx[row * KVB + n];
        if (j >= 0 && j < KVB) s_code[j] = 1;
    }
    for (int n = tid; n < n_f; n += kThreads) {
        const int j = full_idx[row * KVB + n];
        if (j >= 0 && j < KVB) s_code[j] = 3;
    }
    __syncthreads();
    int32_t* out = dq_entries + row * KVB;
    int cnt = 0;
    for (int jb = 0; jb < KVB; jb += kThreads) {
        const int t = jb + tid;
        const int j = descending ? KVB - 1 - t : t;
        const int c = (t < KVB) ? s_code[j] : 0;
        const unsigned b = __ballot_sync(0xffffffffu, c != 0);
        if (lane == 0) s_w[warp] = __popc(b);
        __syncthreads();
        int off = cnt, tot = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) off += s_w[w];
            tot += s_w[w];
        }
        if (c != 0) out[off + __popc(b & ((1u << lane) - 1u))] = j | kLive0 | (c == 3 ? kFull0 : 0);
        cnt += tot;
        __syncthreads();
    }
    for (int t = cnt + tid; t < KVB; t += kThreads) out[t] = 0;
    if (tid == 0) {
        dq_count[row] = cnt;
        dq_cost[row] = cnt + 1;
    }
}

// Lists of 128 x 128 tiles from caller lists of BQ x BKV blocks (BQ = rq * 128,
// BKV = rkv * 128): each tile takes its block's class (a block listed as both partial and full
// counts as partial), a ragged tile is never full, and an index outside the block grid or a
// count outside [0, UKVB] sets *bad and is ignored.  One CTA per (stored b/h, query tile).
__global__ void __launch_bounds__(kThreads)
expand_block_lists_kernel(int UQB, int UKVB, int rq, int rkv, int QB, int KVB, int Q_LEN, int KV_LEN,
                          const int32_t* __restrict__ kv_lens, int maskH,
                          int separate_full, const int32_t* __restrict__ u_kv_num,
                          const int32_t* __restrict__ u_kv_idx, const int32_t* __restrict__ u_full_num,
                          const int32_t* __restrict__ u_full_idx, int32_t* __restrict__ kv_num,
                          int32_t* __restrict__ kv_idx, int32_t* __restrict__ full_num,
                          int32_t* __restrict__ full_idx, int32_t* __restrict__ bad) {
    extern __shared__ uint8_t s_code[];   // class of each of the row's UKVB blocks
    const int i = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int s_wp[kThreads / 32], s_wf[kThreads / 32];
    if (kv_lens) KV_LEN = max(0, min(KV_LEN, kv_lens[bh / maskH]));
    const int ui = i / rq;
    const size_t urow = (size_t)bh * UQB + ui;
    for (int j = tid; j < UKVB; j += kThreads) s_code[j] = kDead;
    __syncthreads();
    int n_p = u_kv_num[urow];
    if (n_p < 0 || n_p > UKVB) {
        if (tid == 0) atomicExch(bad, 2);
        n_p = min(max(n_p, 0), UKVB);
    }
    for (int n = tid; n < n_p; n += kThreads) {
        const int j = u_kv_idx[urow * UKVB + n];
        if (j >= 0 && j < UKVB) s_code[j] = kPartial;
        else atomicExch(bad, 2);
    }
    __syncthreads();
    if (u_full_num) {
        int n_f = u_full_num[urow];
        if (n_f < 0 || n_f > UKVB) {
            if (tid == 0) atomicExch(bad, 2);
            n_f = min(max(n_f, 0), UKVB);
        }
        for (int n = tid; n < n_f; n += kThreads) {
            const int j = u_full_idx[urow * UKVB + n];
            if (j >= 0 && j < UKVB) {
                if (s_code[j] != kPartial) s_code[j] = kFull;
            } else {
                atomicExch(bad, 2);
            }
        }
        __syncthreads();
    }
    const size_t row = (size_t)bh * QB + i;
    int32_t* my_kv = kv_idx + row * KVB;
    int32_t* my_full = full_idx + row * KVB;
    const bool q_ragged = (i + 1) * kBlock > Q_LEN;
    int np = 0, nf = 0;
    for (int jb = 0; jb < KVB; jb += kThreads) {
        const int j = jb + tid;
        int cls = (j < KVB) ? s_code[j / rkv] : kDead;
        if (j * kBlock >= KV_LEN) cls = kDead;          // past this batch's context
        if (cls == kFull && (q_ragged || (j + 1) * kBlock > KV_LEN)) cls = kPartial;
        if (!separate_full && cls == kFull) cls = kPartial;
        const unsigned bp = __ballot_sync(0xffffffffu, cls == kPartial);
        const unsigned bf = __ballot_sync(0xffffffffu, cls == kFull);
        if (lane == 0) {
            s_wp[warp] = __popc(bp);
            s_wf[warp] = __popc(bf);
        }
        __syncthreads();
        int op = np, of = nf, tp = 0, tf = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) {
                op += s_wp[w];
                of += s_wf[w];
            }
            tp += s_wp[w];
            tf += s_wf[w];
        }
        const unsigned lt = (1u << lane) - 1u;
        if (cls == kPartial) my_kv[op + __popc(bp & lt)] = j;
        if (cls == kFull) my_full[of + __popc(bf & lt)] = j;
        np += tp;
        nf += tf;
        __syncthreads();
    }
    for (int t = np + tid; t < KVB; t += kThreads) my_kv[t] = 0;
    for (int t = nf + tid; t < KVB; t += kThreads) my_full[t] = 0;
    if (tid == 0) {
        kv_num[row] = np;
        full_num[row] = nf;
    }
}

}  // namespace

cudaError_t launch_expand_block_lists(int UQB, int UKVB, int rq, int rkv, int QB, int KVB, int Q_LEN,
                                      int KV_LEN, const int32_t* kv_lens, int maskH, int maskBH,
                                      int separate_full,
                                      const int32_t* u_kv_num, const int32_t* u_kv_idx,
                                      const int32_t* u_full_num, const int32_t* u_full_idx,
                                      int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                                      int32_t* full_idx, int32_t* bad, cudaStream_t stream) {
    expand_block_lists_kernel<<<dim3(QB, maskBH), kThreads, UKVB, stream>>>(
        UQB, UKVB, rq, rkv, QB, KVB, Q_LEN, KV_LEN, kv_lens, maskH, separate_full, u_kv_num, u_kv_idx, u_full_num,
        u_full_idx, kv_num, kv_idx, full_num, full_idx, bad);
    return cudaGetLastError();
}

cudaError_t launch_transpose_lists(int QB, int KVB, int maskBH, const int32_t* kv_num,
                                   const int32_t* kv_idx, const int32_t* full_num,
                                   const int32_t* full_idx, int32_t* q_num, int32_t* q_idx,
                                   int32_t* fq_num, int32_t* fq_idx, cudaStream_t stream) {
    transpose_lists_kernel<<<dim3(KVB, maskBH), kThreads, 0, stream>>>(
        QB, KVB, kv_num, kv_idx, full_num, full_idx, q_num, q_idx, fq_num, fq_idx, nullptr, nullptr,
        nullptr);
    return cudaGetLastError();
}

cudaError_t launch_backward_metadata(int QB, int KVB, int maskBH, int dq_descending,
                                     const int32_t* kv_num, const int32_t* kv_idx,
                                     const int32_t* full_num, const int32_t* full_idx,
                                     const BwdMeta& m, cudaStream_t stream) {
    // The ranking keeps every unit's cost in shared memory: up to 16384 ints.
    const int lpt_smem = (QB > KVB ? QB : KVB) * (int)sizeof(int);
    if (lpt_smem > 48 * 1024) {
        cudaError_t ea = cudaFuncSetAttribute(lpt_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              lpt_smem);
        if (ea != cudaSuccess) return ea;
    }
    transpose_lists_kernel<<<dim3(KVB, maskBH), kThreads, 0, stream>>>(
        QB, KVB, kv_num, kv_idx, full_num, full_idx, m.q_num, m.q_idx, m.fq_num, m.fq_idx,
        m.kv_count, m.kv_cost, m.kv_entries);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    lpt_order_kernel<<<maskBH, 1024, KVB * (int)sizeof(int), stream>>>(KVB, m.kv_cost, m.kv_order);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dq_entries_kernel<<<dim3(QB, maskBH), kThreads, KVB, stream>>>(
        QB, KVB, dq_descending, kv_num, kv_idx, full_num, full_idx, m.dq_count, m.dq_cost,
        m.dq_entries);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    lpt_order_kernel<<<maskBH, 1024, QB * (int)sizeof(int), stream>>>(QB, m.dq_cost, m.dq_order);
    return cudaGetLastError();
}

cudaError_t launch_mask_lists(const MaskSpec& spec, int separate_full, int maskBH,
                              int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                              int32_t* full_idx, int32_t* doc_stats, cudaStream_t stream) {
    // Per-block document statistics: one array when the query and kv blocks have one size
    // (max(QB, KVB) entries), else the query blocks' first and the kv blocks' after them.
    MaskSpec s = spec;
    s.doc_stats = doc_stats;
    s.doc_stats_kv = doc_stats;
    if (spec.kind & FA_MASK_DOCUMENT) {
        if (spec.BQ == spec.BKV) {
            const int nblk = spec.QB > spec.KVB ? spec.QB : spec.KVB;
            doc_block_stats_kernel<<<nblk, kThreads, 0, stream>>>(spec.doc, spec.KV_LEN, nblk, spec.BQ,
                                                                  doc_stats);
        } else {
            s.doc_stats_kv = doc_stats + 3 * (size_t)spec.QB;
            doc_block_stats_kernel<<<spec.QB, kThreads, 0, stream>>>(spec.doc, spec.KV_LEN, spec.QB,
                                                                     spec.BQ, doc_stats);
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            doc_block_stats_kernel<<<spec.KVB, kThreads, 0, stream>>>(
                spec.doc, spec.KV_LEN, spec.KVB, spec.BKV, doc_stats + 3 * (size_t)spec.QB);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    classify_compact_kernel<<<dim3(spec.QB, maskBH), kClsThreads, 0, stream>>>(
        s, separate_full, kv_num, kv_idx, full_num, full_idx);
    return cudaGetLastError();
}

cudaError_t launch_mask_build(const MaskSpec& spec, int separate_full, int maskBH, int NP,
                              int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                              int32_t* full_idx, int32_t* doc_stats, int32_t* sched_count,
                              int32_t* sched_cost, int32_t* sched_entries, int32_t* sched_order,
                              cudaStream_t stream) {
    cudaError_t e = launch_mask_lists(spec, separate_full, maskBH, kv_num, kv_idx, full_num,
                                      full_idx, doc_stats, stream);
    if (e != cudaSuccess) return e;
    e = launch_schedule(spec.QB, spec.KVB, maskBH, NP, kv_num, kv_idx, full_num, full_idx,
                        sched_count, sched_cost, sched_entries, sched_order, stream);
    return e;
}

// All units of every stored (b, h) ranked together by descending cost (ties by index): entry r
// is the unit index sidx * NP + pair of rank r.  One CTA; n <= kGlobalOrderMax.
__global__ void __launch_bounds__(1024) global_order_kernel(int n, const int32_t* __restrict__ cost,
                                                           int32_t* __restrict__ order) {
    extern __shared__ int s_gcost[];
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_gcost[i] = cost[i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int c = s_gcost[i];
        int rank = 0;
        for (int o = 0; o < n; ++o) {
            const int co = s_gcost[o];
            rank += (co > c) || (co == c && o < i);
        }
        order[rank] = i;
    }
}

cudaError_t launch_global_order(int n, const int32_t* cost, int32_t* order, cudaStream_t stream) {
    if (n <= 0 || n > kGlobalOrderMax) return cudaErrorInvalidValue;
    const int smem = n * (int)sizeof(int);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(global_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    global_order_kernel<<<1, 1024, smem, stream>>>(n, cost, order);
    return cudaGetLastError();
}

cudaError_t launch_schedule(int QB, int KVB, int maskBH, int NP, const int32_t* kv_num,
                            const int32_t* kv_idx, const int32_t* full_num, const int32_t* full_idx,
                            int32_t* sched_count, int32_t* sched_cost, int32_t* sched_entries,
                            int32_t* sched_order, cudaStream_t stream) {
    const MaskSpec spec{0, 0, 0, 0, QB, KVB, kBlock, kBlock, nullptr, nullptr, nullptr, nullptr, 1};
    cudaError_t e;
    schedule_kernel<<<dim3(NP, maskBH), kThreads, spec.KVB, stream>>>(
        spec.QB, spec.KVB, NP, kv_num, kv_idx, full_num, full_idx, sched_count, sched_cost,
        sched_entries);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    lpt_order_kernel<<<maskBH, 1024, NP * (int)sizeof(int), stream>>>(NP, sched_cost, sched_order);
    return cudaGetLastError();
}

}  // namespace fa
