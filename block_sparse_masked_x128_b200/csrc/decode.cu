// decode.cu -- attention of a few new query tokens over a paged K/V cache, split over CTAs.
//
// What it computes: fa_forward's attention (mask_mod on partial tiles, score_mod, softmax, P V,
// lse) for Q_LEN <= 4 query rows per (b, h), with the keys and values in 128-token pages of a
// pool that a page table maps (PagedAttention through block indices, "PyTorch 2.13 brings
// custom AI attention to Mac", "What Attention Patterns Does FlexAttention Support?").  With
// so few query rows the work is reading K and V once: 2 * D multiply-adds per key and query
// against 4 * D bytes per key, so this path is bound by HBM and runs on the CUDA cores; the
// tensor-core forward would spend a 128-row tile on each query row.
//
// Organisation:
//   decode_split_kernel   grid (chunks, B * H): CTA (c, bh) takes tiles c*T .. c*T+T-1 of the
//                         (b, h)'s live-tile list (the block mask's schedule for query block 0).
//                         Each key is read by D/8 lanes, 16 bytes each (a 256-byte row at
//                         D = 128 is one half-warp); four keys per lane group are loaded ahead
//                         of use.  Each lane group keeps its own running max, sum and slice of
//                         O (in log2 units, rescaled when the max grows), and the CTA combines
//                         its groups through shared memory into one partial (m, l, O) per query
//                         row, written to the workspace.
//   decode_merge_kernel   one CTA per (b, h, query row): combines the chunks' partials,
//                         O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c, lse = (M + log2 L) ln 2.
// No waits between CTAs; the merge runs after the split kernel on the same stream.
#include <cfloat>

#include <cuda_fp16.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecAhead = 4;          // keys a lane group loads ahead of use
constexpr float kDecLog2e = 1.4426950408889634f;
constexpr float kDecLn2 = 0.6931471805599453f;

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (BF16) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        } else {
            f[2 * i] = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
            f[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
        }
    }
}

__device__ __forceinline__ float dec_slope_log2(const DecodeParams& p, int h) {
    float slope;
    if (p.alibi_slopes) {
        slope = __ldg(p.alibi_slopes + h);
    } else {
        const int num = 8 * (h + 1);
        slope = (num % p.H == 0) ? ldexpf(1.0f, -(num / p.H)) : exp2f(-(float)num / (float)p.H);
    }
    return slope * kDecLog2e;
}

template <int D, bool BF16, int SCORE, int Q>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int LPK = D / 8;            // lanes per key (16 bytes each)
    constexpr int KPW = 32 / LPK;         // keys per warp step
    constexpr int KPC = KPW * kDecWarps;  // keys per CTA step
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane % LPK, grp = lane / LPK;
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int b = bh / p.H, h = bh - b * p.H;
    const int mb = (p.maskB == 1) ? 0 : b, mh = (p.maskH == 1) ? 0 : h;
    const size_t sidx = (size_t)mb * p.maskH + mh;
    const int E = __ldg(p.sched_count + 2 * sidx * p.NP);     // entries of query block 0
    const int32_t* entries = p.sched_entries + sidx * p.NP * (size_t)p.KVB;
    const int t0 = chunk * p.tiles_per_chunk, t1 = min(E, t0 + p.tiles_per_chunk);
    const int kv_len = p.kv_lens ? min(p.KV_LEN, __ldg(p.kv_lens + mb)) : p.KV_LEN;
    const float slope_log2 = (SCORE & FA_SCORE_ALIBI) ? dec_slope_log2(p, h) : 0.f;

    // This lane's 8 dims of every query row.
    float qv[Q][8];
#pragma unroll
    for (int qi = 0; qi < Q; ++qi) {
        const uint4 r = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + b * p.q_stride[0] +
                                                        h * p.q_stride[1] + (int64_t)qi * p.q_stride[2] + sub * 8);
        unpack8<BF16>(r, qv[qi]);
    }
    float m[Q], l[Q], o[Q][8];
#pragma unroll
    for (int qi = 0; qi < Q; ++qi) {
        m[qi] = -INFINITY;
        l[qi] = 0.f;
#pragma unroll
        for (int d = 0; d < 8; ++d) o[qi][d] = 0.f;
    }
    const uint16_t* kbase = reinterpret_cast<const uint16_t*>(p.k) + h * p.k_stride[1] + sub * 8;
    const uint16_t* vbase = reinterpret_cast<const uint16_t*>(p.v) + h * p.v_stride[1] + sub * 8;

    for (int t = t0; t < t1; ++t) {
        const int code = __ldg(entries + t);
        int j = code & 0xFFFF;
        FA_DCHECK_INDEX(j, p.KVB, p.status);
        const bool full = (code & kFull0) != 0;
        // The page holding keys j*128 .. j*128+127 (every page of the pools is a whole 128-row
        // page, so all its rows may be read; keys past the context are masked below).
        const int page = __ldg(p.page_table + (size_t)b * p.page_stride + j);
        if (page < 0 || page >= p.n_pages) {   // recorded; the tile is skipped
            if (threadIdx.x == 0) atomicExch(p.status, 2);
            continue;
        }
        const uint16_t* kt = kbase + (int64_t)page * p.k_stride[0];
        const uint16_t* vt = vbase + (int64_t)page * p.v_stride[0];
        for (int k0 = 0; k0 < kBlock; k0 += KPC * kDecAhead) {
            uint4 kr[kDecAhead], vr[kDecAhead];
#pragma unroll
            for (int a = 0; a < kDecAhead; ++a) {
                const int r = k0 + a * KPC + warp * KPW + grp;
                kr[a] = *reinterpret_cast<const uint4*>(kt + (int64_t)r * p.k_stride[2]);
                vr[a] = *reinterpret_cast<const uint4*>(vt + (int64_t)r * p.v_stride[2]);
            }
#pragma unroll
            for (int a = 0; a < kDecAhead; ++a) {
                const int r = k0 + a * KPC + warp * KPW + grp;
                const int kv = j * kBlock + r;
                float kf[8], vf[8];
                unpack8<BF16>(kr[a], kf);
                unpack8<BF16>(vr[a], vf);
#pragma unroll
                for (int qi = 0; qi < Q; ++qi) {
                    float s = 0.f;
#pragma unroll
                    for (int d = 0; d < 8; ++d) s = fmaf(qv[qi][d], kf[d], s);
#pragma unroll
                    for (int off = LPK / 2; off > 0; off >>= 1) s += __shfl_xor_sync(kFullMask, s, off);
                    // score_mod in log2 units, then the mask on partial tiles.
                    float x;
                    if constexpr ((SCORE & FA_SCORE_SOFTCAP) != 0) x = p.softcap_log2 * tanh_approx(s * p.inv_softcap_scale);
                    else x = s * p.scale_log2;
                    if constexpr ((SCORE & FA_SCORE_ALIBI) != 0) x = fmaf(slope_log2, (float)(kv - qi), x);
                    bool live = true;
                    if (!full) {
                        live = kv < kv_len;
                        const int d = qi - kv;
                        if (p.mask_kind & (FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW)) live = live && d >= 0;
                        if (p.mask_kind & FA_MASK_SLIDING_WINDOW) live = live && d < p.window;
                        if (p.mask_kind & FA_MASK_DOCUMENT) live = live && (__ldg(p.doc_id + qi) == __ldg(p.doc_id + kv));
                    }
                    if (live) {
                        if (x > m[qi]) {
                            const float alpha = ex2_approx(m[qi] - x);   // m = -inf gives 0
                            l[qi] *= alpha;
#pragma unroll
                            for (int d = 0; d < 8; ++d) o[qi][d] *= alpha;
                            m[qi] = x;
                        }
                        const float pr = ex2_approx(x - m[qi]);
                        l[qi] += pr;
#pragma unroll
                        for (int d = 0; d < 8; ++d) o[qi][d] = fmaf(pr, vf[d], o[qi][d]);
                    }
                }
            }
        }
    }
    // Combine the CTA's lane groups: group g of warp w is slot w * KPW + g.
    __shared__ float s_m[kDecWarps * KPW][Q], s_l[kDecWarps * KPW][Q];
    __shared__ float s_o[kDecWarps * KPW][Q][D];
    const int slot = warp * KPW + grp;
#pragma unroll
    for (int qi = 0; qi < Q; ++qi) {
        if (sub == 0) {
            s_m[slot][qi] = m[qi];
            s_l[slot][qi] = l[qi];
        }
#pragma unroll
        for (int d = 0; d < 8; ++d) s_o[slot][qi][sub * 8 + d] = o[qi][d];
    }
    __syncthreads();
    // Thread t < Q * D finishes (query t / D, dim t % D); the first D threads also write m, l.
    float* part = p.partials + (((size_t)bh * Q) * p.max_chunks + chunk) * (size_t)(D + 2);
    for (int t = threadIdx.x; t < Q * D; t += kDecThreads) {
        const int qi = t / D, d = t - qi * D;
        float M = -INFINITY;
        for (int g = 0; g < kDecWarps * KPW; ++g) M = fmaxf(M, s_m[g][qi]);
        float L = 0.f, O = 0.f;
        for (int g = 0; g < kDecWarps * KPW; ++g) {
            const float w = (s_m[g][qi] == -INFINITY) ? 0.f : ex2_approx(s_m[g][qi] - M);
            L = fmaf(s_l[g][qi], w, L);
            O = fmaf(s_o[g][qi][d], w, O);
        }
        float* pq = part + (size_t)qi * p.max_chunks * (D + 2);
        pq[2 + d] = O;
        if (d == 0) {
            pq[0] = M;
            pq[1] = L;
        }
    }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(128) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
    const int row = blockIdx.x;                 // (b * H + h) * Q_LEN + qi
    const int qi = row % p.Q_LEN, bh = row / p.Q_LEN;
    const int b = bh / p.H, h = bh - b * p.H;
    const float* part = p.partials + ((size_t)bh * p.Q_LEN + qi) * p.max_chunks * (size_t)(D + 2);
    float M = -INFINITY;
    for (int c = 0; c < p.max_chunks; ++c) M = fmaxf(M, part[(size_t)c * (D + 2)]);
    float L = 0.f;
    for (int c = 0; c < p.max_chunks; ++c) {
        const float mc = part[(size_t)c * (D + 2)];
        if (mc != -INFINITY) L = fmaf(part[(size_t)c * (D + 2) + 1], ex2_approx(mc - M), L);
    }
    const float inv = (L > 0.f) ? 1.0f / L : 0.f;
    uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + b * p.out_stride[0] + h * p.out_stride[1] +
                     (int64_t)qi * p.out_stride[2];
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float O = 0.f;
        for (int c = 0; c < p.max_chunks; ++c) {
            const float mc = part[(size_t)c * (D + 2)];
            if (mc != -INFINITY) O = fmaf(part[(size_t)c * (D + 2) + 2 + d], ex2_approx(mc - M), O);
        }
        const float v = O * inv;
        orow[d] = BF16 ? (uint16_t)(pack2<true>(v, 0.f) & 0xFFFFu) : (uint16_t)(pack2<false>(v, 0.f) & 0xFFFFu);
    }
    if (threadIdx.x == 0 && p.lse)
        p.lse[((int64_t)b * p.H + h) * p.Q_LEN + qi] = (L > 0.f) ? (M + log2f(L)) * kDecLn2 : -INFINITY;
}

template <int D, bool BF16, int SCORE>
cudaError_t launch_split(const DecodeParams& p, cudaStream_t st) {
    const dim3 grid(p.max_chunks, p.B * p.H);
    switch (p.Q_LEN) {
        case 1: decode_split_kernel<D, BF16, SCORE, 1><<<grid, kDecThreads, 0, st>>>(p); break;
        case 2: decode_split_kernel<D, BF16, SCORE, 2><<<grid, kDecThreads, 0, st>>>(p); break;
        case 3: decode_split_kernel<D, BF16, SCORE, 3><<<grid, kDecThreads, 0, st>>>(p); break;
        case 4: decode_split_kernel<D, BF16, SCORE, 4><<<grid, kDecThreads, 0, st>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_merge_kernel<D, BF16><<<p.B * p.H * p.Q_LEN, 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int D, bool bf16, int score_kind, cudaStream_t st) {
#define FA_DEC(DD, BB, SS) \
    if (D == DD && bf16 == BB && score_kind == SS) return launch_split<DD, BB, SS>(p, st);
#define FA_DECS(DD, BB) FA_DEC(DD, BB, 0) FA_DEC(DD, BB, 1) FA_DEC(DD, BB, 2) FA_DEC(DD, BB, 3)
    FA_DECS(64, true)
    FA_DECS(64, false)
    FA_DECS(128, true)
    FA_DECS(128, false)
#undef FA_DECS
#undef FA_DEC
    return cudaErrorInvalidValue;
}

}  // namespace fa
