// masked_softmax.cu -- the causal-masked softmax over materialised scores, fused.
//
// What it computes ("Fuse the causal mask into the SDPA fallback softmax", MLX pull request
// 3919, Summary and Description): the chain
//     keep = q + offset >= kv;  x = keep ? score : finfo(dtype).min;  probs = softmax(x)
// in one pass over memory.  The select is applied where the scores are read, so the
// per-element arithmetic is the plain softmax's on the selected values: the result is
// bit-identical to running this kernel without the mask on where(keep, scores, finfo.min),
// and masked entries are exactly zero (exp(finfo.min - max) underflows).  Scores behind the
// causal boundary are never read: their selected value does not depend on them.
//
// Organisation (HBM-bound; one persistent CTA of 512 threads per SM):
//   * rows (b, h, q) are dealt round robin to the CTAs;
//   * warp 0 only moves data: it stages each row's live prefix into shared memory with one
//     cp.async.bulk load into a ring of `stages` row buffers (completing on the buffer's
//     `full` mbarrier), stores each computed row with one cp.async.bulk store, and as soon as
//     that store has read the buffer, loads the row `stages` ahead into it;
//   * warps 1-15 hold the row in registers (thread c owns the 16-byte vectors c, c + 480,
//     ...), take the row max and the row sum of e = 2^((x - max) log2 e) with warp shuffles
//     and a fixed-order cross-warp step on a named barrier of their own, write p = e / sum
//     back over the buffer as 16-bit values and arrive on the buffer's `done` mbarrier.
// Every reduction has the same order in the masked and the unmasked run, which is what
// makes them bit-identical.  Waits are bounded: a wait that runs out sets the status word,
// and the CTA drains its own copies before it returns.
#include <cfloat>

#include <cuda_fp16.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {

struct SoftmaxParams {
    const uint16_t* in;
    uint16_t* out;
    int64_t in_stride[3];   // b, h, q strides in elements (the key stride is 1)
    int64_t out_stride[3];
    int32_t B, H, Q, K;
    int64_t offset;         // query row q keeps keys kv <= q + offset
    int32_t causal;
    int64_t rows;           // B * H * Q
    int32_t stages;
    uint32_t stage_bytes;   // K * 2 rounded up to 128
    int32_t* status;
    int32_t stall_loads;    // test hook: the producer loads the first buffers only
};

namespace {

constexpr int kSmThreads = 512;
constexpr int kSmWarps = kSmThreads / 32;
constexpr int kSmCompute = kSmThreads - 32;   // warp 0 moves data, warps 1.. compute
constexpr uint64_t kSmWaitLimitNs = 2000000000ull;
constexpr float kSmLog2e = 1.4426950408889634f;

__device__ int32_t g_softmax_status;

template <bool BF16>
__device__ __forceinline__ float dtype_min() {
    // finfo(bfloat16).min = -(2 - 2^-7) * 2^127 and finfo(float16).min = -65504, as float.
    return BF16 ? -3.38953138925153547590e38f : -65504.0f;
}

// Two 16-bit values (lo in bits 0-15) as floats.
template <bool BF16>
__device__ __forceinline__ float2 to_f32x2(uint32_t w) {
    if constexpr (BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

__device__ __forceinline__ int64_t live_keys(const SoftmaxParams& p, int64_t q) {
    if (!p.causal) return p.K;
    int64_t n = q + p.offset + 1;
    return n < 0 ? 0 : (n > p.K ? p.K : n);
}

__device__ __forceinline__ void row_coords(const SoftmaxParams& p, int64_t r, int64_t& b, int64_t& h,
                                           int64_t& q) {
    q = r % p.Q;
    const int64_t bh = r / p.Q;
    h = bh % p.H;
    b = bh / p.H;
}

// Bytes the bulk load brings for row r: its live prefix rounded up to 16 bytes (K is a
// multiple of 8, so the rounding stays inside the row).
__device__ __forceinline__ uint32_t load_bytes(const SoftmaxParams& p, int64_t r) {
    int64_t b, h, q;
    row_coords(p, r, b, h, q);
    const int64_t n = live_keys(p, q);
    return (uint32_t)(((n + 7) & ~7ll) * 2);
}

__device__ __forceinline__ void issue_row_load(const SoftmaxParams& p, int64_t r, uint32_t dst,
                                               uint32_t bar) {
    int64_t b, h, q;
    row_coords(p, r, b, h, q);
    const uint32_t bytes = load_bytes(p, r);
    mbar_arrive_expect_tx(bar, bytes);
    if (bytes > 0)
        bulk_load(dst, p.in + b * p.in_stride[0] + h * p.in_stride[1] + q * p.in_stride[2], bytes, bar);
}

// Bounded wait on an mbarrier phase by the calling thread.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 127u) == 0u && global_timer_ns() - t0 > kSmWaitLimitNs) return false;
    }
}

// The compute warps' barrier (named barrier 1; warp 0 never takes part), with the AND of `v`.
__device__ __forceinline__ bool compute_bar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "n"(kSmCompute)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void compute_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kSmCompute) : "memory");
}

template <bool BF16, int VPT>
__global__ void __launch_bounds__(kSmThreads, 1) masked_softmax_kernel(const __grid_constant__ SoftmaxParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                               ~static_cast<uintptr_t>(127));
    const uint32_t sbase = smem_u32(smem);
    // Barriers: full[s] (the row's bulk load landed), done[s] (the compute warps wrote p).
    const uint32_t bars = sbase + (uint32_t)p.stages * p.stage_bytes;
    auto full_bar = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto done_bar = [&](int s) { return bars + 8u * (uint32_t)(p.stages + s); };
    float* red = reinterpret_cast<float*>(smem + (size_t)p.stages * p.stage_bytes + 16 * p.stages);
    float* red_max = red;
    float* red_sum = red + kSmWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t grid = gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(done_bar(s), kSmCompute / 32);   // one arrival per compute warp
        }
        fence_mbar_init();
    }
    __syncthreads();
    // Rows of this CTA: blockIdx.x + k * grid, k = 0, 1, ...; row k lives in buffer k % stages.
    const int64_t my_rows = (p.rows > blockIdx.x) ? (p.rows - blockIdx.x + grid - 1) / grid : 0;

    if (warp == 0) {
        // Producer: loads rows ahead into free buffers; stores each computed row, and once the
        // store has read its buffer, loads the row `stages` ahead into it.
        if (lane == 0) {
            int64_t issued = 0;
            for (; issued < my_rows && issued < p.stages; ++issued)
                issue_row_load(p, blockIdx.x + issued * grid, sbase + (uint32_t)issued * p.stage_bytes,
                               full_bar((int)issued));
            int64_t k = 0;
            bool ok = true;
            if (p.stall_loads) {   // test hook: the compute warps' wait for row `stages` runs out
                for (int64_t kk = 0; kk < issued; ++kk) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(full_bar((int)kk), 0u) && global_timer_ns() - t0 < kSmWaitLimitNs) {
                    }
                }
                k = my_rows;   // store nothing
            }
            for (; k < my_rows; ++k) {
                const int s = (int)(k % p.stages);
                if (!wait_bounded(done_bar(s), (uint32_t)((k / p.stages) & 1))) { ok = false; break; }
                int64_t b, h, q;
                row_coords(p, blockIdx.x + k * grid, b, h, q);
                bulk_store(p.out + b * p.out_stride[0] + h * p.out_stride[1] + q * p.out_stride[2],
                           sbase + (uint32_t)s * p.stage_bytes, (uint32_t)(p.K * 2));
                bulk_commit();
                if (issued < my_rows) {
                    bulk_wait_read<0>();
                    fence_proxy_async_smem();
                    issue_row_load(p, blockIdx.x + issued * grid, sbase + (uint32_t)s * p.stage_bytes,
                                   full_bar(s));
                    ++issued;
                }
            }
            if (!ok) {
                atomicExch(p.status, 1);
                // Let the loads already issued land before the CTA's shared memory goes away.
                for (int64_t kk = k; kk < issued; ++kk) {
                    const uint32_t bar = full_bar((int)(kk % p.stages));
                    const uint32_t par = (uint32_t)((kk / p.stages) & 1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar, par) && global_timer_ns() - t0 < kSmWaitLimitNs) {
                    }
                }
            }
            bulk_wait_all();
        }
        __syncwarp();
        return;
    }

    // Compute warps 1 .. kSmWarps-1: thread c = tid - 32 owns the 16-byte vectors c, c + kSmCompute, ...
    const int c = tid - 32, cw = warp - 1;
    const float kMasked = dtype_min<BF16>();
    for (int64_t k = 0; k < my_rows; ++k) {
        const int s = (int)(k % p.stages);
        const bool landed = wait_bounded(full_bar(s), (uint32_t)((k / p.stages) & 1));
        if (!compute_bar_and(landed)) {
            if (c == 0) atomicExch(p.status, 1);
            return;
        }
        const int64_t r = blockIdx.x + k * grid;
        int64_t b, h, q;
        row_coords(p, r, b, h, q);
        const int64_t n_live = live_keys(p, q);
        const uint16_t* srow = reinterpret_cast<const uint16_t*>(smem + (size_t)s * p.stage_bytes);

        // Pass 1: the selected values in registers (pairs), and the row max.  32-bit indices
        // (K <= 32768); vectors wholly inside the live prefix need no select.
        const int K = p.K, nl = (int)n_live;
        float2 x[VPT * 4];
        float mc0 = -INFINITY, mc1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int e0 = 8 * (c + kSmCompute * j);
            if (e0 >= K) {
#pragma unroll
                for (int i = 0; i < 4; ++i) x[4 * j + i] = make_float2(-INFINITY, -INFINITY);   // no key
            } else if (e0 >= nl) {
#pragma unroll
                for (int i = 0; i < 4; ++i) x[4 * j + i] = make_float2(kMasked, kMasked);
                mc0 = fmaxf(mc0, kMasked);
            } else {
                const uint4 raw = *reinterpret_cast<const uint4*>(srow + e0);
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) x[4 * j + i] = to_f32x2<BF16>(w[i]);
                if (e0 + 8 > nl) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (e0 + 2 * i >= nl) x[4 * j + i].x = kMasked;
                        if (e0 + 2 * i + 1 >= nl) x[4 * j + i].y = kMasked;
                    }
                }
                mc0 = max3(mc0, x[4 * j].x, x[4 * j].y);
                mc1 = max3(mc1, x[4 * j + 1].x, x[4 * j + 1].y);
                mc0 = max3(mc0, x[4 * j + 2].x, x[4 * j + 2].y);
                mc1 = max3(mc1, x[4 * j + 3].x, x[4 * j + 3].y);
            }
        }
        float m = fmaxf(mc0, mc1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        if (lane == 0) red_max[cw] = m;
        compute_bar();
        m = red_max[0];
#pragma unroll
        for (int w = 1; w < kSmCompute / 32; ++w) m = fmaxf(m, red_max[w]);

        // Pass 2: e = 2^((x - m) log2 e) and the row sum, in a fixed order (two running sums
        // over the pairs' halves).  A vector wholly past the causal boundary holds
        // exp(finfo.min - m) = 0 unless the whole row is masked (m == finfo.min), where it is
        // computed like any other.
        const float2 nm2 = make_float2(-m, -m), l2e = make_float2(kSmLog2e, kSmLog2e);
        float2 sum2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int e0 = 8 * (c + kSmCompute * j);
            if (e0 >= K) continue;
            if (e0 >= nl && m != kMasked) {
#pragma unroll
                for (int i = 0; i < 4; ++i) x[4 * j + i] = make_float2(0.f, 0.f);
                continue;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 t = __fmul2_rn(__fadd2_rn(x[4 * j + i], nm2), l2e);
                const float2 e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                x[4 * j + i] = e;
                sum2 = __fadd2_rn(sum2, e);
            }
        }
        float sum = sum2.x + sum2.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFullMask, sum, o);
        if (lane == 0) red_sum[cw] = sum;
        compute_bar();
        sum = red_sum[0];
#pragma unroll
        for (int w = 1; w < kSmCompute / 32; ++w) sum += red_sum[w];
        const float inv = 1.0f / sum;
        const float2 inv2 = make_float2(inv, inv);

        // Pass 3: p = e / sum as 16-bit values over the buffer; the producer stores it.
        uint16_t* wrow = reinterpret_cast<uint16_t*>(smem + (size_t)s * p.stage_bytes);
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int e0 = 8 * (c + kSmCompute * j);
            if (e0 >= K) continue;
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 pr = __fmul2_rn(x[4 * j + i], inv2);
                w[i] = pack2<BF16>(pr.x, pr.y);
            }
            *reinterpret_cast<uint4*>(wrow + e0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive_warp(done_bar(s));
        // The next row's max reduction reuses red_max only after every warp read this one's
        // sum (they all passed the barrier above before any can pass the next one).
    }
}

template <bool BF16, int VPT>
cudaError_t launch_t(const SoftmaxParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = masked_softmax_kernel<BF16, VPT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kSmThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int masked_softmax_max_keys() { return 32768; }

cudaError_t launch_masked_softmax(SoftmaxParams p, bool bf16, int num_sms, cudaStream_t stream) {
    // Row buffers: as many as fit in 200 KiB, 2 to 8.
    p.stage_bytes = (uint32_t)(((int64_t)p.K * 2 + 127) & ~127ll);
    int stages = (int)((200 * 1024) / p.stage_bytes);
    stages = stages > 8 ? 8 : stages;
    if (stages < 2) return cudaErrorInvalidValue;
    p.stages = stages;
    if (!p.status) {
        void* addr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&addr, g_softmax_status);
        if (e != cudaSuccess) return e;
        p.status = static_cast<int32_t*>(addr);
    }
    const size_t smem = 128 + (size_t)stages * p.stage_bytes + 16 * stages + 2 * kSmWarps * sizeof(float);
    const int grid = (int)(p.rows < num_sms ? p.rows : num_sms);
    const int vpt_needed = (p.K + 8 * kSmCompute - 1) / (8 * kSmCompute);
#define FA_SM_CASE(V)                                                              \
    if (vpt_needed <= V)                                                           \
        return bf16 ? launch_t<true, V>(p, grid, smem, stream)                     \
                    : launch_t<false, V>(p, grid, smem, stream);
    FA_SM_CASE(1)
    FA_SM_CASE(2)
    FA_SM_CASE(3)
    FA_SM_CASE(5)
    FA_SM_CASE(9)
#undef FA_SM_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_masked_softmax_checked(const void* in, void* out, const int64_t in_stride[3],
                                          const int64_t out_stride[3], int B, int H, int Q, int K,
                                          int64_t offset, bool causal, bool bf16, int num_sms,
                                          int stall_loads, cudaStream_t stream) {
    SoftmaxParams p;
    p.stall_loads = stall_loads;
    p.in = static_cast<const uint16_t*>(in);
    p.out = static_cast<uint16_t*>(out);
    for (int i = 0; i < 3; ++i) {
        p.in_stride[i] = in_stride[i];
        p.out_stride[i] = out_stride[i];
    }
    p.B = B;
    p.H = H;
    p.Q = Q;
    p.K = K;
    p.offset = offset;
    p.causal = causal ? 1 : 0;
    p.rows = (int64_t)B * H * Q;
    p.stages = 0;
    p.stage_bytes = 0;
    p.status = nullptr;
    return launch_masked_softmax(p, bf16, num_sms, stream);
}

// Read and clear the status word of the masked-softmax kernels (1 = a bounded wait ran out).
cudaError_t masked_softmax_status(cudaStream_t stream, int32_t* out) {
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_softmax_status);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyAsync(out, addr, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *out != 0) {
        e = cudaMemsetAsync(addr, 0, 4, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    return e;
}

}  // namespace fa
