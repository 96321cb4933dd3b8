// fa_trace.cuh -- optional phase tracer of the forward and backward kernels (compile-time FA_TRACE).
//
// Off by default: without FA_TRACE every trace point compiles to nothing.  The trace build
// (build.py --trace, libfa_b200_trace.so) records, for CTA 0 only, a 64-bit word per
// event: tag in bits 56-63 and the SM cycle counter in bits 0-55, into a caller-provided
// device buffer of kTraceSlots x kTraceCap words (one slot per recording warp).
#pragma once

#include <cstdint>

namespace fa {
constexpr int kTraceSlots = 24;
constexpr int kTraceCap = 16384;
}  // namespace fa

#ifdef FA_TRACE
// One per translation unit that includes this header (attn_fwd.cu, attn_bwd.cu), each with
// its own setter.
static __device__ unsigned long long* g_fa_trace = nullptr;
// Declares the role's trace cursor; the buffer pointer is read once, kept in a register.
#define FA_TRACE_DECL                                                                \
    unsigned long long* fa_tbuf_ = (blockIdx.x == 0) ? g_fa_trace : nullptr;         \
    int fa_tn_ = 0;
#define FA_TRACE_EV(slot, tag)                                                       \
    do {                                                                             \
        if (fa_tbuf_ && (threadIdx.x & 31) == 0 && fa_tn_ < fa::kTraceCap)           \
            fa_tbuf_[(slot) * fa::kTraceCap + fa_tn_] =                              \
                ((unsigned long long)(tag) << 56) | (clock64() & 0x00FFFFFFFFFFFFFFull); \
        ++fa_tn_;                                                                    \
    } while (0)
#else
#define FA_TRACE_DECL
#define FA_TRACE_EV(slot, tag) ((void)0)
#endif
