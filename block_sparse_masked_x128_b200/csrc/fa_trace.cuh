// fa_trace.cuh -- optional phase tracer of the forward kernel (compile-time FA_TRACE).
//
// Off by default: without FA_TRACE every trace point compiles to nothing.  The trace build
// (build.py --trace, libfa_b200_trace.so) records, for CTA 0 only, a 64-bit word per
// event: tag in bits 56-63 and the SM cycle counter in bits 0-55, into a caller-provided
// device buffer of kTraceSlots x kTraceCap words (one slot per recording warp).
#pragma once

#include <cstdint>

namespace fa {
constexpr int kTraceSlots = 16;
constexpr int kTraceCap = 16384;
}  // namespace fa

#ifdef FA_TRACE
// Defined in the one translation unit that includes this header (attn_fwd.cu).
static __device__ unsigned long long* g_fa_trace = nullptr;
__device__ __forceinline__ void fa_trace_event(int slot, int& n, int tag) {
    if (blockIdx.x == 0 && (threadIdx.x & 31) == 0 && g_fa_trace && n < fa::kTraceCap) {
        g_fa_trace[slot * fa::kTraceCap + n] =
            ((unsigned long long)tag << 56) | (clock64() & 0x00FFFFFFFFFFFFFFull);
    }
    ++n;
}
#define FA_TRACE_EV(slot, n, tag) fa_trace_event((slot), (n), (tag))
#else
#define FA_TRACE_EV(slot, n, tag) ((void)0)
#endif
