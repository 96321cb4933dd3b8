// noalloc.cu -- block-mask construction into caller-owned buffers, with no device allocation.
//
// Some callers cannot let a library call cudaMalloc: a framework whose caching allocator
// or arena already owns the device memory (an allocation behind its back escapes its
// accounting and can fail once the pool has reserved most of the GPU), a plugin of an
// inference runtime whose enqueue path must not allocate, or a real-time deployment that
// forbids allocation after start-up.  cudaMalloc can also synchronise the device, which a
// latency-critical caller cannot afford.  fa_create_block_mask_noalloc serves them: the
// caller passes the four output lists, and the only scratch the build needs -- per-block
// document statistics {min, max, uniform} -- lives in the fixed array below.
//
// The array is a file-scope __device__ variable, so every GPU that loads this library
// holds it (48 KiB) until the process exits.  Host code cannot use its name as a device
// address; the address is fetched once per device with cudaGetSymbolAddress and kept for
// the life of the process, so the entry point must not be used across a cudaDeviceReset
// (the module is reloaded then and the array may move).  All calls
// share the array and it keeps the last call's contents; every entry a call reads is
// written earlier by the same call, so nothing has to start at zero.  Two calls whose
// work overlaps on the GPU (for example on two streams) race on the array.
#include <mutex>

#include "fa_internal.h"

constexpr int kNoAllocMaxBlocks = 4096;  // query or kv blocks: Q_LEN, KV_LEN <= 524288

// Per-block document statistics of fa_create_block_mask_noalloc: 3 x 4096 int32 = 48 KiB.
static __device__ __align__(256) int32_t g_doc_stats_scratch[3 * kNoAllocMaxBlocks];

namespace fa {
// Defined in api.cu: FA_OK when ptr is memory of device dev, else FA_ERR_INVALID_ARG.
fa_status_t check_device_memory(const void* ptr, int dev, const char* name);
}  // namespace fa

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device `dev` (set up on first use).
fa_status_t scratch_address(int dev, int32_t** out) {
    if (dev < 0 || dev >= kMaxDevices)
        return fa::record_error(FA_ERR_UNSUPPORTED, "device ordinal beyond the no-alloc set-up table");
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_doc_stats_scratch);
        if (e != cudaSuccess || !p)
            return fa::record_error(FA_ERR_CUDA, "cudaGetSymbolAddress of the no-alloc scratch failed");
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_addr[dev];
    return FA_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" fa_status_t fa_create_block_mask_noalloc(
    uint32_t mask_kind, const fa_mask_params_t* params, int32_t B, int32_t H, int32_t Q_LEN,
    int32_t KV_LEN, int32_t BLOCK_SIZE, int32_t* kv_num_blocks, int32_t* kv_indices,
    int32_t* full_kv_num_blocks, int32_t* full_kv_indices, void* stream) {
    const uint32_t known = FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW | FA_MASK_DOCUMENT;
    if (mask_kind & ~known) return fa::record_error(FA_ERR_INVALID_ARG, "unknown mask_kind bits");
    if (B < 0 || H < 0) return fa::record_error(FA_ERR_INVALID_ARG, "B and H must be >= 0 (0 = broadcast)");
    if (Q_LEN <= 0 || KV_LEN <= 0)
        return fa::record_error(FA_ERR_INVALID_ARG, "Q_LEN and KV_LEN must be > 0");
    if (BLOCK_SIZE != fa::kBlock)
        return fa::record_error(FA_ERR_UNSUPPORTED, "BLOCK_SIZE: only 128 is implemented");
    if (!kv_num_blocks || !kv_indices || !full_kv_num_blocks || !full_kv_indices)
        return fa::record_error(FA_ERR_INVALID_ARG, "an output list pointer is NULL");
    if (!aligned4(kv_num_blocks) || !aligned4(kv_indices) || !aligned4(full_kv_num_blocks) ||
        !aligned4(full_kv_indices))
        return fa::record_error(FA_ERR_INVALID_ARG, "output lists must be 4-byte aligned");
    const int32_t window = params ? params->window : 0;
    const int32_t sep = params ? (params->separate_full_blocks ? 1 : 0) : 1;
    if ((mask_kind & FA_MASK_SLIDING_WINDOW) && window <= 0)
        return fa::record_error(FA_ERR_INVALID_ARG, "sliding window needs params->window > 0");
    if (mask_kind & FA_MASK_DOCUMENT) {
        if (!params || !params->doc_id)
            return fa::record_error(FA_ERR_INVALID_ARG, "document mask needs params->doc_id");
        if (Q_LEN != KV_LEN)
            return fa::record_error(FA_ERR_INVALID_ARG, "document mask needs Q_LEN == KV_LEN");
        if (!aligned4(params->doc_id))
            return fa::record_error(FA_ERR_INVALID_ARG, "doc_id must be 4-byte aligned");
    }
    const int QB = (Q_LEN + fa::kBlock - 1) / fa::kBlock;
    const int KVB = (KV_LEN + fa::kBlock - 1) / fa::kBlock;
    if (QB > kNoAllocMaxBlocks || KVB > kNoAllocMaxBlocks)
        return fa::record_error(FA_ERR_UNSUPPORTED,
                                "fa_create_block_mask_noalloc: Q_LEN and KV_LEN are limited to "
                                "4096 blocks of 128 (524288 positions) by its fixed scratch");
    const int Bm = B ? B : 1, Hm = H ? H : 1;
    if ((size_t)Bm * Hm > 65535)
        return fa::record_error(FA_ERR_UNSUPPORTED, "B*H of a non-broadcast mask above 65535");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fa::record_error(FA_ERR_CUDA, "cudaGetDevice failed");
    // The kernels write the four outputs and read doc_id directly: device memory only.
    fa_status_t s;
    if ((s = fa::check_device_memory(kv_num_blocks, dev, "kv_num_blocks")) != FA_OK ||
        (s = fa::check_device_memory(kv_indices, dev, "kv_indices")) != FA_OK ||
        (s = fa::check_device_memory(full_kv_num_blocks, dev, "full_kv_num_blocks")) != FA_OK ||
        (s = fa::check_device_memory(full_kv_indices, dev, "full_kv_indices")) != FA_OK)
        return s;
    if ((mask_kind & FA_MASK_DOCUMENT) &&
        (s = fa::check_device_memory(params->doc_id, dev, "doc_id")) != FA_OK)
        return s;
    int32_t* scratch = nullptr;
    s = scratch_address(dev, &scratch);
    if (s != FA_OK) return s;

    fa::MaskSpec spec;
    spec.kind = mask_kind;
    spec.window = window;
    spec.Q_LEN = Q_LEN;
    spec.KV_LEN = KV_LEN;
    spec.QB = QB;
    spec.KVB = KVB;
    spec.BQ = fa::kBlock;
    spec.BKV = fa::kBlock;
    spec.doc = (mask_kind & FA_MASK_DOCUMENT) ? params->doc_id : nullptr;
    spec.doc_stats = scratch;
    spec.doc_stats_kv = scratch;
    spec.kv_lens = nullptr;
    spec.maskH = Hm;
    e = fa::launch_mask_lists(spec, sep, Bm * Hm, kv_num_blocks, kv_indices, full_kv_num_blocks,
                              full_kv_indices, scratch, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fa::record_error(FA_ERR_CUDA, cudaGetErrorString(e));
    return fa::record_ok();
}
