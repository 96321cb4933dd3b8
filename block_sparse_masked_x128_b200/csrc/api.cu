// api.cu -- the C ABI declared in include/fa_b200.h: argument checks, device memory of
// block masks, TMA descriptors, and kernel launches.  No compute happens on the host.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "fa_internal.h"

namespace {

// An NVTX range over a host entry point (what a profiler's timeline shows as the call that
// enqueued the kernels); costs a few nanoseconds when no tool listens.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

thread_local std::string g_last_error;
std::atomic<int> g_stall_loads{0};

fa_status_t fail(fa_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
fa_status_t fail(fa_status_t s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

fa_status_t ok() {
    g_last_error.clear();
    return FA_OK;
}

fa_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- driver entry point for TMA descriptors (no link-time dependency on libcuda)

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int sm_count(int device) {
    static int cache[64] = {0};
    if (device < 0 || device >= 64) return 0;
    if (cache[device] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) == cudaSuccess)
            cache[device] = n;
    }
    return cache[device];
}

// 4-D tiled map over a (B, H, S, D) tensor, box = 64 columns x 128 rows, 128-byte swizzle.
fa_status_t make_tmap(CUtensorMap* map, const fa_tensor_t* t, const char* name) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const CUtensorMapDataType dt = (t->dtype == FA_DTYPE_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    // A size-1 dimension's stride is irrelevant; give it a legal value.
    int64_t st_s = t->stride[2], st_h = t->stride[1], st_b = t->stride[0];
    if (t->S == 1) st_s = t->D;
    if (t->H == 1) st_h = st_s * t->S;
    if (t->B == 1) st_b = st_h * t->H;
    cuuint64_t dims[4] = {(cuuint64_t)t->D, (cuuint64_t)t->S, (cuuint64_t)t->H, (cuuint64_t)t->B};
    cuuint64_t strides[3] = {(cuuint64_t)st_s * 2, (cuuint64_t)st_h * 2, (cuuint64_t)st_b * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)fa::kBlock, 1, 1};
    cuuint32_t elem[4] = {1, 1, 1, 1};
    CUresult r = enc(map, dt, 4, t->data, dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", name, (int)r);
    return FA_OK;
}

fa_status_t check_tensor(const fa_tensor_t* t, const char* name) {
    if (!t) return fail(FA_ERR_INVALID_ARG, "%s is NULL", name);
    if (t->dtype != FA_DTYPE_F16 && t->dtype != FA_DTYPE_BF16)
        return fail(FA_ERR_INVALID_ARG, "%s.dtype %d is not FA_DTYPE_F16/BF16", name, t->dtype);
    if (t->B < 0 || t->H < 0 || t->S < 0 || t->D <= 0)
        return fail(FA_ERR_INVALID_ARG, "%s has a negative or zero extent", name);
    // An empty tensor (B, H or S of 0) may have no storage; nothing ever reads it.
    if (!t->data && t->B != 0 && t->H != 0 && t->S != 0)
        return fail(FA_ERR_INVALID_ARG, "%s.data is NULL", name);
    if (t->stride[3] != 1) return fail(FA_ERR_INVALID_ARG, "%s.stride[3] must be 1", name);
    for (int i = 0; i < 3; ++i)
        if (t->stride[i] <= 0 || (t->stride[i] % 8) != 0)
            return fail(FA_ERR_INVALID_ARG, "%s.stride[%d]=%lld must be a positive multiple of 8",
                        name, i, (long long)t->stride[i]);
    if ((reinterpret_cast<uintptr_t>(t->data) & 15u) != 0)
        return fail(FA_ERR_INVALID_ARG, "%s.data is not 16-byte aligned", name);
    return FA_OK;
}

// Hand the units of one (b, h) out together when the streamed K and V of all heads (2 tensors
// of B*H*KV_LEN*D 16-bit values) exceed half of the 126 MB L2.
bool head_major_order(int64_t BH, int64_t KV_LEN, int64_t D) {
    return BH * KV_LEN * D * 2 * 2 > (int64_t)64 * 1024 * 1024;
}

// Launch a forward-type kernel with a pair of unit counters of its own (the kernel's last CTA
// returns them to zero, also after a timeout).  The pairs are taken round robin; before a pair
// is reused, the stream waits (on the GPU) for the event recorded after its previous user, so
// however many forwards are enqueued on one mask, at most kSchedCtrSlots share the pairs at
// once and none ever shares a pair with another that is still running.  Under stream capture
// no event is recorded or waited on: a captured forward keeps the pair it was given for every
// replay, and the caller orders replays against other work on the same mask.
template <class Launch>
fa_status_t launch_with_counter_pair(fa_block_mask_t* m, cudaStream_t st, Launch&& launch) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    const bool capturing = cap != cudaStreamCaptureStatusNone;
    std::lock_guard<std::mutex> lock(m->ctr_mutex);
    const uint32_t slot = m->next_ctr++ % fa::kSchedCtrSlots;
    cudaEvent_t& ev = m->ctr_event[slot];
    if (!capturing) {
        if (ev) {
            e = cudaStreamWaitEvent(st, ev, 0);
            if (e != cudaSuccess) return cuda_fail(e, "waiting for the previous user of a counter pair");
        } else {
            e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
            if (e != cudaSuccess) {
                ev = nullptr;
                return cuda_fail(e, "cudaEventCreateWithFlags");
            }
        }
    }
    e = launch(m->sched_ctr + 2 * slot);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    if (!capturing) {
        e = cudaEventRecord(ev, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord after the forward");
    }
    return ok();
}

}  // namespace

namespace fa {
// Device memory of `dev` (cudaMalloc'd or managed); host and unregistered pointers are
// rejected.  Leaves no CUDA error pending.
fa_status_t check_device_memory(const void* ptr, int dev, const char* name) {
    cudaPointerAttributes a;
    const cudaError_t e = cudaPointerGetAttributes(&a, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(FA_ERR_INVALID_ARG, "%s is not a CUDA pointer (%s)", name, cudaGetErrorString(e));
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return fail(FA_ERR_INVALID_ARG, "%s is not device memory (memory type %d)", name, (int)a.type);
    if (a.device != dev)
        return fail(FA_ERR_INVALID_ARG, "%s lives on device %d, current is %d", name, a.device, dev);
    return FA_OK;
}

fa_status_t record_error(fa_status_t status, const char* message) {
    return fail(status, "%s", message);
}
fa_status_t record_ok() { return ok(); }
}  // namespace fa

extern "C" {

const char* fa_status_string(fa_status_t s) {
    switch (s) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
        case FA_ERR_CUDA: return "FA_ERR_CUDA";
        case FA_ERR_OOM: return "FA_ERR_OOM";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
        case FA_ERR_INTERNAL: return "FA_ERR_INTERNAL";
    }
    return "FA_ERR_UNKNOWN";
}

const char* fa_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"

namespace {

// Checks shared by the mask constructors; fills the stored extents.
fa_status_t check_mask_args(uint32_t mask_kind, const fa_mask_params_t* params, int32_t B, int32_t H,
                            int32_t Q_LEN, int32_t KV_LEN) {
    const uint32_t known = FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW | FA_MASK_DOCUMENT;
    if (mask_kind & ~known) return fail(FA_ERR_INVALID_ARG, "unknown mask_kind bits 0x%x", mask_kind);
    if (B < 0 || H < 0) return fail(FA_ERR_INVALID_ARG, "B and H must be >= 0 (0 = broadcast)");
    if (Q_LEN <= 0 || KV_LEN <= 0) return fail(FA_ERR_INVALID_ARG, "Q_LEN and KV_LEN must be > 0");
    const int32_t window = params ? params->window : 0;
    if ((mask_kind & FA_MASK_SLIDING_WINDOW) && window <= 0)
        return fail(FA_ERR_INVALID_ARG, "sliding window needs params->window > 0");
    if (mask_kind & FA_MASK_DOCUMENT) {
        if (!params || !params->doc_id) return fail(FA_ERR_INVALID_ARG, "document mask needs params->doc_id");
        if (Q_LEN != KV_LEN) return fail(FA_ERR_INVALID_ARG, "document mask needs Q_LEN == KV_LEN");
    }
    if (params && params->kv_lens && B <= 0)
        return fail(FA_ERR_INVALID_ARG, "per-batch kv_lens need B > 0 (one mask per batch element)");
    const int QB = (Q_LEN + fa::kBlock - 1) / fa::kBlock;
    const int KVB = (KV_LEN + fa::kBlock - 1) / fa::kBlock;
    if (QB > fa::kMaxBlocks || KVB > fa::kMaxBlocks)
        return fail(FA_ERR_UNSUPPORTED, "more than %d blocks per side", fa::kMaxBlocks);
    if ((size_t)(B ? B : 1) * (H ? H : 1) > 65535)
        return fail(FA_ERR_UNSUPPORTED, "B*H of a non-broadcast mask above 65535");
    return FA_OK;
}

// One device allocation for every array of a mask: the kernel's 128 x 128 lists, the caller's
// lists at block size BQ x BKV when that differs from 128 (or when `own_user_lists`), the
// unit schedule, the backward metadata, the status word and the counter pairs.  Copies
// doc_id (padded to whole blocks) on `st`.  On success *out holds the new mask.
fa_status_t allocate_mask(uint32_t mask_kind, const fa_mask_params_t* params, int32_t B, int32_t H,
                          int32_t Q_LEN, int32_t KV_LEN, int32_t BQ, int32_t BKV, bool own_user_lists,
                          cudaStream_t st, fa_block_mask_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const int32_t window = params ? params->window : 0;
    const int32_t sep = params ? (params->separate_full_blocks ? 1 : 0) : 1;
    const int QB = (Q_LEN + fa::kBlock - 1) / fa::kBlock;
    const int KVB = (KV_LEN + fa::kBlock - 1) / fa::kBlock;
    const int UQB = (Q_LEN + BQ - 1) / BQ, UKVB = (KV_LEN + BKV - 1) / BKV;
    const bool user = own_user_lists || BQ != fa::kBlock || BKV != fa::kBlock;
    const int Bm = B ? B : 1, Hm = H ? H : 1;
    const int NP = (QB + 1) / 2;
    const size_t BH = (size_t)Bm * Hm;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    const size_t o_kvn = take(BH * QB * 4), o_kvi = take(BH * QB * KVB * 4);
    const size_t o_fn = take(BH * QB * 4), o_fi = take(BH * QB * KVB * 4);
    const bool has_doc = (mask_kind & FA_MASK_DOCUMENT) != 0;
    // The copy of doc_id is padded to whole blocks (the kernels read ids by 128-key tile).
    const size_t doc_pad = (size_t)KVB * fa::kBlock;
    const size_t o_doc = take(has_doc ? doc_pad * 4 : 0);
    const bool has_lens = params && params->kv_lens;
    const size_t o_lens = take(has_lens ? (size_t)Bm * 4 : 0);
    // Document statistics: 128-blocks, then (when the caller's block sizes differ) its blocks.
    const size_t o_dst = take(has_doc ? (size_t)(QB > KVB ? QB : KVB) * 3 * 4 : 0);
    const size_t o_udst = take((has_doc && user) ? (size_t)(UQB + UKVB) * 3 * 4 : 0);
    const size_t o_sc = take(BH * NP * 8), o_scost = take(BH * NP * 4);
    const size_t o_se = take(BH * NP * KVB * 4), o_so = take(BH * NP * 4);
    const bool global_order = BH * NP <= (size_t)fa::kGlobalOrderMax;
    const size_t o_sgo = take(global_order ? BH * NP * 4 : 0);
    const size_t n_kv = BH * KVB, n_q = BH * QB, n_tiles = BH * QB * KVB;
    const size_t o_qn = take(n_kv * 4), o_qi = take(n_tiles * 4), o_fqn = take(n_kv * 4),
                 o_fqi = take(n_tiles * 4);
    const size_t o_kvc = take(n_kv * 4), o_kvcost = take(n_kv * 4), o_kve = take(n_tiles * 4),
                 o_kvo = take(n_kv * 4);
    const size_t o_dqc = take(n_q * 4), o_dqcost = take(n_q * 4), o_dqe = take(n_tiles * 4),
                 o_dqo = take(n_q * 4);
    const size_t u_rows = user ? BH * UQB : 0, u_cols = user ? BH * UKVB : 0;
    const size_t u_tiles = user ? BH * (size_t)UQB * UKVB : 0;
    const size_t o_ukvn = take(u_rows * 4), o_ukvi = take(u_tiles * 4), o_ufn = take(u_rows * 4),
                 o_ufi = take(u_tiles * 4);
    const size_t o_uqn = take(u_cols * 4), o_uqi = take(u_tiles * 4), o_ufqn = take(u_cols * 4),
                 o_ufqi = take(u_tiles * 4);
    // Status word, then the unit counters of the kernels (two words per slot), all zero.
    const size_t ctr_bytes = 4 + (size_t)fa::kSchedCtrSlots * 8;
    const size_t o_status = take(ctr_bytes);
    void* base = nullptr;
    e = cudaMalloc(&base, off);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(FA_ERR_OOM, "cudaMalloc(%zu) for the block mask: %s", off, cudaGetErrorString(e));
    }
    fa_block_mask_t* m = new fa_block_mask_t();
    m->mask_kind = mask_kind;
    m->window = window;
    m->separate_full = sep;
    m->B = Bm;
    m->H = Hm;
    m->Q_LEN = Q_LEN;
    m->KV_LEN = KV_LEN;
    m->QB = QB;
    m->KVB = KVB;
    m->NP = NP;
    m->device = dev;
    m->dev_base = base;
    char* b8 = static_cast<char*>(base);
    auto at = [&](size_t o) { return reinterpret_cast<int32_t*>(b8 + o); };
    m->kv_num = at(o_kvn);
    m->kv_idx = at(o_kvi);
    m->full_num = at(o_fn);
    m->full_idx = at(o_fi);
    m->doc = has_doc ? at(o_doc) : nullptr;
    m->doc_stats = has_doc ? at(o_dst) : nullptr;
    m->kv_lens = has_lens ? at(o_lens) : nullptr;
    m->sched_count = at(o_sc);
    m->sched_cost = at(o_scost);
    m->sched_entries = at(o_se);
    m->sched_order = at(o_so);
    m->sched_gorder = global_order ? at(o_sgo) : nullptr;
    m->dq_kv_order = params ? (params->dq_kv_order ? 1 : 0) : 1;
    m->bwd = fa::BwdMeta{at(o_qn),  at(o_qi),     at(o_fqn), at(o_fqi), at(o_kvc),    at(o_kvcost),
                         at(o_kve), at(o_kvo),    at(o_dqc), at(o_dqcost), at(o_dqe), at(o_dqo)};
    m->BQ = BQ;
    m->BKV = BKV;
    m->UQB = UQB;
    m->UKVB = UKVB;
    if (user) {
        m->u_kv_num = at(o_ukvn);
        m->u_kv_idx = at(o_ukvi);
        m->u_full_num = at(o_ufn);
        m->u_full_idx = at(o_ufi);
        m->u_q_num = at(o_uqn);
        m->u_q_idx = at(o_uqi);
        m->u_fq_num = at(o_ufqn);
        m->u_fq_idx = at(o_ufqi);
        m->u_doc_stats = (has_doc) ? at(o_udst) : nullptr;
    } else {
        m->u_kv_num = m->kv_num;
        m->u_kv_idx = m->kv_idx;
        m->u_full_num = m->full_num;
        m->u_full_idx = m->full_idx;
        m->u_q_num = m->bwd.q_num;
        m->u_q_idx = m->bwd.q_idx;
        m->u_fq_num = m->bwd.fq_num;
        m->u_fq_idx = m->bwd.fq_idx;
        m->u_doc_stats = nullptr;
    }
    m->status = at(o_status);
    m->sched_ctr = m->status + 1;
    if ((e = cudaMemsetAsync(m->status, 0, ctr_bytes, st)) != cudaSuccess ||
        (has_doc && (e = cudaMemcpyAsync(m->doc, params->doc_id, (size_t)KV_LEN * 4, cudaMemcpyDefault, st)) !=
                        cudaSuccess) ||
        (has_doc && doc_pad > (size_t)KV_LEN &&
         (e = cudaMemsetAsync(m->doc + KV_LEN, 0, (doc_pad - KV_LEN) * 4, st)) != cudaSuccess) ||
        (has_lens && (e = cudaMemcpyAsync(m->kv_lens, params->kv_lens, (size_t)Bm * 4, cudaMemcpyDefault,
                                          st)) != cudaSuccess)) {
        cudaStreamSynchronize(st);
        cudaFree(base);
        delete m;
        return cuda_fail(e, "mask set-up copies");
    }
    *out = m;
    return FA_OK;
}

void release_mask(fa_block_mask_t* m, cudaStream_t st) {
    cudaStreamSynchronize(st);
    cudaFree(m->dev_base);
    delete m;
}

// The schedule of the forward and the backward metadata, from the kernel's 128 x 128 lists.
cudaError_t build_derived(fa_block_mask_t* m, cudaStream_t st) {
    const int BH = m->B * m->H;
    cudaError_t e = fa::launch_schedule(m->QB, m->KVB, BH, m->NP, m->kv_num, m->kv_idx, m->full_num,
                                        m->full_idx, m->sched_count, m->sched_cost, m->sched_entries,
                                        m->sched_order, st);
    if (e != cudaSuccess) return e;
    if (m->sched_gorder) e = fa::launch_global_order(BH * m->NP, m->sched_cost, m->sched_gorder, st);
    if (e != cudaSuccess) return e;
    return fa::launch_backward_metadata(m->QB, m->KVB, BH, m->dq_kv_order, m->kv_num, m->kv_idx,
                                        m->full_num, m->full_idx, m->bwd, st);
}

fa::MaskSpec mask_spec(const fa_block_mask_t* m, int BQ, int BKV) {
    fa::MaskSpec spec;
    spec.kind = m->mask_kind;
    spec.window = m->window;
    spec.Q_LEN = m->Q_LEN;
    spec.KV_LEN = m->KV_LEN;
    spec.BQ = BQ;
    spec.BKV = BKV;
    spec.QB = (m->Q_LEN + BQ - 1) / BQ;
    spec.KVB = (m->KV_LEN + BKV - 1) / BKV;
    spec.doc = m->doc;
    spec.doc_stats = nullptr;
    spec.doc_stats_kv = nullptr;
    spec.kv_lens = m->kv_lens;
    spec.maskH = m->H;
    return spec;
}

}  // namespace

extern "C" {

fa_status_t fa_create_block_mask(uint32_t mask_kind, const fa_mask_params_t* params, int32_t B,
                                 int32_t H, int32_t Q_LEN, int32_t KV_LEN, int32_t BLOCK_SIZE,
                                 void* stream, fa_block_mask_t** out_mask) {
    NvtxRange nvtx_range("fa_create_block_mask");
    if (!out_mask) return fail(FA_ERR_INVALID_ARG, "out_mask is NULL");
    *out_mask = nullptr;
    fa_status_t s = check_mask_args(mask_kind, params, B, H, Q_LEN, KV_LEN);
    if (s != FA_OK) return s;
    const int32_t BQ = BLOCK_SIZE;
    const int32_t BKV = (params && params->kv_block_size > 0) ? params->kv_block_size : BLOCK_SIZE;
    if (BQ <= 0 || BKV <= 0 || (params && params->kv_block_size < 0))
        return fail(FA_ERR_INVALID_ARG, "block sizes must be positive");
    if ((Q_LEN + BQ - 1) / BQ > fa::kMaxBlocks || (KV_LEN + BKV - 1) / BKV > fa::kMaxBlocks)
        return fail(FA_ERR_UNSUPPORTED, "more than %d blocks per side", fa::kMaxBlocks);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    fa_block_mask_t* m = nullptr;
    if ((s = allocate_mask(mask_kind, params, B, H, Q_LEN, KV_LEN, BQ, BKV, false, st, &m)) != FA_OK)
        return s;
    const int BH = m->B * m->H;
    // The kernel's 128 x 128 lists, then everything derived from them.
    cudaError_t e = fa::launch_mask_lists(mask_spec(m, fa::kBlock, fa::kBlock), m->separate_full, BH,
                                          m->kv_num, m->kv_idx, m->full_num, m->full_idx,
                                          m->doc_stats, st);
    if (e == cudaSuccess) e = build_derived(m, st);
    // The caller's lists at its own block size, and their transposes.
    if (e == cudaSuccess && m->u_kv_num != m->kv_num) {
        const fa::MaskSpec us = mask_spec(m, BQ, BKV);
        e = fa::launch_mask_lists(us, m->separate_full, BH, m->u_kv_num, m->u_kv_idx, m->u_full_num,
                                  m->u_full_idx, m->u_doc_stats, st);
        if (e == cudaSuccess)
            e = fa::launch_transpose_lists(us.QB, us.KVB, BH, m->u_kv_num, m->u_kv_idx, m->u_full_num,
                                           m->u_full_idx, m->u_q_num, m->u_q_idx, m->u_fq_num,
                                           m->u_fq_idx, st);
    }
    if (e != cudaSuccess) {
        release_mask(m, st);
        return cuda_fail(e, "mask-builder launch");
    }
    *out_mask = m;
    return ok();
}

fa_status_t fa_block_mask_from_kv_blocks(uint32_t mask_kind, const fa_mask_params_t* params, int32_t B,
                                         int32_t H, int32_t Q_LEN, int32_t KV_LEN, int32_t Q_BLOCK,
                                         int32_t KV_BLOCK, const int32_t* kv_num_blocks,
                                         const int32_t* kv_indices, const int32_t* full_kv_num_blocks,
                                         const int32_t* full_kv_indices, void* stream,
                                         fa_block_mask_t** out_mask) {
    NvtxRange nvtx_range("fa_block_mask_from_kv_blocks");
    if (!out_mask) return fail(FA_ERR_INVALID_ARG, "out_mask is NULL");
    *out_mask = nullptr;
    fa_status_t s = check_mask_args(mask_kind, params, B, H, Q_LEN, KV_LEN);
    if (s != FA_OK) return s;
    if (Q_BLOCK <= 0 || KV_BLOCK <= 0 || (Q_BLOCK % fa::kBlock) != 0 || (KV_BLOCK % fa::kBlock) != 0)
        return fail(FA_ERR_UNSUPPORTED, "block sizes (%d, %d): caller lists need multiples of 128",
                    Q_BLOCK, KV_BLOCK);
    if (!kv_num_blocks || !kv_indices) return fail(FA_ERR_INVALID_ARG, "kv_num_blocks and kv_indices are required");
    if ((full_kv_num_blocks == nullptr) != (full_kv_indices == nullptr))
        return fail(FA_ERR_INVALID_ARG, "full_kv_num_blocks and full_kv_indices go together");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if ((s = fa::check_device_memory(kv_num_blocks, dev, "kv_num_blocks")) != FA_OK ||
        (s = fa::check_device_memory(kv_indices, dev, "kv_indices")) != FA_OK)
        return s;
    if (full_kv_num_blocks &&
        ((s = fa::check_device_memory(full_kv_num_blocks, dev, "full_kv_num_blocks")) != FA_OK ||
         (s = fa::check_device_memory(full_kv_indices, dev, "full_kv_indices")) != FA_OK))
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    fa_block_mask_t* m = nullptr;
    if ((s = allocate_mask(mask_kind, params, B, H, Q_LEN, KV_LEN, Q_BLOCK, KV_BLOCK, true, st, &m)) != FA_OK)
        return s;
    const int BH = m->B * m->H;
    const size_t rows = (size_t)BH * m->UQB, tiles = rows * m->UKVB;
    // The caller's lists, kept as given (read back by fa_block_mask_get); no full lists = none.
    e = cudaMemcpyAsync(m->u_kv_num, kv_num_blocks, rows * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(m->u_kv_idx, kv_indices, tiles * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
        e = full_kv_num_blocks ? cudaMemcpyAsync(m->u_full_num, full_kv_num_blocks, rows * 4, cudaMemcpyDeviceToDevice, st)
                               : cudaMemsetAsync(m->u_full_num, 0, rows * 4, st);
    if (e == cudaSuccess)
        e = full_kv_indices ? cudaMemcpyAsync(m->u_full_idx, full_kv_indices, tiles * 4, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(m->u_full_idx, 0, tiles * 4, st);
    // The kernel's 128 x 128 lists by expanding each block into its tiles.
    if (e == cudaSuccess)
        e = fa::launch_expand_block_lists(m->UQB, m->UKVB, Q_BLOCK / fa::kBlock, KV_BLOCK / fa::kBlock,
                                          m->QB, m->KVB, Q_LEN, KV_LEN, m->kv_lens, m->H, BH,
                                          m->separate_full,
                                          m->u_kv_num, m->u_kv_idx, m->u_full_num, m->u_full_idx,
                                          m->kv_num, m->kv_idx, m->full_num, m->full_idx, m->status, st);
    if (e == cudaSuccess) e = build_derived(m, st);
    if (e == cudaSuccess)
        e = fa::launch_transpose_lists(m->UQB, m->UKVB, BH, m->u_kv_num, m->u_kv_idx, m->u_full_num,
                                       m->u_full_idx, m->u_q_num, m->u_q_idx, m->u_fq_num, m->u_fq_idx, st);
    if (e != cudaSuccess) {
        release_mask(m, st);
        return cuda_fail(e, "block-list expansion launch");
    }
    *out_mask = m;
    return ok();
}

fa_status_t fa_block_mask_get(const fa_block_mask_t* m, fa_block_mask_info_t* info) {
    if (!m || !info) return fail(FA_ERR_INVALID_ARG, "NULL argument");
    info->B = m->B;
    info->H = m->H;
    info->Q_LEN = m->Q_LEN;
    info->KV_LEN = m->KV_LEN;
    info->BLOCK_SIZE = m->BQ;
    info->q_blocks = m->UQB;
    info->kv_blocks = m->UKVB;
    info->mask_kind = m->mask_kind;
    info->window = m->window;
    info->separate_full_blocks = m->separate_full;
    info->kv_num_blocks = m->u_kv_num;
    info->kv_indices = m->u_kv_idx;
    info->full_kv_num_blocks = m->u_full_num;
    info->full_kv_indices = m->u_full_idx;
    info->q_num_blocks = m->u_q_num;
    info->q_indices = m->u_q_idx;
    info->full_q_num_blocks = m->u_fq_num;
    info->full_q_indices = m->u_fq_idx;
    info->dq_kv_order = m->dq_kv_order;
    info->KV_BLOCK_SIZE = m->BKV;
    return ok();
}

void fa_destroy_block_mask(fa_block_mask_t* m) {
    if (!m) return;
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != m->device) cudaSetDevice(m->device);
    for (cudaEvent_t ev : m->ctr_event)
        if (ev) cudaEventDestroy(ev);
    cudaFree(m->dev_base);
    if (cur != m->device) cudaSetDevice(cur);
    delete m;
}

fa_status_t fa_get_device_status(const fa_block_mask_t* m, void* stream) {
    if (!m) return fail(FA_ERR_INVALID_ARG, "block_mask is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, m->status, 4, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (h != 0) {
        e = cudaMemsetAsync(m->status, 0, 4, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
        if (h == 2)
            return fail(FA_ERR_INVALID_ARG, "the caller's block lists held a count or index outside the block grid");
        if (h == fa::kStatusBadIndex)
            return fail(FA_ERR_INTERNAL, "a kernel met a metadata index out of range (debug build check)");
        return fail(FA_ERR_TIMEOUT, "a device-side wait ran past its limit (status %d)", h);
    }
    return ok();
}

}  // extern "C"

namespace {

// The forward of fa_forward and fa_forward_paged.  With a page table, k and v are page pools
// (n_pages, H, 128, D) and the mask's KV_LEN is the logical context length.
// Split decode: tiles per CTA so that about 32 CTAs per SM (four waves of 8 resident CTAs)
// share the (b, h)'s tiles.  Short chunks keep the last wave short when the sequences'
// lengths differ (measured on 1k-8k contexts: 8 CTAs per SM 0.71 of the copy bandwidth,
// 16 0.77, 32 0.81, 64 0.75, where the merge's partials start to cost).
void decode_chunking(int KVB, int64_t BH, int nsm, int& tiles_per_chunk, int& max_chunks) {
    const int64_t target = 32 * (int64_t)(nsm > 0 ? nsm : 148);
    const int64_t per_bh = (target + BH - 1) / BH;
    int64_t tpc = (KVB + per_bh - 1) / per_bh;
    if (tpc < 1) tpc = 1;
    tiles_per_chunk = (int)tpc;
    max_chunks = (int)((KVB + tpc - 1) / tpc);
}

fa_status_t forward_impl(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                         const int32_t* page_table, int64_t page_stride, const fa_block_mask_t* m,
                         uint32_t score_mod_kind, const fa_score_params_t* params, float scale,
                         fa_tensor_t* out, float* lse, void* stream, bool check_only = false) {
    fa_status_t s;
    if ((s = check_tensor(q, "q")) != FA_OK) return s;
    if ((s = check_tensor(k, "k")) != FA_OK) return s;
    if ((s = check_tensor(v, "v")) != FA_OK) return s;
    if ((s = check_tensor(out, "out")) != FA_OK) return s;
    if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype)
        return fail(FA_ERR_INVALID_ARG, "q, k, v and out must share one dtype");
    if ((!page_table && (k->B != q->B || v->B != q->B)) || k->B != v->B || out->B != q->B ||
        k->H != q->H || v->H != q->H || out->H != q->H)
        return fail(FA_ERR_INVALID_ARG, "q, k, v and out must share B and H");
    if (page_table) {
        if (k->S != fa::kBlock || v->S != fa::kBlock)
            return fail(FA_ERR_INVALID_ARG, "paged k and v must be (n_pages, H, 128, D) pools");
        if (k->B <= 0 || k->B > 0x7fffffffLL) return fail(FA_ERR_INVALID_ARG, "page pools must hold pages");
        if (page_stride < m->KVB)
            return fail(FA_ERR_INVALID_ARG, "page_table_stride %lld below the mask's %d kv blocks",
                        (long long)page_stride, m->KVB);
    }
    if (k->D != q->D || v->D != q->D || out->D != q->D)
        return fail(FA_ERR_INVALID_ARG, "q, k, v and out must share D");
    if (k->S != v->S) return fail(FA_ERR_INVALID_ARG, "k and v must share S");
    if (out->S != q->S) return fail(FA_ERR_INVALID_ARG, "out must have q's S");
    if (q->D != 64 && q->D != 128)
        return fail(FA_ERR_UNSUPPORTED, "head_dim %lld: only 64 and 128 are implemented", (long long)q->D);
    const uint32_t known = FA_SCORE_SOFTCAP | FA_SCORE_ALIBI;
    if (score_mod_kind & ~known) return fail(FA_ERR_INVALID_ARG, "unknown score_mod_kind bits 0x%x", score_mod_kind);
    if ((score_mod_kind & FA_SCORE_SOFTCAP) && (!params || !(params->softcap > 0.f)))
        return fail(FA_ERR_INVALID_ARG, "soft-cap needs params->softcap > 0");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
        return fail(FA_ERR_INVALID_ARG, "lse is not 4-byte aligned");
    if (!m) return fail(FA_ERR_INVALID_ARG, "block_mask is NULL");
    if (q->S != m->Q_LEN || (!page_table && k->S != m->KV_LEN))
        return fail(FA_ERR_INVALID_ARG, "q/k lengths (%lld, %lld) differ from the mask's (%d, %d)",
                    (long long)q->S, (long long)k->S, m->Q_LEN, m->KV_LEN);
    if (!(m->B == 1 || m->B == q->B) || !(m->H == 1 || m->H == q->H))
        return fail(FA_ERR_INVALID_ARG, "mask B/H (%d, %d) neither broadcast nor equal to q's", m->B, m->H);
    if ((int64_t)m->NP * q->B * q->H > 0x7fffffffLL)
        return fail(FA_ERR_UNSUPPORTED, "too many work units");
    if (q->B == 0 || q->H == 0 || q->S == 0) return ok();

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != m->device) return fail(FA_ERR_INVALID_ARG, "block_mask lives on device %d, current is %d", m->device, dev);
    // Every buffer the kernel touches must be memory of this device (a host pointer would
    // make the kernel fault instead of returning an error).
    if ((s = fa::check_device_memory(q->data, dev, "q")) != FA_OK) return s;
    if ((s = fa::check_device_memory(k->data, dev, "k")) != FA_OK) return s;
    if ((s = fa::check_device_memory(v->data, dev, "v")) != FA_OK) return s;
    if ((s = fa::check_device_memory(out->data, dev, "out")) != FA_OK) return s;
    if (lse && (s = fa::check_device_memory(lse, dev, "lse")) != FA_OK) return s;
    if (params && params->alibi_slopes &&
        (s = fa::check_device_memory(params->alibi_slopes, dev, "alibi_slopes")) != FA_OK)
        return s;
    if (page_table && (s = fa::check_device_memory(page_table, dev, "page_table")) != FA_OK) return s;

    if (check_only) return FA_OK;
    CUtensorMap tq, tk, tv;
    if ((s = make_tmap(&tq, q, "q")) != FA_OK) return s;
    if ((s = make_tmap(&tk, k, "k")) != FA_OK) return s;
    if ((s = make_tmap(&tv, v, "v")) != FA_OK) return s;

    const float sc = (scale > 0.f) ? scale : (float)(1.0 / std::sqrt((double)q->D));
    fa::FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = (int32_t)q->B;
    p.H = (int32_t)q->H;
    p.Q_LEN = m->Q_LEN;
    p.KV_LEN = m->KV_LEN;
    p.QB = m->QB;
    p.KVB = m->KVB;
    p.NP = m->NP;
    p.maskB = m->B;
    p.maskH = m->H;
    p.n_units = (int32_t)((int64_t)m->NP * q->B * q->H);
    p.head_major = head_major_order(q->B * q->H, k->S, q->D) ? 1 : 0;
    p.mask_kind = m->mask_kind;
    p.window = m->window;
    p.score_kind = score_mod_kind;
    p.doc_id = m->doc;
    p.kv_lens = m->kv_lens;
    p.page_table = page_table;
    p.page_stride = (int32_t)(page_table ? page_stride : 0);
    p.n_pages = (int32_t)(page_table ? k->B : 0);
    p.sched_order = m->sched_order;
    p.sched_gorder = m->sched_gorder;
    p.sched_count = m->sched_count;
    p.sched_entries = m->sched_entries;
    p.scale = sc;
    p.scale_log2 = sc * 1.4426950408889634f;
    const float cap = (score_mod_kind & FA_SCORE_SOFTCAP) ? params->softcap : 1.f;
    p.softcap = cap;
    p.softcap_log2 = cap * 1.4426950408889634f;
    p.inv_softcap_scale = sc / cap;
    p.alibi_slopes = params ? params->alibi_slopes : nullptr;
    p.out = out->data;
    p.out_stride[0] = out->stride[0];
    p.out_stride[1] = out->stride[1];
    p.out_stride[2] = out->stride[2];
    p.lse = lse;
    p.status = m->status;
    p.stall_loads = g_stall_loads.load(std::memory_order_relaxed);

    const int nsm = sm_count(dev);
    if (nsm <= 0) return fail(FA_ERR_CUDA, "could not read the SM count");
    const int grid = p.n_units < nsm ? p.n_units : nsm;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launch_with_counter_pair(const_cast<fa_block_mask_t*>(m), st, [&](int32_t* ctr) {
        p.sched_ctr = ctr;
        return fa::launch_attn_fwd(p, (int)q->D, q->dtype == FA_DTYPE_BF16, (int)score_mod_kind,
                                   tq, tk, tv, grid, st);
    });
}

}  // namespace

extern "C" {

size_t fa_backward_workspace_bytes(int64_t B, int64_t H, int64_t Q_LEN) {
    if (B <= 0 || H <= 0 || Q_LEN <= 0) return 0;
    const int64_t q_pad = (Q_LEN + fa::kBlock - 1) / fa::kBlock * fa::kBlock;
    return (size_t)(2 * B * H * q_pad * 4);
}

fa_status_t fa_backward(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                        const fa_tensor_t* out, const fa_tensor_t* dout, const float* lse,
                        const fa_block_mask_t* m, uint32_t score_mod_kind,
                        const fa_score_params_t* params, float scale, fa_tensor_t* dq,
                        fa_tensor_t* dk, fa_tensor_t* dv, void* workspace, size_t workspace_bytes,
                        void* stream) {
    NvtxRange nvtx_range("fa_backward");
    fa_status_t s;
    const fa_tensor_t* all[8] = {q, k, v, out, dout, dq, dk, dv};
    const char* names[8] = {"q", "k", "v", "out", "dout", "dq", "dk", "dv"};
    for (int i = 0; i < 8; ++i)
        if ((s = check_tensor(all[i], names[i])) != FA_OK) return s;
    for (int i = 1; i < 8; ++i)
        if (all[i]->dtype != q->dtype) return fail(FA_ERR_INVALID_ARG, "%s has another dtype than q", names[i]);
    for (int i = 1; i < 8; ++i)
        if (all[i]->B != q->B || all[i]->H != q->H || all[i]->D != q->D)
            return fail(FA_ERR_INVALID_ARG, "%s must share q's B, H and D", names[i]);
    if (k->S != v->S || dk->S != k->S || dv->S != k->S)
        return fail(FA_ERR_INVALID_ARG, "k, v, dk and dv must share one length");
    if (out->S != q->S || dout->S != q->S || dq->S != q->S)
        return fail(FA_ERR_INVALID_ARG, "out, dout and dq must have q's length");
    if (q->D != 64 && q->D != 128)
        return fail(FA_ERR_UNSUPPORTED, "head_dim %lld: only 64 and 128 are implemented", (long long)q->D);
    const uint32_t known = FA_SCORE_SOFTCAP | FA_SCORE_ALIBI;
    if (score_mod_kind & ~known) return fail(FA_ERR_INVALID_ARG, "unknown score_mod_kind bits 0x%x", score_mod_kind);
    if ((score_mod_kind & FA_SCORE_SOFTCAP) && (!params || !(params->softcap > 0.f)))
        return fail(FA_ERR_INVALID_ARG, "soft-cap needs params->softcap > 0");
    const bool empty = q->B == 0 || q->H == 0 || q->S == 0 || k->S == 0;   // nothing to compute
    if ((!lse && !empty) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return fail(FA_ERR_INVALID_ARG, "lse must be a 4-byte aligned device pointer");
    if (!m) return fail(FA_ERR_INVALID_ARG, "block_mask is NULL");
    if (q->S != m->Q_LEN || k->S != m->KV_LEN)
        return fail(FA_ERR_INVALID_ARG, "q/k lengths (%lld, %lld) differ from the mask's (%d, %d)",
                    (long long)q->S, (long long)k->S, m->Q_LEN, m->KV_LEN);
    if (!(m->B == 1 || m->B == q->B) || !(m->H == 1 || m->H == q->H))
        return fail(FA_ERR_INVALID_ARG, "mask B/H (%d, %d) neither broadcast nor equal to q's", m->B, m->H);
    if ((int64_t)(m->QB > m->KVB ? m->QB : m->KVB) * q->B * q->H > 0x7fffffffLL)
        return fail(FA_ERR_UNSUPPORTED, "too many work units");
    if (empty) return ok();
    const size_t need = fa_backward_workspace_bytes(q->B, q->H, q->S);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15u))
        return fail(FA_ERR_INVALID_ARG, "workspace must be 16-byte aligned device memory of at least %zu bytes", need);

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != m->device) return fail(FA_ERR_INVALID_ARG, "block_mask lives on device %d, current is %d", m->device, dev);
    for (int i = 0; i < 8; ++i)
        if ((s = fa::check_device_memory(all[i]->data, dev, names[i])) != FA_OK) return s;
    if ((s = fa::check_device_memory(lse, dev, "lse")) != FA_OK) return s;
    if ((s = fa::check_device_memory(workspace, dev, "workspace")) != FA_OK) return s;
    if (params && params->alibi_slopes &&
        (s = fa::check_device_memory(params->alibi_slopes, dev, "alibi_slopes")) != FA_OK)
        return s;
    CUtensorMap tq, tk, tv, tdo;
    if ((s = make_tmap(&tq, q, "q")) != FA_OK) return s;
    if ((s = make_tmap(&tk, k, "k")) != FA_OK) return s;
    if ((s = make_tmap(&tv, v, "v")) != FA_OK) return s;
    if ((s = make_tmap(&tdo, dout, "dout")) != FA_OK) return s;
    const int nsm = sm_count(dev);
    if (nsm <= 0) return fail(FA_ERR_CUDA, "could not read the SM count");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = q->dtype == FA_DTYPE_BF16;
    const int D = (int)q->D;
    const int q_pad = m->QB * fa::kBlock;
    float* neg_lse_log2 = static_cast<float*>(workspace);
    float* neg_delta = neg_lse_log2 + (size_t)q->B * q->H * q_pad;

    e = fa::launch_bwd_preprocess(out->data, out->stride, dout->data, dout->stride, lse, (int)q->B,
                                  (int)q->H, (int)q->S, q_pad, D, bf16, neg_lse_log2, neg_delta, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward pre-pass launch");

    const float sc = (scale > 0.f) ? scale : (float)(1.0 / std::sqrt((double)q->D));
    const float cap = (score_mod_kind & FA_SCORE_SOFTCAP) ? params->softcap : 1.f;
    fa::BwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = (int32_t)q->B;
    p.H = (int32_t)q->H;
    p.Q_LEN = m->Q_LEN;
    p.KV_LEN = m->KV_LEN;
    p.QB = m->QB;
    p.KVB = m->KVB;
    p.maskB = m->B;
    p.maskH = m->H;
    p.mask_kind = m->mask_kind;
    p.window = m->window;
    p.score_kind = score_mod_kind;
    p.doc_id = m->doc;
    p.kv_lens = m->kv_lens;
    p.scale = sc;
    p.scale_log2 = sc * 1.4426950408889634f;
    p.softcap_log2 = cap * 1.4426950408889634f;
    p.inv_softcap_scale = sc / cap;
    p.alibi_slopes = params ? params->alibi_slopes : nullptr;
    p.neg_lse_log2 = neg_lse_log2;
    p.neg_delta = neg_delta;
    p.q_pad = q_pad;
    p.status = m->status;
    p.stall_loads = g_stall_loads.load(std::memory_order_relaxed);
    fa_block_mask_t* mm = const_cast<fa_block_mask_t*>(m);

    // dK, dV: one unit per kv block; Q and dO stream, so order by head when they outgrow L2.
    fa::BwdParams pk = p;
    pk.units_per_bh = m->KVB;
    pk.entries_stride = m->QB;
    pk.n_units = (int32_t)((int64_t)m->KVB * q->B * q->H);
    pk.head_major = head_major_order(q->B * q->H, q->S, q->D) ? 1 : 0;
    pk.order = m->bwd.kv_order;
    pk.count = m->bwd.kv_count;
    pk.entries = m->bwd.kv_entries;
    pk.grad0 = dk->data;
    pk.grad1 = dv->data;
    for (int i = 0; i < 3; ++i) {
        pk.grad0_stride[i] = dk->stride[i];
        pk.grad1_stride[i] = dv->stride[i];
    }
    const int grid_k = pk.n_units < nsm ? pk.n_units : nsm;
    s = launch_with_counter_pair(mm, st, [&](int32_t* ctr) {
        pk.sched_ctr = ctr;
        return fa::launch_attn_bwd_dkdv(pk, D, bf16, (int)score_mod_kind, tq, tk, tv, tdo, grid_k, st);
    });
    if (s != FA_OK) return s;

    // dQ: one unit per query block; K and V stream in the mask's dQ write order.
    fa::BwdParams pq = p;
    pq.units_per_bh = m->QB;
    pq.entries_stride = m->KVB;
    pq.n_units = (int32_t)((int64_t)m->QB * q->B * q->H);
    pq.head_major = head_major_order(q->B * q->H, k->S, q->D) ? 1 : 0;
    pq.order = m->bwd.dq_order;
    pq.count = m->bwd.dq_count;
    pq.entries = m->bwd.dq_entries;
    pq.grad0 = dq->data;
    for (int i = 0; i < 3; ++i) pq.grad0_stride[i] = dq->stride[i];
    const int grid_q = pq.n_units < nsm ? pq.n_units : nsm;
    return launch_with_counter_pair(mm, st, [&](int32_t* ctr) {
        pq.sched_ctr = ctr;
        return fa::launch_attn_bwd_dq(pq, D, bf16, (int)score_mod_kind, tq, tk, tv, tdo, grid_q, st);
    });
}

fa_status_t fa_masked_softmax(const fa_tensor_t* scores, uint32_t mask_kind, int64_t offset,
                              fa_tensor_t* probs, void* stream) {
    NvtxRange nvtx_range("fa_masked_softmax");
    fa_status_t s;
    if ((s = check_tensor(scores, "scores")) != FA_OK) return s;
    if ((s = check_tensor(probs, "probs")) != FA_OK) return s;
    if (probs->dtype != scores->dtype) return fail(FA_ERR_INVALID_ARG, "scores and probs must share one dtype");
    if (probs->B != scores->B || probs->H != scores->H || probs->S != scores->S || probs->D != scores->D)
        return fail(FA_ERR_INVALID_ARG, "scores and probs must have the same shape");
    if (mask_kind != 0 && mask_kind != FA_MASK_CAUSAL)
        return fail(FA_ERR_UNSUPPORTED, "mask_kind 0x%x: the fused softmax takes FA_MASK_CAUSAL or 0", mask_kind);
    const int64_t K = scores->D;
    if ((K % 8) != 0) return fail(FA_ERR_UNSUPPORTED, "K=%lld: rows must be whole 16-byte vectors (K %% 8 == 0)", (long long)K);
    if (K > fa::masked_softmax_max_keys())
        return fail(FA_ERR_UNSUPPORTED, "K=%lld above the %d keys a row may hold", (long long)K, fa::masked_softmax_max_keys());
    if (scores->B > 0x7fffffff || scores->H > 0x7fffffff || scores->S > 0x7fffffff)
        return fail(FA_ERR_UNSUPPORTED, "extent above 2^31 - 1");
    if (probs->data != scores->data) {
        // Distinct buffers must not overlap (the same buffer with the same strides is fine:
        // every row is read before it is written).
    } else {
        for (int i = 0; i < 3; ++i)
            if (probs->stride[i] != scores->stride[i])
                return fail(FA_ERR_INVALID_ARG, "in-place softmax needs probs and scores to share strides");
    }
    if (scores->B == 0 || scores->H == 0 || scores->S == 0) return ok();
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if ((s = fa::check_device_memory(scores->data, dev, "scores")) != FA_OK) return s;
    if ((s = fa::check_device_memory(probs->data, dev, "probs")) != FA_OK) return s;
    const int nsm = sm_count(dev);
    if (nsm <= 0) return fail(FA_ERR_CUDA, "could not read the SM count");
    e = fa::launch_masked_softmax_checked(scores->data, probs->data, scores->stride, probs->stride,
                                          (int)scores->B, (int)scores->H, (int)scores->S, (int)K,
                                          offset, mask_kind == FA_MASK_CAUSAL,
                                          scores->dtype == FA_DTYPE_BF16, nsm,
                                          g_stall_loads.load(std::memory_order_relaxed),
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "masked-softmax launch");
    return ok();
}

fa_status_t fa_masked_softmax_status(void* stream) {
    int32_t h = 0;
    cudaError_t e = fa::masked_softmax_status(static_cast<cudaStream_t>(stream), &h);
    if (e != cudaSuccess) return cuda_fail(e, "reading the masked-softmax status word");
    if (h != 0) return fail(FA_ERR_TIMEOUT, "a masked-softmax wait ran past its limit (status %d)", h);
    return ok();
}


fa_status_t fa_forward(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                       const fa_block_mask_t* m, uint32_t score_mod_kind,
                       const fa_score_params_t* params, float scale, fa_tensor_t* out, float* lse,
                       void* stream) {
    NvtxRange nvtx_range("fa_forward");
    return forward_impl(q, k, v, nullptr, 0, m, score_mod_kind, params, scale, out, lse, stream);
}

size_t fa_forward_paged_workspace_bytes(const fa_block_mask_t* m, int64_t B, int64_t H,
                                        int64_t Q_LEN, int64_t D) {
    if (!m || B <= 0 || H <= 0 || Q_LEN <= 0 || Q_LEN > fa::kDecodeMaxQ || (D != 64 && D != 128) ||
        B * H > 65535)
        return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    int tpc = 0, chunks = 0;
    decode_chunking(m->KVB, B * H, sm_count(dev), tpc, chunks);
    return (size_t)(B * H * Q_LEN) * chunks * (size_t)(D + 2) * 4;
}

fa_status_t fa_forward_paged(const fa_tensor_t* q, const fa_tensor_t* k_pages,
                             const fa_tensor_t* v_pages, const int32_t* page_table,
                             int64_t page_table_stride, const fa_block_mask_t* m,
                             uint32_t score_mod_kind, const fa_score_params_t* params, float scale,
                             fa_tensor_t* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream) {
    NvtxRange nvtx_range("fa_forward_paged");
    if (!page_table) return fail(FA_ERR_INVALID_ARG, "page_table is NULL");
    if ((reinterpret_cast<uintptr_t>(page_table) & 3u) != 0)
        return fail(FA_ERR_INVALID_ARG, "page_table is not 4-byte aligned");
    const bool split = workspace && q && q->S >= 1 && q->S <= fa::kDecodeMaxQ && q->B * q->H <= 65535;
    if (!split)
        return forward_impl(q, k_pages, v_pages, page_table, page_table_stride, m, score_mod_kind, params,
                            scale, out, lse, stream);
    // The split decode path: every argument check of the forward first (nothing is launched
    // on an error), then the workspace.
    fa_status_t s = forward_impl(q, k_pages, v_pages, page_table, page_table_stride, m, score_mod_kind,
                                 params, scale, out, lse, stream, /*check_only=*/true);
    if (s != FA_OK) return s;
    if (q->B == 0 || q->H == 0) return ok();
    const size_t need = fa_forward_paged_workspace_bytes(m, q->B, q->H, q->S, q->D);
    if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15u))
        return fail(FA_ERR_INVALID_ARG, "workspace must be 16-byte aligned device memory of at least %zu bytes", need);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if ((s = fa::check_device_memory(workspace, dev, "workspace")) != FA_OK) return s;
    fa::DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = (int32_t)q->B;
    p.H = (int32_t)q->H;
    p.Q_LEN = (int32_t)q->S;
    p.KV_LEN = m->KV_LEN;
    p.KVB = m->KVB;
    p.NP = m->NP;
    p.maskB = m->B;
    p.maskH = m->H;
    p.mask_kind = m->mask_kind;
    p.window = m->window;
    p.doc_id = m->doc;
    p.kv_lens = m->kv_lens;
    p.sched_count = m->sched_count;
    p.sched_entries = m->sched_entries;
    p.q = q->data;
    p.k = k_pages->data;
    p.v = v_pages->data;
    for (int i = 0; i < 3; ++i) {
        p.q_stride[i] = q->stride[i];
        p.k_stride[i] = k_pages->stride[i];
        p.v_stride[i] = v_pages->stride[i];
        p.out_stride[i] = out->stride[i];
    }
    p.page_table = page_table;
    p.page_stride = (int32_t)page_table_stride;
    p.n_pages = (int32_t)k_pages->B;
    const float sc = (scale > 0.f) ? scale : (float)(1.0 / std::sqrt((double)q->D));
    const float cap = (score_mod_kind & FA_SCORE_SOFTCAP) ? params->softcap : 1.f;
    p.scale_log2 = sc * 1.4426950408889634f;
    p.softcap_log2 = cap * 1.4426950408889634f;
    p.inv_softcap_scale = sc / cap;
    p.alibi_slopes = params ? params->alibi_slopes : nullptr;
    p.out = out->data;
    p.lse = lse;
    p.partials = static_cast<float*>(workspace);
    decode_chunking(m->KVB, q->B * q->H, sm_count(dev), p.tiles_per_chunk, p.max_chunks);
    p.status = m->status;
    e = fa::launch_decode(p, (int)q->D, q->dtype == FA_DTYPE_BF16, (int)score_mod_kind,
                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return ok();
}

// Test hook for failure detection (see the header): read by every later fa_forward.
fa_status_t fa_debug_set_stall(int32_t enable) {
    g_stall_loads.store(enable ? 1 : 0, std::memory_order_relaxed);
    return ok();
}

}  // extern "C"
