// api.cu -- the C ABI declared in include/fa_b200.h: argument checks, device memory of
// block masks, TMA descriptors, and kernel launches.  No compute happens on the host.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>

#include "fa_internal.h"

namespace {

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
    if (!t->data) return fail(FA_ERR_INVALID_ARG, "%s.data is NULL", name);
    if (t->dtype != FA_DTYPE_F16 && t->dtype != FA_DTYPE_BF16)
        return fail(FA_ERR_INVALID_ARG, "%s.dtype %d is not FA_DTYPE_F16/BF16", name, t->dtype);
    if (t->B < 0 || t->H < 0 || t->S < 0 || t->D <= 0)
        return fail(FA_ERR_INVALID_ARG, "%s has a negative or zero extent", name);
    if (t->stride[3] != 1) return fail(FA_ERR_INVALID_ARG, "%s.stride[3] must be 1", name);
    for (int i = 0; i < 3; ++i)
        if (t->stride[i] <= 0 || (t->stride[i] % 8) != 0)
            return fail(FA_ERR_INVALID_ARG, "%s.stride[%d]=%lld must be a positive multiple of 8",
                        name, i, (long long)t->stride[i]);
    if ((reinterpret_cast<uintptr_t>(t->data) & 15u) != 0)
        return fail(FA_ERR_INVALID_ARG, "%s.data is not 16-byte aligned", name);
    return FA_OK;
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
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
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

fa_status_t fa_create_block_mask(uint32_t mask_kind, const fa_mask_params_t* params, int32_t B,
                                 int32_t H, int32_t Q_LEN, int32_t KV_LEN, int32_t BLOCK_SIZE,
                                 void* stream, fa_block_mask_t** out_mask) {
    if (!out_mask) return fail(FA_ERR_INVALID_ARG, "out_mask is NULL");
    *out_mask = nullptr;
    const uint32_t known = FA_MASK_CAUSAL | FA_MASK_SLIDING_WINDOW | FA_MASK_DOCUMENT;
    if (mask_kind & ~known) return fail(FA_ERR_INVALID_ARG, "unknown mask_kind bits 0x%x", mask_kind);
    if (B < 0 || H < 0) return fail(FA_ERR_INVALID_ARG, "B and H must be >= 0 (0 = broadcast)");
    if (Q_LEN <= 0 || KV_LEN <= 0) return fail(FA_ERR_INVALID_ARG, "Q_LEN and KV_LEN must be > 0");
    if (BLOCK_SIZE != fa::kBlock)
        return fail(FA_ERR_UNSUPPORTED, "BLOCK_SIZE %d: only 128 is implemented", BLOCK_SIZE);
    const int32_t window = params ? params->window : 0;
    const int32_t sep = params ? (params->separate_full_blocks ? 1 : 0) : 1;
    if ((mask_kind & FA_MASK_SLIDING_WINDOW) && window <= 0)
        return fail(FA_ERR_INVALID_ARG, "sliding window needs params->window > 0");
    if (mask_kind & FA_MASK_DOCUMENT) {
        if (!params || !params->doc_id) return fail(FA_ERR_INVALID_ARG, "document mask needs params->doc_id");
        if (Q_LEN != KV_LEN) return fail(FA_ERR_INVALID_ARG, "document mask needs Q_LEN == KV_LEN");
    }
    const int QB = (Q_LEN + fa::kBlock - 1) / fa::kBlock;
    const int KVB = (KV_LEN + fa::kBlock - 1) / fa::kBlock;
    if (QB > fa::kMaxBlocks || KVB > fa::kMaxBlocks)
        return fail(FA_ERR_UNSUPPORTED, "more than %d blocks per side", fa::kMaxBlocks);
    const int Bm = B ? B : 1, Hm = H ? H : 1;
    const int NP = (QB + 1) / 2;
    const size_t BH = (size_t)Bm * Hm;
    if (BH > 65535) return fail(FA_ERR_UNSUPPORTED, "B*H of a non-broadcast mask above 65535");

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");

    // One allocation holds every device array of the mask.
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    const size_t o_kvn = take(BH * QB * 4), o_kvi = take(BH * QB * KVB * 4);
    const size_t o_fn = take(BH * QB * 4), o_fi = take(BH * QB * KVB * 4);
    const bool has_doc = (mask_kind & FA_MASK_DOCUMENT) != 0;
    // The copy of doc_id is padded to whole blocks (the forward reads ids by 128-key tile).
    const size_t doc_pad = (size_t)KVB * fa::kBlock;
    const size_t o_doc = take(has_doc ? doc_pad * 4 : 0);
    const size_t o_dst = take(has_doc ? (size_t)(QB > KVB ? QB : KVB) * 3 * 4 : 0);
    const size_t o_sc = take(BH * NP * 8), o_scost = take(BH * NP * 4);
    const size_t o_se = take(BH * NP * KVB * 4), o_so = take(BH * NP * 4);
    // Backward metadata: transposed lists, the dK/dV kernel's kv-major units, the dQ units.
    const size_t n_kv = BH * KVB, n_q = BH * QB, n_tiles = BH * QB * KVB;
    const size_t o_qn = take(n_kv * 4), o_qi = take(n_tiles * 4), o_fqn = take(n_kv * 4),
                 o_fqi = take(n_tiles * 4);
    const size_t o_kvc = take(n_kv * 4), o_kvcost = take(n_kv * 4), o_kve = take(n_tiles * 4),
                 o_kvo = take(n_kv * 4);
    const size_t o_dqc = take(n_q * 4), o_dqcost = take(n_q * 4), o_dqe = take(n_tiles * 4),
                 o_dqo = take(n_q * 4);
    // Status word, then the forward's unit counters (two words per slot), all zero.
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
    m->kv_num = reinterpret_cast<int32_t*>(b8 + o_kvn);
    m->kv_idx = reinterpret_cast<int32_t*>(b8 + o_kvi);
    m->full_num = reinterpret_cast<int32_t*>(b8 + o_fn);
    m->full_idx = reinterpret_cast<int32_t*>(b8 + o_fi);
    m->doc = has_doc ? reinterpret_cast<int32_t*>(b8 + o_doc) : nullptr;
    m->doc_stats = has_doc ? reinterpret_cast<int32_t*>(b8 + o_dst) : nullptr;
    m->sched_count = reinterpret_cast<int32_t*>(b8 + o_sc);
    m->sched_cost = reinterpret_cast<int32_t*>(b8 + o_scost);
    m->sched_entries = reinterpret_cast<int32_t*>(b8 + o_se);
    m->sched_order = reinterpret_cast<int32_t*>(b8 + o_so);
    auto at = [&](size_t o) { return reinterpret_cast<int32_t*>(b8 + o); };
    m->dq_kv_order = params ? (params->dq_kv_order ? 1 : 0) : 1;
    m->bwd = fa::BwdMeta{at(o_qn),  at(o_qi),     at(o_fqn), at(o_fqi), at(o_kvc),    at(o_kvcost),
                         at(o_kve), at(o_kvo),    at(o_dqc), at(o_dqcost), at(o_dqe), at(o_dqo)};
    m->status = reinterpret_cast<int32_t*>(b8 + o_status);
    m->sched_ctr = m->status + 1;

    auto bail = [&](cudaError_t err, const char* what) {
        cudaStreamSynchronize(st);
        cudaFree(base);
        delete m;
        return cuda_fail(err, what);
    };
    if ((e = cudaMemsetAsync(m->status, 0, ctr_bytes, st)) != cudaSuccess) return bail(e, "cudaMemsetAsync");
    if (has_doc &&
        (e = cudaMemcpyAsync(m->doc, params->doc_id, (size_t)KV_LEN * 4, cudaMemcpyDefault, st)) !=
            cudaSuccess)
        return bail(e, "copy of doc_id");
    if (has_doc && doc_pad > (size_t)KV_LEN &&
        (e = cudaMemsetAsync(m->doc + KV_LEN, 0, (doc_pad - KV_LEN) * 4, st)) != cudaSuccess)
        return bail(e, "padding of doc_id");
    fa::MaskSpec spec;
    spec.kind = mask_kind;
    spec.window = window;
    spec.Q_LEN = Q_LEN;
    spec.KV_LEN = KV_LEN;
    spec.QB = QB;
    spec.KVB = KVB;
    spec.doc = m->doc;
    spec.doc_stats = m->doc_stats;
    e = fa::launch_mask_build(spec, sep, (int)BH, NP, m->kv_num, m->kv_idx, m->full_num,
                              m->full_idx, m->doc_stats, m->sched_count, m->sched_cost,
                              m->sched_entries, m->sched_order, st);
    if (e != cudaSuccess) return bail(e, "mask-builder launch");
    e = fa::launch_backward_metadata(QB, KVB, (int)BH, m->dq_kv_order, m->kv_num, m->kv_idx,
                                     m->full_num, m->full_idx, m->bwd, st);
    if (e != cudaSuccess) return bail(e, "backward-metadata launch");
    *out_mask = m;
    return ok();
}

fa_status_t fa_block_mask_get(const fa_block_mask_t* m, fa_block_mask_info_t* info) {
    if (!m || !info) return fail(FA_ERR_INVALID_ARG, "NULL argument");
    info->B = m->B;
    info->H = m->H;
    info->Q_LEN = m->Q_LEN;
    info->KV_LEN = m->KV_LEN;
    info->BLOCK_SIZE = fa::kBlock;
    info->q_blocks = m->QB;
    info->kv_blocks = m->KVB;
    info->mask_kind = m->mask_kind;
    info->window = m->window;
    info->separate_full_blocks = m->separate_full;
    info->kv_num_blocks = m->kv_num;
    info->kv_indices = m->kv_idx;
    info->full_kv_num_blocks = m->full_num;
    info->full_kv_indices = m->full_idx;
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
        return fail(FA_ERR_TIMEOUT, "a device-side wait ran past its limit (status %d)", h);
    }
    return ok();
}

fa_status_t fa_forward(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                       const fa_block_mask_t* m, uint32_t score_mod_kind,
                       const fa_score_params_t* params, float scale, fa_tensor_t* out, float* lse,
                       void* stream) {
    fa_status_t s;
    if ((s = check_tensor(q, "q")) != FA_OK) return s;
    if ((s = check_tensor(k, "k")) != FA_OK) return s;
    if ((s = check_tensor(v, "v")) != FA_OK) return s;
    if ((s = check_tensor(out, "out")) != FA_OK) return s;
    if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype)
        return fail(FA_ERR_INVALID_ARG, "q, k, v and out must share one dtype");
    if (k->B != q->B || v->B != q->B || out->B != q->B || k->H != q->H || v->H != q->H ||
        out->H != q->H)
        return fail(FA_ERR_INVALID_ARG, "q, k, v and out must share B and H");
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
    if (q->S != m->Q_LEN || k->S != m->KV_LEN)
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
    p.mask_kind = m->mask_kind;
    p.window = m->window;
    p.score_kind = score_mod_kind;
    p.doc_id = m->doc;
    p.sched_order = m->sched_order;
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

fa_status_t fa_masked_softmax(const fa_tensor_t* scores, uint32_t mask_kind, int64_t offset,
                              fa_tensor_t* probs, void* stream) {
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

// Test hook for failure detection (see the header): read by every later fa_forward.
fa_status_t fa_debug_set_stall(int32_t enable) {
    g_stall_loads.store(enable ? 1 : 0, std::memory_order_relaxed);
    return ok();
}

}  // extern "C"
