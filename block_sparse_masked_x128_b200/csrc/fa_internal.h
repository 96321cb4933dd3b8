// fa_internal.h -- structures shared by the host API (api.cu) and the kernels.
#pragma once

#include <atomic>
#include <mutex>

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_b200.h"

namespace fa {

constexpr int kBlock = 128;          // BLOCK_SIZE: query rows and keys per tile
constexpr int kMaxBlocks = 16384;    // q_blocks and kv_blocks limit (2M positions)

// Debug builds (FA_DEBUG, build.py --debug): kernels check each index they read from the
// mask's metadata before using it; an index out of range is recorded in the mask's status
// word (kStatusBadIndex) and replaced by 0, so the kernel finishes instead of faulting.  The
// product build compiles the checks away.
constexpr int kStatusBadIndex = 3;
#ifdef FA_DEBUG
#define FA_DCHECK_INDEX(idx, limit, status)                              \
    do {                                                                 \
        if ((unsigned)(idx) >= (unsigned)(limit)) {                      \
            atomicExch((status), kStatusBadIndex);                       \
            (idx) = 0;                                                   \
        }                                                                \
    } while (0)
#else
#define FA_DCHECK_INDEX(idx, limit, status) \
    do {                                    \
    } while (0)
#endif

// Tile classes written by the mask builder.
constexpr int kDead = 0, kPartial = 1, kFull = 2, kAmbiguous = 3;

// Schedule entry: bits 0-15 kv block, then per-tile live / full flags for the two
// query tiles of a work unit (query blocks 2p and 2p+1).
constexpr int kLive0 = 1 << 16, kFull0 = 1 << 17, kLive1 = 1 << 18, kFull1 = 1 << 19;

// Inputs of the mask-builder kernels.  Tiles are BQ query rows by BKV keys (128 x 128 for the
// lists the attention kernels walk; a caller's BLOCK_SIZE for the lists it reads back).
struct MaskSpec {
    uint32_t kind;
    int32_t window;
    int32_t Q_LEN, KV_LEN, QB, KVB;
    int32_t BQ, BKV;
    const int32_t* doc;           // [KV_LEN] or null
    const int32_t* doc_stats;     // [QB][3] = {min, max, uniform} per query block, or null
    const int32_t* doc_stats_kv;  // [KVB][3] per kv block (== doc_stats when BQ == BKV)
    const int32_t* kv_lens;       // [B] per-batch context lengths, or null
    int32_t maskH;                // stored H (row bh of the lists is batch bh / maskH)
};

// Kernel parameters of the fused forward (passed by value, __grid_constant__).
struct FwdParams {
    int32_t B, H, Q_LEN, KV_LEN;
    int32_t QB, KVB, NP;          // query blocks, kv blocks, work-unit pairs per (b, h)
    int32_t maskB, maskH;         // stored mask extents (1 = broadcast)
    int32_t n_units;              // NP * B * H
    int32_t head_major;           // 1: the units of one (b, h) are handed out together
    uint32_t mask_kind;
    int32_t window;
    uint32_t score_kind;
    const int32_t* doc_id;
    const int32_t* kv_lens;       // [B] per-batch context lengths, or null (all KV_LEN)
    const int32_t* page_table;    // [B][page_stride] physical page of each kv block, or null
    int32_t page_stride;
    int32_t n_pages;              // pages in the K/V pools (the pools' batch extent)
    const int32_t* sched_order;   // [maskB*maskH][NP]  pairs by descending cost
    const int32_t* sched_gorder;  // [maskB*maskH*NP] all units by descending cost, or null
    const int32_t* sched_count;   // [maskB*maskH][NP][2]  entries; live tiles t0 | t1 << 16
    const int32_t* sched_entries; // [maskB*maskH][NP][KVB]
    float scale;                  // multiplies q k^T
    float scale_log2;             // scale * log2(e)
    float softcap;
    float softcap_log2;           // softcap * log2(e)
    float inv_softcap_scale;      // scale / softcap
    const float* alibi_slopes;    // device [H] or null (then 2^(-8(h+1)/H))
    void* out;
    int64_t out_stride[3];        // B, H, S strides in elements (D stride is 1)
    float* lse;                   // [B][H][Q_LEN] or null
    int32_t* status;              // device status word (1 = a bounded wait ran out)
    int32_t* sched_ctr;           // [0] next unit to hand out, [1] CTAs done; both 0 between launches
    int32_t stall_loads;          // test hook: the TMA warp stops after the first Q tiles
};

// Backward metadata of a mask (all int32, maskBH = stored B * H):
//   q_num, fq_num [maskBH][KVB]; q_idx, fq_idx [maskBH][KVB][QB]: per kv block, the query
//     blocks whose tile is partial / full, ascending, zero padded (the transposed lists);
//   kv_count, kv_cost, kv_order [maskBH][KVB]; kv_entries [maskBH][KVB][QB]: the dK/dV
//     kernel's units, one per kv block: entries query block | kLive0 (| kFull0) ascending,
//     units ranked by cost (longest first);
//   dq_count, dq_cost, dq_order [maskBH][QB]; dq_entries [maskBH][QB][KVB]: the dQ kernel's
//     units, one per query block: kv block | kLive0 (| kFull0) in the mask's dQ write order.
struct BwdMeta {
    int32_t *q_num, *q_idx, *fq_num, *fq_idx;
    int32_t *kv_count, *kv_cost, *kv_entries, *kv_order;
    int32_t *dq_count, *dq_cost, *dq_entries, *dq_order;
};

cudaError_t launch_backward_metadata(int QB, int KVB, int maskBH, int dq_descending,
                                     const int32_t* kv_num, const int32_t* kv_idx,
                                     const int32_t* full_num, const int32_t* full_idx,
                                     const BwdMeta& m, cudaStream_t stream);

// Kernel parameters of the backward kernels (attn_bwd.cu).  A unit is one kv block (dK/dV
// kernel) or one query block (dQ kernel) of one (b, h); its entries are the tiles it visits.
struct BwdParams {
    int32_t B, H, Q_LEN, KV_LEN, QB, KVB;
    int32_t maskB, maskH;
    int32_t units_per_bh;         // KVB (dK/dV kernel) or QB (dQ kernel)
    int32_t entries_stride;       // QB (dK/dV kernel) or KVB (dQ kernel)
    int32_t n_units;              // units_per_bh * B * H
    int32_t head_major;           // 1: units of one (b, h) are handed out together
    uint32_t mask_kind;
    int32_t window;
    uint32_t score_kind;
    const int32_t* doc_id;
    const int32_t* kv_lens;       // [B] per-batch context lengths, or null (all KV_LEN)
    const int32_t* order;         // [maskB*maskH][units_per_bh]  units by descending cost
    const int32_t* count;         // [maskB*maskH][units_per_bh]  entries per unit
    const int32_t* entries;       // [maskB*maskH][units_per_bh][entries_stride]
    float scale;
    float scale_log2;             // scale * log2(e)
    float softcap_log2;           // softcap * log2(e)
    float inv_softcap_scale;      // scale / softcap
    const float* alibi_slopes;    // device [H] or null (then 2^(-8(h+1)/H))
    const float* neg_lse_log2;    // workspace [B*H][q_pad]: -lse * log2(e), -inf without keys
    const float* neg_delta;       // workspace [B*H][q_pad]: -rowsum(dO * O)
    int32_t q_pad;                // QB * 128
    void* grad0;                  // dK/dV kernel: dK; dQ kernel: dQ
    void* grad1;                  // dK/dV kernel: dV; dQ kernel: unused
    int64_t grad0_stride[3];      // B, H, S strides in elements
    int64_t grad1_stride[3];
    int32_t* status;
    int32_t* sched_ctr;
    int32_t stall_loads;          // test hook: the TMA warp stops after the first unit's fixed tiles
};

// Parameters of the split decode path (decode.cu): Q_LEN <= 4 query rows over paged K/V.
struct DecodeParams {
    int32_t B, H, Q_LEN, KV_LEN, KVB, NP, maskB, maskH;
    uint32_t mask_kind;
    int32_t window;
    const int32_t* doc_id;
    const int32_t* kv_lens;
    const int32_t* sched_count;   // the block mask's forward schedule (query block 0 of each pair)
    const int32_t* sched_entries;
    const void* q;
    const void* k;                // page pools (n_pages, H, 128, D)
    const void* v;
    int64_t q_stride[3], k_stride[3], v_stride[3];
    const int32_t* page_table;
    int32_t page_stride, n_pages;
    float scale_log2, softcap_log2, inv_softcap_scale;
    const float* alibi_slopes;
    void* out;
    int64_t out_stride[3];
    float* lse;
    float* partials;              // workspace [B*H][Q_LEN][max_chunks][D + 2]: m, l, O
    int32_t max_chunks, tiles_per_chunk;
    int32_t* status;
};
constexpr int kDecodeMaxQ = 4;
cudaError_t launch_decode(const DecodeParams& p, int D, bool bf16, int score_kind, cudaStream_t st);

cudaError_t launch_bwd_preprocess(const void* out, const int64_t out_stride[3], const void* dout,
                                  const int64_t dout_stride[3], const float* lse, int B, int H,
                                  int Q_LEN, int q_pad, int D, bool bf16, float* neg_lse_log2,
                                  float* neg_delta, cudaStream_t stream);
cudaError_t launch_attn_bwd_dkdv(const BwdParams& p, int D, bool bf16, int score_kind,
                                 const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const CUtensorMap& tdo, int grid, cudaStream_t stream);
cudaError_t launch_attn_bwd_dq(const BwdParams& p, int D, bool bf16, int score_kind,
                               const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tdo, int grid, cudaStream_t stream);

cudaError_t launch_expand_block_lists(int UQB, int UKVB, int rq, int rkv, int QB, int KVB, int Q_LEN,
                                      int KV_LEN, const int32_t* kv_lens, int maskH, int maskBH,
                                      int separate_full,
                                      const int32_t* u_kv_num, const int32_t* u_kv_idx,
                                      const int32_t* u_full_num, const int32_t* u_full_idx,
                                      int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                                      int32_t* full_idx, int32_t* bad, cudaStream_t stream);
cudaError_t launch_transpose_lists(int QB, int KVB, int maskBH, const int32_t* kv_num,
                                   const int32_t* kv_idx, const int32_t* full_num,
                                   const int32_t* full_idx, int32_t* q_num, int32_t* q_idx,
                                   int32_t* fq_num, int32_t* fq_idx, cudaStream_t stream);
cudaError_t launch_schedule(int QB, int KVB, int maskBH, int NP, const int32_t* kv_num,
                            const int32_t* kv_idx, const int32_t* full_num, const int32_t* full_idx,
                            int32_t* sched_count, int32_t* sched_cost, int32_t* sched_entries,
                            int32_t* sched_order, cudaStream_t stream);

// The forward's units of all stored (b, h) ranked together (longest first), for masks with at
// most this many units; larger masks rank within each (b, h) only.
constexpr int kGlobalOrderMax = 16384;
cudaError_t launch_global_order(int n, const int32_t* cost, int32_t* order, cudaStream_t stream);

cudaError_t launch_mask_build(const MaskSpec& spec, int separate_full, int maskBH, int NP,
                              int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                              int32_t* full_idx, int32_t* doc_stats, int32_t* sched_count,
                              int32_t* sched_cost, int32_t* sched_entries, int32_t* sched_order,
                              cudaStream_t stream);

// Only the tile classification and list compaction of launch_mask_build (no schedule),
// with the per-block document statistics at `doc_stats`.
cudaError_t launch_mask_lists(const MaskSpec& spec, int separate_full, int maskBH,
                              int32_t* kv_num, int32_t* kv_idx, int32_t* full_num,
                              int32_t* full_idx, int32_t* doc_stats, cudaStream_t stream);

// Set the calling thread's last-error message (read by fa_last_error_message).
fa_status_t record_error(fa_status_t status, const char* message);
fa_status_t record_ok();

cudaError_t launch_attn_fwd(const FwdParams& p, int D, bool bf16, int score_kind,
                            const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            int grid, cudaStream_t stream);

// Causal-masked softmax over materialised scores (masked_softmax.cu).
struct SoftmaxParams;
int masked_softmax_max_keys();
cudaError_t launch_masked_softmax_checked(const void* in, void* out, const int64_t in_stride[3],
                                          const int64_t out_stride[3], int B, int H, int Q, int K,
                                          int64_t offset, bool causal, bool bf16, int num_sms,
                                          int stall_loads, cudaStream_t stream);
cudaError_t masked_softmax_status(cudaStream_t stream, int32_t* out);

// Counter pairs per mask for the forward's run-time unit hand-out: each launch takes the
// next pair, so up to this many forwards may run at once on one mask.
constexpr int kSchedCtrSlots = 64;

}  // namespace fa

struct fa_block_mask {
    uint32_t mask_kind;
    int32_t window;
    int32_t separate_full;
    int32_t B, H;            // stored extents (1 when broadcast)
    int32_t Q_LEN, KV_LEN, QB, KVB, NP;
    int device;
    void* dev_base;
    int32_t* kv_num;
    int32_t* kv_idx;
    int32_t* full_num;
    int32_t* full_idx;
    int32_t* doc;
    int32_t* doc_stats;
    int32_t* kv_lens;         // copy of the per-batch context lengths, or null
    int32_t* sched_count;
    int32_t* sched_cost;
    int32_t* sched_entries;
    int32_t* sched_order;
    int32_t* sched_gorder;    // units of all stored (b, h) by cost, or null when too many
    int32_t* status;
    // The lists a caller reads back (fa_block_mask_get), at its block size BQ x BKV: the
    // kernel's own 128 x 128 lists when that is the block size, separate arrays otherwise.
    int32_t BQ, BKV, UQB, UKVB;
    int32_t *u_kv_num, *u_kv_idx, *u_full_num, *u_full_idx;
    int32_t *u_q_num, *u_q_idx, *u_fq_num, *u_fq_idx;
    int32_t* u_doc_stats;
    int32_t dq_kv_order;      // 1: dQ accumulates kv blocks in descending order, 0: ascending
    fa::BwdMeta bwd;
    int32_t* sched_ctr;       // fa::kSchedCtrSlots pairs of unit counters after the status word
    // Round-robin pick of a counter pair per forward.  ctr_event[s] is recorded after the
    // last forward that used pair s; the next forward on pair s waits for it on the GPU, so
    // no more than kSchedCtrSlots forwards ever share the pairs at once.
    std::mutex ctr_mutex;
    uint32_t next_ctr = 0;
    cudaEvent_t ctr_event[fa::kSchedCtrSlots] = {};
};
