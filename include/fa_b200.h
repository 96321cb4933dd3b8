/*
 * fa_b200.h -- C ABI of the B200 (sm_100a) block-sparse masked attention library.
 *
 * Two operations make up the path:
 *
 *   fa_create_block_mask   evaluates a fixed mask_mod over the 128 x 128 tile grid
 *                          and emits, per query block, the ascending lists of
 *                          partially masked and fully unmasked key/value blocks
 *                          ("tensorplay.nn.attention.create_block_mask", Parameters:
 *                          BLOCK_SIZE, separate_full_blocks; "How to Use FlexAttention
 *                          on Apple Silicon", sections "The two hooks" and "Mask 1").
 *   fa_forward             one fused attention forward over the live tiles only:
 *                          mask_mod on partial tiles, score_mod on live scores, online
 *                          softmax, O and the log-sum-exp written out; the N x N score
 *                          matrix never exists ("How to Use FlexAttention on Apple
 *                          Silicon", "The two hooks" and "Bonus: a score_mod for
 *                          soft-capping").
 *
 * Conventions shared by every call:
 *   - All tensor data pointers are DEVICE pointers owned by the caller unless stated.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls are asynchronous on that stream; they never synchronise it except
 *     fa_get_device_status.
 *   - Every call returns a status and never throws or aborts across the ABI.  All
 *     argument checks happen before any launch; on an error nothing is launched and
 *     no output is written.  fa_last_error_message() gives a one-line reason.
 *   - Library objects are not thread-safe against concurrent destroy; concurrent
 *     fa_forward calls on one mask, from any threads and streams, are allowed (the lists
 *     are read-only for them).  Each launch takes the next of the mask's 64 pairs of
 *     work-distribution counters, which its kernel leaves zero; before a pair is reused the
 *     new launch's stream waits on the GPU for the previous user of that pair, so a 65th
 *     forward in flight is delayed, never corrupted.  Under stream capture that wait is not
 *     recorded: a captured forward keeps its pair for every replay, and replays must not
 *     overlap other forwards on the same mask.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, bad flag bits, mismatched tensors */
    FA_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
    FA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or a launch failed */
    FA_ERR_OOM = 4,           /* device allocation failed */
    FA_ERR_TIMEOUT = 5,       /* a device-side wait ran past its limit (see fa_get_device_status) */
    FA_ERR_INTERNAL = 6
} fa_status_t;

/* mask_mod kinds: bit flags, OR-ed together meaning the conjunction (AND) of the
 * predicates ("How to Use FlexAttention on Apple Silicon", Masks 2 and 3 combine
 * predicates with &).  0 means every pair is allowed. */
#define FA_MASK_CAUSAL          1u   /* q_idx >= kv_idx                        ("Mask 1: causal")          */
#define FA_MASK_SLIDING_WINDOW  2u   /* 0 <= q_idx - kv_idx < window           ("Sliding-Window Self-Attention",
                                        "State the boundary precisely"; includes causality)               */
#define FA_MASK_DOCUMENT        4u   /* doc_id[q_idx] == doc_id[kv_idx]        ("Mask 3: document-packed") */

/* score_mod kinds: bit flags.  With both, the soft-cap is applied first and the
 * ALiBi bias is added to the capped score. */
#define FA_SCORE_NONE     0u
#define FA_SCORE_SOFTCAP  1u   /* softcap * tanh(score / softcap)  ("Bonus: a score_mod for soft-capping") */
#define FA_SCORE_ALIBI    2u   /* score + slope_h * (kv_idx - q_idx)  (additive distance bias, "The two hooks") */

#define FA_DTYPE_F16   0
#define FA_DTYPE_BF16  1

typedef struct fa_mask_params {
    int32_t        window;                /* W > 0, used when FA_MASK_SLIDING_WINDOW is set        */
    const int32_t* doc_id;                /* device, KV_LEN int32 ids (FA_MASK_DOCUMENT); requires
                                             Q_LEN == KV_LEN.  Copied: the caller may free it after
                                             fa_create_block_mask returns and the stream has run.  */
    int32_t        separate_full_blocks;  /* 1: fully unmasked tiles go to the full_* lists so the
                                             kernel skips mask_mod there; 0: every live tile is
                                             listed as partial ("create_block_mask", Parameters)   */
    int32_t        dq_kv_order;           /* order in which the backward accumulates each query
                                             block's dQ over its kv blocks: 1 descending, 0
                                             ascending ("create_block_mask", Parameters,
                                             dq_kv_order; either order is deterministic)          */
    int32_t        kv_block_size;         /* kv block size of the lists a caller reads back; 0 =
                                             BLOCK_SIZE ("create_block_mask", Parameters:
                                             BLOCK_SIZE int or (q, kv) tuple)                     */
    const int32_t* kv_lens;               /* device, B int32 context lengths, or NULL: key kv of
                                             batch b exists iff kv < kv_lens[b] (a batch of
                                             sequences of different lengths, e.g. paged decode);
                                             needs B > 0.  Copied like doc_id.                   */
} fa_mask_params_t;

typedef struct fa_score_params {
    float        softcap;        /* > 0 when FA_SCORE_SOFTCAP is set (30 in the soft-capping example) */
    const float* alibi_slopes;   /* device, H contiguous fp32 slopes (slope h at index h), or NULL for
                                    the slopes 2^(-8(h+1)/H)                                           */
} fa_score_params_t;

/* A (B, H, S, D) tensor: batch, heads, sequence, head_dim, the layout shared with
 * scaled_dot_product_attention ("How to Use FlexAttention on Apple Silicon", Setup). */
typedef struct fa_tensor {
    void*   data;        /* device pointer, 16-byte aligned; may be NULL when B, H or S is 0
                            (an empty tensor: every call on empty operands does nothing
                            and returns FA_OK)                                       */
    int32_t dtype;       /* FA_DTYPE_F16 or FA_DTYPE_BF16                           */
    int64_t B, H, S, D;
    int64_t stride[4];   /* element strides of B, H, S, D; stride[3] must be 1 and the
                            others positive multiples of 8 (16 bytes)               */
} fa_tensor_t;

typedef struct fa_block_mask fa_block_mask_t;   /* opaque, owned by the library */

/* Read-only view of a block mask (all pointers are device pointers owned by the mask). */
typedef struct fa_block_mask_info {
    int32_t  B, H;              /* stored extents: 1 where the mask was created broadcast */
    int32_t  Q_LEN, KV_LEN, BLOCK_SIZE;
    int32_t  q_blocks, kv_blocks;
    uint32_t mask_kind;
    int32_t  window;
    int32_t  separate_full_blocks;
    const int32_t* kv_num_blocks;       /* [B][H][q_blocks]            partial tiles per query block   */
    const int32_t* kv_indices;          /* [B][H][q_blocks][kv_blocks] ascending, zero padded          */
    const int32_t* full_kv_num_blocks;  /* [B][H][q_blocks]            full tiles per query block      */
    const int32_t* full_kv_indices;     /* [B][H][q_blocks][kv_blocks] ascending, zero padded          */
    /* The same tiles listed per kv block (the transposed lists the backward's dK/dV pass walks): */
    const int32_t* q_num_blocks;        /* [B][H][kv_blocks]           partial tiles per kv block      */
    const int32_t* q_indices;           /* [B][H][kv_blocks][q_blocks] ascending, zero padded          */
    const int32_t* full_q_num_blocks;   /* [B][H][kv_blocks]           full tiles per kv block         */
    const int32_t* full_q_indices;      /* [B][H][kv_blocks][q_blocks] ascending, zero padded          */
    int32_t  dq_kv_order;               /* dQ accumulation order over kv blocks: 1 descending, 0 ascending */
    int32_t  KV_BLOCK_SIZE;             /* kv block size of the lists (BLOCK_SIZE is the query one)   */
} fa_block_mask_info_t;

/*
 * fa_create_block_mask -- build the block mask of a fixed mask_mod on the GPU.
 *
 * Follows "tensorplay.nn.attention.create_block_mask" (signature and Parameters) and
 * "How to Use FlexAttention on Apple Silicon" ("Mask 1": B=None, H=None broadcast the
 * mask; build it once and reuse it).  A tile is dead when no pair in it is allowed,
 * full when every pair is allowed and the tile lies wholly inside Q_LEN x KV_LEN, and
 * partial otherwise.  Lists hold ascending kv-block indices padded with 0.
 *
 *   mask_kind   OR of FA_MASK_* bits (0 = no mask)
 *   params      may be NULL when mask_kind needs neither window nor doc_id
 *               (separate_full_blocks then defaults to 1, dq_kv_order to 1)
 *   B, H        batch and head extents; 0 means broadcast (stored as 1)
 *   Q_LEN, KV_LEN > 0
 *   BLOCK_SIZE  query block size of the lists fa_block_mask_get returns; the kv block size is
 *               params->kv_block_size, or BLOCK_SIZE when that is 0 (the page's int or
 *               (q, kv) tuple).  Any positive sizes with at most 16384 blocks per side.  The
 *               kernels always walk their own 128 x 128 tile lists, built alongside, so the
 *               block size changes what is read back, not the attention result.
 *   out_mask    receives the new mask; release it with fa_destroy_block_mask
 *
 * Work is enqueued on `stream`; the mask may be used by fa_forward on the same stream
 * at once, or on another stream after synchronising.  Errors: FA_ERR_INVALID_ARG,
 * FA_ERR_UNSUPPORTED, FA_ERR_OOM, FA_ERR_CUDA.
 */
fa_status_t fa_create_block_mask(uint32_t mask_kind, const fa_mask_params_t* params,
                                 int32_t B, int32_t H, int32_t Q_LEN, int32_t KV_LEN,
                                 int32_t BLOCK_SIZE, void* stream, fa_block_mask_t** out_mask);

/*
 * fa_block_mask_from_kv_blocks -- a block mask from caller-supplied block lists
 * ("tensorplay.nn.attention.create_block_mask", Parameters, dq_kv_order: explicit schedules
 * are taken by BlockMask.from_kv_blocks).
 *
 *   kv_num_blocks, kv_indices            device int32 [B'][H'][QBu][KVBu] (counts [B'][H'][QBu]):
 *                                        the partially masked blocks of each query block
 *   full_kv_num_blocks, full_kv_indices  the same for fully unmasked blocks, or both NULL
 *                                        (then every listed block is partial)
 * with B' = max(B, 1), H' = max(H, 1), QBu = ceil(Q_LEN / Q_BLOCK), KVBu = ceil(KV_LEN /
 * KV_BLOCK).  Q_BLOCK and KV_BLOCK must be multiples of 128 (else FA_ERR_UNSUPPORTED): each
 * block becomes its 128 x 128 tiles, with the block's class (a ragged tile is never full).
 * mask_kind and params give the mask_mod applied on partial tiles (0: none, every position
 * of a listed partial block attends).  Lists need not be sorted; the mask keeps a copy, read
 * back by fa_block_mask_get.  A count outside [0, KVBu] or an index outside the block grid is
 * ignored and recorded: fa_get_device_status then returns FA_ERR_INVALID_ARG.
 */
fa_status_t fa_block_mask_from_kv_blocks(uint32_t mask_kind, const fa_mask_params_t* params,
                                         int32_t B, int32_t H, int32_t Q_LEN, int32_t KV_LEN,
                                         int32_t Q_BLOCK, int32_t KV_BLOCK,
                                         const int32_t* kv_num_blocks, const int32_t* kv_indices,
                                         const int32_t* full_kv_num_blocks,
                                         const int32_t* full_kv_indices, void* stream,
                                         fa_block_mask_t** out_mask);

/*
 * fa_forward -- fused block-sparse attention forward.
 *
 * out = softmax(mask(score_mod(scale * q k^T))) v  and  lse = log(sum(exp(...))) per query
 * row, natural log, fp32 ("How to Use FlexAttention on Apple Silicon", "The two hooks":
 * mask_mod decides which pairs live, score_mod changes only live scores).  Only the
 * tiles the mask lists are visited; mask_mod is evaluated only on partial tiles.
 *
 *   q           (B, H, Q_LEN, D);  k, v (B, H, KV_LEN, D);  all the same dtype
 *   block_mask  from fa_create_block_mask with matching Q_LEN/KV_LEN and with B, H
 *               equal to q's or broadcast
 *   score_mod_kind / params   FA_SCORE_* bits; params may be NULL for FA_SCORE_NONE
 *   scale       multiplies q k^T before score_mod; <= 0 selects 1/sqrt(D)
 *   out         (B, H, Q_LEN, D), q's dtype, caller-owned
 *   lse         device fp32 [B][H][Q_LEN] contiguous, or NULL to skip it
 *
 * Supported: D in {64, 128} (else FA_ERR_UNSUPPORTED); any Q_LEN and KV_LEN >= 1 (a
 * ragged last tile is loaded zero-filled, its keys past KV_LEN are masked and its rows past
 * Q_LEN are not stored).  q, k, v, out, lse and alibi_slopes must be memory of the current
 * device (cudaMalloc or managed; host memory, pinned or not, gives FA_ERR_INVALID_ARG).  A query row with no allowed key gets out = 0, lse = -inf.
 * Device-side waits are bounded; a wait that runs out sets the mask's status word
 * (read it with fa_get_device_status) and the kernel returns early.
 */
fa_status_t fa_forward(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                       const fa_block_mask_t* block_mask, uint32_t score_mod_kind,
                       const fa_score_params_t* params, float scale,
                       fa_tensor_t* out, float* lse, void* stream);

/*
 * fa_create_block_mask_noalloc -- the block-mask build of fa_create_block_mask, writing into
 * caller-owned lists and allocating no device memory.  (The pages have no counterpart: it
 * exists for callers that cannot let a library allocate.)
 *
 * Who needs it: code running inside a framework whose caching allocator or arena already
 * owns the GPU's memory (a cudaMalloc behind its back escapes its accounting and can fail
 * once the pool holds most of HBM), plugins of inference runtimes whose enqueue path must
 * not allocate, and real-time deployments that forbid allocation after start-up; cudaMalloc
 * can also synchronise the device, which latency-critical callers cannot afford.
 *
 * Arguments are those of fa_create_block_mask, except that the four lists are written to
 * caller-owned device buffers laid out as in fa_block_mask_info_t:
 *   kv_num_blocks, full_kv_num_blocks   int32 [B'][H'][q_blocks]
 *   kv_indices, full_kv_indices         int32 [B'][H'][q_blocks][kv_blocks]
 * with B' = max(B, 1), H' = max(H, 1), q_blocks = ceil(Q_LEN/128), kv_blocks =
 * ceil(KV_LEN/128); every element is written.  params->doc_id is read in place (not copied)
 * and must stay valid until the stream has run the build.  The four buffers and doc_id must
 * be memory of the current device (host memory gives FA_ERR_INVALID_ARG).
 *
 * Limit and scratch: Q_LEN and KV_LEN may not exceed 4096 blocks (524288 positions); larger
 * requests return FA_ERR_UNSUPPORTED.  Document statistics go to a fixed 48 KiB
 * __device__ array that every GPU loading this library holds until exit.  All calls share
 * it (it keeps the last call's contents; each call writes every entry it reads), so calls
 * whose work overlaps on the GPU -- e.g. on two streams -- race.  The first call on a
 * device looks up the array's address (cudaGetSymbolAddress) with that device current and
 * keeps it for the life of the process; make that first call before any stream capture, and
 * do not use this entry point across a cudaDeviceReset of that device.
 */
fa_status_t fa_create_block_mask_noalloc(uint32_t mask_kind, const fa_mask_params_t* params,
                                         int32_t B, int32_t H, int32_t Q_LEN, int32_t KV_LEN,
                                         int32_t BLOCK_SIZE, int32_t* kv_num_blocks,
                                         int32_t* kv_indices, int32_t* full_kv_num_blocks,
                                         int32_t* full_kv_indices, void* stream);

/*
 * fa_forward_paged -- fa_forward with the keys and values in pages of a K/V cache: the
 * PagedAttention pattern expressed through block indices ("PyTorch 2.13 brings custom AI
 * attention to Mac", "What Attention Patterns Does FlexAttention Support?").
 *
 *   k_pages, v_pages   (n_pages, H, 128, D) pools, q's dtype: page p holds 128 consecutive
 *                      keys of one sequence for every head
 *   page_table         device int32 [B][page_table_stride]: entry (b, j) is the page holding
 *                      keys j*128 .. j*128+127 of batch b; page_table_stride >= the mask's
 *                      kv_blocks; only the entries of listed tiles are read
 *   block_mask         built for the logical lengths Q_LEN x KV_LEN (usually with kv_lens,
 *                      one context length per batch element, and no mask kind for decode)
 *   workspace          NULL, or device scratch of fa_forward_paged_workspace_bytes(block_mask,
 *                      B, H, Q_LEN, D) bytes, 16-byte aligned, caller-owned.  With Q_LEN <= 4 and
 *                      a workspace the call runs the split decode path: each (b, h)'s pages are
 *                      shared out to several CTAs on the CUDA cores (the work is reading K and
 *                      V once), whose partial results a second kernel merges; otherwise the
 *                      tensor-core forward runs.  Calls that overlap need distinct workspaces.
 * Everything else is fa_forward's.  A page index outside [0, n_pages) reads as zeros (the
 * split path skips the page) and is recorded: fa_get_device_status then returns
 * FA_ERR_INVALID_ARG.
 */
size_t fa_forward_paged_workspace_bytes(const fa_block_mask_t* block_mask, int64_t B, int64_t H,
                                        int64_t Q_LEN, int64_t D);   /* 0: no split path */
fa_status_t fa_forward_paged(const fa_tensor_t* q, const fa_tensor_t* k_pages,
                             const fa_tensor_t* v_pages, const int32_t* page_table,
                             int64_t page_table_stride, const fa_block_mask_t* block_mask,
                             uint32_t score_mod_kind, const fa_score_params_t* params, float scale,
                             fa_tensor_t* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * fa_backward -- gradients of fa_forward over the same block mask, deterministic.
 *
 * Given the forward's out and lse and the upstream gradient dout, writes
 *   dv = P^T dout,  dq = scale * dS k,  dk = scale * dS^T q,  with
 *   P = exp(score_mod(scale * q k^T) - lse) on live positions (0 elsewhere),
 *   dS = P * (dout v^T - rowsum(dout * out)) * score_mod'
 * ("PyTorch 2.13 brings custom AI attention to Mac", "What Else Shipped in PyTorch 2.13?":
 * a deterministic FlexAttention backward; "tensorplay.nn.attention.create_block_mask",
 * Parameters compute_dq_write_order / dq_kv_order: dQ accumulates its kv blocks in a fixed
 * order).  Here every sum runs in a fixed order on one CTA (no atomics), so repeated calls
 * give bitwise identical gradients; dQ accumulates in the mask's dq_kv_order.
 *
 *   q, k, v, out, lse, block_mask, score_mod_kind, params, scale: as passed to fa_forward,
 *               with out and lse the forward's results (lse must not be NULL here)
 *   dout        (B, H, Q_LEN, D), q's dtype
 *   dq          (B, H, Q_LEN, D); dk, dv (B, H, KV_LEN, D); q's dtype, caller-owned
 *   workspace   device scratch of at least fa_backward_workspace_bytes(B, H, Q_LEN) bytes,
 *               16-byte aligned, caller-owned; the call leaves nothing in it that a later call
 *               needs.  Calls that overlap on the GPU need distinct workspaces.
 *
 * Three kernels run on `stream`: a pre-pass (rowsum(dout * out) and lse into the workspace),
 * the dK/dV pass (one unit per kv block) and the dQ pass (one unit per query block).  Shapes,
 * dtypes and limits are fa_forward's.  Device-side waits are bounded as in fa_forward.
 */
size_t fa_backward_workspace_bytes(int64_t B, int64_t H, int64_t Q_LEN);
fa_status_t fa_backward(const fa_tensor_t* q, const fa_tensor_t* k, const fa_tensor_t* v,
                        const fa_tensor_t* out, const fa_tensor_t* dout, const float* lse,
                        const fa_block_mask_t* block_mask, uint32_t score_mod_kind,
                        const fa_score_params_t* params, float scale, fa_tensor_t* dq,
                        fa_tensor_t* dk, fa_tensor_t* dv, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * fa_masked_softmax -- the causal-masked softmax over materialised scores, in one kernel.
 *
 * probs[b,h,q,kv] = softmax over kv of  (q + offset >= kv ? scores[b,h,q,kv] : finfo.min)
 *
 * ("Fuse the causal mask into the SDPA fallback softmax", MLX pull request 3919, Summary and
 * Description: the chain greater_equal -> where(finfo.min) -> softmax with the select folded
 * into the softmax's loads.)  finfo.min is the scores dtype's lowest finite value; masked
 * entries come out exactly 0, and a row whose keys are all masked is uniform, 1/K, as the
 * chain gives.  The arithmetic is float32 (max, then the sum of 2^((x - max) log2 e), then
 * e / sum rounded to the output dtype), with the same reduction order whether or not the
 * mask is applied: with FA_MASK_CAUSAL the result is bit-identical to mask_kind 0 applied to
 * where(keep, scores, finfo.min).  Scores past the causal boundary are never read.
 *
 *   scores     (B, H, Q, K) fp16 or bf16 in an fa_tensor_t (S = Q rows, D = K keys); the key
 *              stride is 1, other strides multiples of 8 elements, data 16-byte aligned
 *   mask_kind  FA_MASK_CAUSAL, or 0 for the plain softmax (the chain's last step alone)
 *   offset     the position of query row 0 among the keys: row q keeps keys kv <= q + offset
 *              (K - Q when a chunk of Q queries closes a context of K keys; may be negative)
 *   probs      (B, H, Q, K), scores' dtype, caller-owned; may be `scores` itself with the same
 *              strides (each row is read before it is written), otherwise must not overlap it
 *
 * Limits: K a multiple of 8 and at most 32768 (else FA_ERR_UNSUPPORTED).  scores and probs
 * must be memory of the current device.  Asynchronous on `stream`; device-side waits are
 * bounded, and a wait that runs out sets a status word read by fa_masked_softmax_status.
 */
fa_status_t fa_masked_softmax(const fa_tensor_t* scores, uint32_t mask_kind, int64_t offset,
                              fa_tensor_t* probs, void* stream);

/* Synchronise `stream`, read and clear the status word of the fa_masked_softmax kernels:
 * FA_OK, FA_ERR_TIMEOUT (a bounded wait ran out), or FA_ERR_CUDA. */
fa_status_t fa_masked_softmax_status(void* stream);

/* Fill `info` with the mask's extents and device pointers.  FA_ERR_INVALID_ARG on NULL. */
fa_status_t fa_block_mask_get(const fa_block_mask_t* block_mask, fa_block_mask_info_t* info);

/*
 * Synchronise `stream`, read and clear the device status word that kernels using this
 * mask write when a bounded device-side wait runs out, or that fa_block_mask_from_kv_blocks
 * writes when the caller's lists were out of range, or fa_forward_paged when a page index
 * was.  Returns FA_OK, FA_ERR_TIMEOUT, FA_ERR_INVALID_ARG (lists or pages out of range), or
 * FA_ERR_CUDA if the stream reports an error.
 */
fa_status_t fa_get_device_status(const fa_block_mask_t* block_mask, void* stream);

/* Free a mask (NULL is ignored).  The caller must ensure no enqueued work still uses it. */
void fa_destroy_block_mask(fa_block_mask_t* block_mask);

/* Static string naming a status code. */
const char* fa_status_string(fa_status_t status);

/* One-line description of the last error returned on the calling thread ("" if none). */
const char* fa_last_error_message(void);

/*
 * Test hook for failure detection (no counterpart on the pages).  While `enable` is nonzero,
 * the data-moving warp of every kernel launched afterwards (process-wide) stops early: the
 * forward's TMA warp after the first query tiles, the backward's after the first unit's fixed
 * tiles, fa_masked_softmax's producer after its first row buffers.  A bounded wait then runs
 * past its limit (about two seconds), every role of the kernel unwinds and releases its tensor
 * memory, and the status word is set: fa_get_device_status (fa_masked_softmax_status for the
 * softmax) then returns FA_ERR_TIMEOUT.
 * The outputs of such a call are unspecified.  Pass 0 to restore normal operation.  Process
 * global state: not for use while other threads launch forwards.  Returns FA_OK.
 */
fa_status_t fa_debug_set_stall(int32_t enable);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
