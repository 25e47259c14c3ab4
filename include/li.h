/*
 * li.h -- C ABI of the Lightning Indexer forward pass for NVIDIA B200 (sm_100a).
 *
 * The operation (custom_pypto.npu_lightning_indexer_pto, function description formula;
 * lightning_indexer, "Function" steps 1-3 and "Formula"; aclnnLightningIndexerV2, formula and
 * main computation steps): for every query row t of batch b and every key j in the row's window,
 *
 *     I[t,j] = sum_{h < N1} w[t,h] * ReLU( q[t,h,:] . k[j,:] ),      D = 128, one key head,
 *
 * then the topk keys with the largest I, sorted by I descending (lower key index first on equal
 * scores), returned as int32 sparse_indices (-1 padded) and fp32 sparse_values (-inf padded)
 * (lightning_indexer and aclnnLightningIndexerV2, constraints on the invalid part).
 *
 * Windows (custom_pypto.npu_lightning_indexer_pto, parameter sparse_mode):
 *     mask_mode 0 (defaultMask):       0 <= j < L2_b
 *     mask_mode 3 (rightDownCausal):   0 <= j < L2_b  and  j <= i + L2_b - L1_b
 * where i is the row's position inside batch b, L1_b the batch's query rows in use (seqused_q[b]
 * when given, else all of them) and L2_b its key count. Indices are positions inside batch b's key
 * sequence, plus output_idx_offset[b] when given.
 *
 * Conventions shared by every entry point
 *   - All data pointers are DEVICE pointers of the current CUDA device (li_merge_topk's input
 *     lists may also be a peer GPU's memory); NULL means "absent".
 *   - The caller owns every buffer; the library never allocates device or pinned memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every launch
 *     is stream-ordered; no entry point except li_check_status synchronizes or reads device
 *     memory on the host, so li_metadata and li_indexer can be captured in a CUDA graph.
 *   - Argument errors are detected on the host before anything is launched and are returned as a
 *     status; the message is available from li_last_error_string(). Errors that depend on device
 *     data (non-monotone cu_seqlens, out-of-range block table entries, offsets overflowing int32,
 *     lengths above the declared maxima) are recorded in a device status word inside the
 *     workspace and reported by li_check_status(); the affected rows hold unspecified values but
 *     no access leaves the caller's buffers.
 */
#ifndef LI_H_
#define LI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LI_ABI_VERSION 6

typedef enum li_layout {
    LI_LAYOUT_BSND = 0,     /* dense batch: q (B,S1,N1,D), k (B,S2,1,D), w (B,S1,N1)            */
    LI_LAYOUT_TND = 1,      /* packed varlen: q (T1,N1,D), k (T2,1,D), w (T1,N1) + cu_seqlens   */
    LI_LAYOUT_PA_BSND = 2   /* paged keys only: k (num_blocks, block_size, 1, D) + block_table  */
} li_layout;

typedef enum li_status {
    LI_OK = 0,
    LI_ERR_INVALID_ARG = 1,     /* an argument violates the documented contract             */
    LI_ERR_UNSUPPORTED = 2,     /* a valid request this build does not implement, e.g. more
                                   than 2^31-1 query-head rows (query rows x num_heads_q) or
                                   key rows (B*S2, T2 or num_blocks*block_size)                 */
    LI_ERR_WORKSPACE = 3,       /* workspace / metadata buffer too small or misaligned      */
    LI_ERR_CUDA = 4,            /* a CUDA runtime call failed (message has the CUDA error)  */
    LI_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait gave up (li_check_status)     */
    LI_ERR_DEVICE_DATA = 6      /* device-resident lengths/tables/offsets were invalid      */
} li_status;

typedef enum li_dtype {
    LI_DTYPE_BF16 = 0,
    LI_DTYPE_FP16 = 1,
    LI_DTYPE_FP32 = 2,                  /* w only                                              */
    LI_DTYPE_FP8_E4M3 = 3               /* q and k only, with q_descale and k_descale          */
} li_dtype;

/* Device status word bits, as reported through li_check_status(). */
#define LI_DEVERR_TIMEOUT   0x1u   /* a bounded wait (mbarrier / scheduler) ran out            */
#define LI_DEVERR_LENGTHS   0x2u   /* cu_seqlens not monotone, or a length above its maximum  */
#define LI_DEVERR_TABLE     0x4u   /* a block_table entry in use is outside [0, num_blocks)    */
#define LI_DEVERR_OFFSET    0x8u   /* output_idx_offset < 0, or index + offset > INT32_MAX     */
#define LI_DEVERR_METADATA  0x10u   /* the metadata passed was built for other arguments        */
#define LI_DEVERR_INTERNAL  0x20u   /* the score kernel's shared memory came misaligned         */
#define LI_DEVERR_MERGE_ORDER 0x40u /* li_merge_topk: an input row out of order, or a valid entry
                                       after padding                                          */
#define LI_DEVERR_DESCALE   0x80u   /* fp8 q/k: a q_descale or k_descale in use is not a positive
                                       finite number                                          */
#define LI_DEVERR_BOUNDS    0x100u  /* bounds-checked build only (compiled with LI_DEBUG): a
                                       computed shared- or global-memory index fell outside its
                                       buffer; the access was skipped. Never set by the release
                                       library, whose indices are bounded by construction.     */

/*
 * Arguments of one indexer call. Mirrors the pages' prototypes (lightning_indexer, "Prototype":
 * q, k, w, topk, cu_seqlens_q/k, seqused_q/k, block_table, output_idx_offset, max_seqlen_q/k,
 * layout_q/k, mask_mode, return_value) with the tensor shapes made explicit.
 */
typedef struct li_args {
    const void *q;                      /* dtype_qk, BSND (B,S1,N1,128) or TND (T1,N1,128),
                                           dense                                               */
    const void *k;                      /* dtype_qk, BSND (B,S2,1,128), TND (T2,1,128) or
                                           PA_BSND (num_blocks, block_size, 1, 128), dense     */
    const void *w;                      /* dtype_w, (B,S1,N1) or (T1,N1), dense                 */
    const int32_t *cu_seqlens_q;        /* [B+1], non-decreasing; required iff layout_q == TND  */
    const int32_t *cu_seqlens_k;        /* [B+1], non-decreasing; required iff layout_k == TND  */
    const int32_t *seqused_q;           /* [B] or NULL: query rows in use per batch; rows past
                                           it are all padding and the causal window aligns to it */
    const int32_t *seqused_k;           /* [B]: keys per batch. Required for PA_BSND; for the
                                           other layouts, when given, caps the batch's keys      */
    const int32_t *block_table;         /* [B, block_table_stride]; required for PA_BSND        */
    int64_t block_table_stride;         /* entries per batch row of block_table                 */
    const int32_t *output_idx_offset;   /* [B] or NULL: added to every valid output index      */
    int32_t batch;                      /* B (number of sequences)                              */
    int32_t q_len;                      /* BSND: S1 ; TND: T1 (rows of q)                       */
    int32_t k_len;                      /* BSND: S2 ; TND: T2 (rows of k) ; PA_BSND: ignored    */
    int32_t max_seqlen_q;               /* upper bound of every batch's query rows (BSND: S1)   */
    int32_t max_seqlen_k;               /* upper bound of every batch's key count (BSND: S2)    */
    int32_t num_blocks;                 /* PA_BSND: blocks in the cache                         */
    int32_t block_size;                 /* PA_BSND: keys per block, 1..1024                     */
    int32_t num_heads_q;                /* N1, 1..64                                            */
    int32_t num_heads_k;                /* N2, must be 1                                        */
    int32_t head_dim;                   /* D, must be 128                                       */
    int32_t topk;                       /* 1..8192                                              */
    int32_t layout_q;                   /* li_layout: BSND or TND                               */
    int32_t layout_k;                   /* li_layout: BSND, TND or PA_BSND                      */
    int32_t mask_mode;                  /* 0 (no mask) or 3 (right-down causal)                 */
    int32_t dtype_qk;                   /* li_dtype of q and k (one type, lightning_indexer,
                                           "Constraints"): LI_DTYPE_BF16, LI_DTYPE_FP16 or
                                           LI_DTYPE_FP8_E4M3 (with q_descale / k_descale,
                                           below); products accumulate in fp32 in every case */
    int32_t dtype_w;                    /* li_dtype of w: BF16, FP16 or FP32 (the pages'
                                           single-operator example passes fp16 q, k and fp32
                                           w); fp32 w must be 4-byte aligned               */
    int32_t return_value;               /* 1: write sparse_values too; 0: indices only          */
    /* Compressed keys (lightning_indexer, "Prototype": cmp_ratio, cmp_residual_k; "Constraints":
     * cmp_residual_k[b] < cmp_ratio, passed only with cmp_ratio > 1 and mask_mode 3). Each key
     * stands for cmp_ratio original tokens and batch b's sequence has cmp_residual_k[b] tokens
     * past its last whole key. The pages state no mask rule for them; the reading implemented:
     * under mask_mode 3 key j is kept for query row i when its last original token is visible,
     * (j+1)*cmp_ratio - 1 <= i + L2_b*cmp_ratio + cmp_residual_k[b] - L1_b. Device values outside
     * [0, cmp_ratio) set LI_DEVERR_LENGTHS. */
    const int32_t *cmp_residual_k;      /* [B] int32, or NULL                                   */
    int32_t cmp_ratio;                  /* original tokens per key; 0 or 1 = not compressed     */
    /* Quantized q and k (aclnnLightningIndexerV2, parameter dimensions: q_descale and k_descale
     * are named with q, k and w and nothing more is said). The reading implemented: with
     * dtype_qk = LI_DTYPE_FP8_E4M3, q and k hold OCP E4M3 codes (1 byte per element, rows of
     * 128 bytes, 16-byte aligned) and the values they stand for are code x q_descale[row, head]
     * and code x k_descale[key row]. Both arrays are fp32, 4-byte aligned, required with fp8
     * and NULL otherwise. Scales in use must be positive and finite (LI_DEVERR_DESCALE). */
    const float *q_descale;             /* [rows x num_heads_q], laid out like w                */
    const float *k_descale;             /* one per key row, laid out like k without D: BSND
                                           (B, S2), TND (T2), PA_BSND (num_blocks, block_size)  */
} li_args;

/*
 * li_metadata_workspace_size -- bytes of the metadata buffer li_metadata() fills.
 * Host only. Validates `args` (same checks as li_indexer_workspace_size, device pointers are not
 * dereferenced). Counterpart of the pages' lightning_indexer_metadata sizing (lightning_indexer,
 * "Function": the metadata op produces the per-core task list) and of the first phase of the
 * two-phase call (aclnnLightningIndexerV2: GetWorkspaceSize validates and sizes, then execute).
 * Returns LI_OK and writes *bytes, or an argument error.
 */
li_status li_metadata_workspace_size(const li_args *args, size_t *bytes);

/*
 * li_metadata -- build the schedule (work list) for li_indexer on `stream`.
 * Replaces the pages' per-AI-core task list (lightning_indexer, "Function" and "Prototype":
 * lightning_indexer_metadata must run before lightning_indexer) by a list of query blocks and key
 * ranges ordered longest first, read by the persistent sm_100a kernels. It reads the
 * device-resident lengths (cu_seqlens, seqused) on the device; nothing is read back to the host.
 * `metadata` is a device buffer of at least li_metadata_workspace_size() bytes, 256-byte aligned,
 * owned by the caller and valid until the li_indexer calls that use it have completed. Invalid
 * device data sets bits in the metadata's status word, which li_indexer copies to its own.
 */
li_status li_metadata(const li_args *args, void *metadata, size_t bytes, void *stream);

/*
 * li_plan -- the schedule li_indexer() will use for `args`, and how many kernels it launches.
 * Host only; validates like li_metadata_workspace_size and dereferences no device pointer. The
 * pages split the work per AI core inside lightning_indexer_metadata (lightning_indexer,
 * "Function"); this reports the sm_100a counterpart's choices so callers can size graphs and
 * count launches:
 *   tq            query rows per work item (tq x num_heads_q <= 256 MMA columns)
 *   kc            keys per work item, 0 when each item covers its rows' whole window
 *   max_items     capacity of the work list
 *   dense         0: a schedule kernel builds the work list; 1: dense BSND closed form; 2: closed
 *                 form for one query block per batch with per-batch key lengths (decode); with
 *                 1 or 2 no schedule kernel runs
 *   kernels       kernels one li_indexer call launches with metadata == NULL (0 when there are no
 *                 query rows); one fewer schedule kernel when a metadata buffer is passed
 *   score_tc      1 when the score step runs on the tcgen05 kernel (every block_size of a
 *                 paged cache included), 0 on the CUDA-core kernel (LI_SCORE_KERNEL=simple, or
 *                 a shape outside the kernel's limits)
 *   select_pieces key pieces each row's selection is cut into (1: one CTA per row). Few very long
 *                 rows (decode over a long context) are split so that more SMs work on them;
 *                 the pieces' lists are merged as li_merge_topk merges key ranges, one more
 *                 kernel, and the workspace holds the partial lists
 * Returns LI_OK and fills *info, or an argument error.
 */
typedef struct li_plan_info {
    int32_t tq;
    int32_t kc;
    int32_t max_items;
    int32_t dense;
    int32_t kernels;
    int32_t score_tc;
    int32_t select_pieces;
} li_plan_info;
li_status li_plan(const li_args *args, li_plan_info *info);

/*
 * li_indexer_workspace_size -- bytes of scratch li_indexer() needs for `args`.
 * Host only; validates like li_metadata_workspace_size. The size covers the device status word,
 * the scheduler counters, room for an inline schedule, and the fp32 score rows the selection step
 * reads (rows x max_seqlen_k x 4 bytes).
 */
li_status li_indexer_workspace_size(const li_args *args, size_t *bytes);

/*
 * li_indexer -- the forward pass (lightning_indexer, "Prototype" and "Function"): scores,
 * ReLU, weights, head sum, mask, top-k, padding, for every query row.
 *   metadata        schedule from li_metadata() for the same args, or NULL to build it inline
 *                   into the workspace (one extra small kernel launch).
 *   workspace       device scratch of >= li_indexer_workspace_size() bytes, 256-byte aligned.
 *                   Contents on entry are ignored; after the call it holds the status word.
 *   sparse_indices  int32 output, (B,S1,1,topk) for BSND q or (T1,1,topk) for TND q.
 *   sparse_values   fp32 output of the same shape, or NULL when args->return_value == 0.
 * Every output row is written (valid entries first, then -1 / -inf). Deterministic: the same
 * inputs give bit-identical outputs (aclnnLightningIndexerV2 and lightning_indexer, deterministic
 * computation). Returns after queueing the kernels; use li_check_status to learn about device
 * data errors.
 */
li_status li_indexer(const li_args *args, const void *metadata, void *workspace,
                     size_t workspace_bytes, int32_t *sparse_indices, float *sparse_values,
                     void *stream);

/*
 * li_check_status -- synchronize `stream`, read the device status word of `workspace` (the one
 * passed to the last li_indexer on that stream) into *device_bits (LI_DEVERR_* bits, may be NULL)
 * and map it to a status: LI_OK, LI_ERR_DEVICE_TIMEOUT or LI_ERR_DEVICE_DATA. A CUDA error
 * raised by the stream is returned as LI_ERR_CUDA.
 */
li_status li_check_status(const void *workspace, void *stream, uint32_t *device_bits);

/*
 * li_set_stage_events -- benchmarking hook. With n_events == 6, every later li_indexer call
 * records events[0]/[1] around the inline schedule build (only when metadata == NULL),
 * events[2]/[3] around the score kernel and events[4]/[5] around the selection kernel, on the
 * call's stream, so a caller can time each kernel with cudaEventElapsedTime. The events are
 * cudaEvent_t handles passed as void*, created by the caller (timing enabled) and owned by it.
 * n_events == 0 turns the hook off. The setting is process-wide; do not change it while another
 * host thread is inside li_indexer. Returns LI_ERR_INVALID_ARG for any other count.
 */
li_status li_set_stage_events(void *const *events, int32_t n_events);

/*
 * li_indexer_noalloc -- li_indexer for callers that may not allocate device memory.
 * The pages have no counterpart; this entry point exists for integrations where the caller
 * cannot obtain a workspace: plugin or custom-op interfaces whose enqueue step offers no
 * allocator, runtimes that reserve all device memory up front and forbid allocation afterwards,
 * and real-time loops where cudaMalloc's implicit synchronization and latency are not allowed.
 *
 * It runs exactly the li_indexer path with metadata built inline, using as workspace a scratch
 * array compiled into the library (a static device array of LI_NOALLOC_SCRATCH_BYTES). The
 * caller passes the inputs in `args` and the outputs as with li_indexer, plus `device_status`:
 * a device uint32 (or NULL) that receives the call's device status word, stream-ordered, so
 * li_check_status(device_status, stream, &bits) reports data errors of this call. It is written
 * only when the call returns LI_OK; on any error return it keeps its previous contents, and the
 * returned status (with li_last_error_string) is the call's result.
 *
 *   - Problems whose workspace (li_indexer_workspace_size) exceeds LI_NOALLOC_SCRATCH_BYTES are
 *     rejected on the host with LI_ERR_WORKSPACE and a message giving both sizes.
 *   - No cudaMalloc, cudaFree or other allocating call is made. The array occupies
 *     LI_NOALLOC_SCRATCH_BYTES on every device where the library's module is loaded (from the
 *     first call on that device, or from library load under eager module loading) until the
 *     process exits.
 *   - The first call on a device looks up the array's device address (once per device, with that
 *     device current); make that first call before any stream capture.
 *   - Every call on a device shares the one array, and its contents persist between calls (the
 *     call clears what must start at zero). Calls whose kernels overlap on the GPU -- concurrent
 *     streams, or several host threads -- race on the array and give undefined results:
 *     serialize them.
 */
#define LI_NOALLOC_SCRATCH_BYTES (32u << 20)
li_status li_indexer_noalloc(const li_args *args, int32_t *sparse_indices, float *sparse_values,
                             uint32_t *device_status, void *stream);

/*
 * li_merge_topk -- the split-merge step after a key-range split: the top-k of the union of
 * several per-row top-k lists. A row whose keys are split into disjoint ranges (one range per GPU,
 * or per piece of a very long row), each range selected by li_indexer with output_idx_offset set
 * to the range's first key (so the indices are global), is merged back here. [reading] The pages
 * select over a row's whole window (lightning_indexer, "Function" step 3; aclnnLightningIndexerV2,
 * "主要计算过程"); the first topk of the union under the same order is that selection.
 *
 *   idx_in[l], val_in[l]  list l < n_lists: [rows, topk_in] int32 / fp32, row-major, as li_indexer
 *                         writes them: each row ordered by score descending, then index ascending,
 *                         with its padding (index < 0) after the valid entries. Indices must be
 *                         distinct across lists. Device memory, or a peer GPU's memory that the
 *                         current device can load from (plain loads, nothing else).
 *   idx_out, val_out      [rows, topk_out]: the first topk_out valid entries of the union in that
 *                         order, then -1 / -inf. val_out may be NULL (indices only).
 *   device_status         device uint32 or NULL: LI_DEVERR_MERGE_ORDER is OR-ed in when an input
 *                         row (its first topk_out entries) is out of order or has a valid entry
 *                         after padding; the output is then unspecified. Read it with
 *                         li_check_status(device_status, stream, &bits).
 *
 * Entries equal in score and index found in two lists (not a valid input) both appear, the lower
 * list first. Only the first topk_out entries of an input row are read. Returns LI_ERR_INVALID_ARG
 * for n_lists outside [1, LI_MERGE_MAX_LISTS], rows < 0, topk_in or topk_out outside [1, 8192], a
 * NULL list or idx_out, or a pointer not 4-byte aligned; LI_ERR_UNSUPPORTED for rows > 2^31-1;
 * LI_ERR_CUDA when the launch fails. Stream-ordered, allocates nothing, graph-capturable, and
 * deterministic.
 */
#define LI_MERGE_MAX_LISTS 16
typedef struct li_merge_args {
    const int32_t *idx_in[LI_MERGE_MAX_LISTS];
    const float *val_in[LI_MERGE_MAX_LISTS];
    int32_t *idx_out;
    float *val_out;
    uint32_t *device_status;
    int64_t rows;
    int32_t n_lists;
    int32_t topk_in;
    int32_t topk_out;
    int32_t reserved;                   /* must be 0 */
} li_merge_args;
li_status li_merge_topk(const li_merge_args *args, void *stream);

/*
 * li_kl_grad -- the indexer's backward with the KL loss (torch_npu.npu_sparse_lightning_indexer_
 * grad_kl_loss, formulas 1-4). For every query row r and its selected keys s (sparse_indices,
 * positions in the row's batch, -1 padded):
 *     I[s] = sum_h w[r,h] ReLU(qi[r,h,:] . ki[s,:])
 *     p[s] ~ sum_g exp(scale (q[r,g,:] . k[s,:] + q_rope[r,g,:] . k_rope[s,:]) - softmax_max[r,g])
 *            / softmax_sum[r,g], normalised to 1 over the row's selected keys
 *     loss = sum_r sum_s p[s] log(p[s] / softmax(I)[s]),   dI = softmax(I) - p
 *     d_w[r,h] = sum_s dI[s] ReLU(S[h,s]),  dS[h,s] = dI[s] w[r,h] [S[h,s] > 0]  (S = qi . ki)
 *     d_qi[r,h,:] = sum_s dS[h,s] ki[s,:],   d_ki[s,:] = sum over rows of sum_h dS[h,s] qi[r,h,:]
 * [reading] the sums over keys run over the selected keys; p is the head sum of the main
 * attention softmax rebuilt from its forward statistics and renormalised; the loss sums the rows.
 * Layout BSND: q (B,S1,G,Dm), k (B,S2,1,Dm), q_rope (B,S1,G,Dr) / k_rope (B,S2,1,Dr) or both NULL
 * (Dr = 0), qi (B,S1,H,128), ki (B,S2,1,128), w (B,S1,H), all bf16; sparse_indices
 * (B,S1,1,topk) int32; softmax_max / softmax_sum (B,1,S1,G) fp32. Outputs, fp32: *loss (one
 * value), d_qi like qi, d_ki like ki (zeroed by the call, then accumulated), d_w like w.
 * G in [1, 128], Dm in [1, 576] and Dr in [0, 64] multiples of 8, H in [1, 64], topk in
 * [1, 2048]. Selected positions must lie in [0, S2) and be distinct within a row; others set
 * LI_DEVERR_LENGTHS and are skipped. Stream-ordered, no allocation, loss summed in a fixed order.
 * Two kernels: shapes with Dm a multiple of 64 up to 512, Dr 0 or 64, G <= 32 and H <= 64 run on
 * the tensor cores (tcgen05: the scores and both gradient products; dS enters the products as a
 * bf16 hi + lo pair, 16 significant bits), every output bit-reproducible: each CTA owns a fixed
 * set of rows and adds its d_ki rows into its own slice of a partial buffer in the workspace,
 * and the slices are summed per key in a fixed order. Other shapes run on CUDA cores with d_ki
 * accumulated by atomic adds (rounding may differ from run to run). li_kl_grad_workspace_size
 * gives the bytes: the status word, one fp32 per row, and on the tensor-core path
 * SMs x B x S2 x 128 fp32 of partial d_ki (the SM count of the current device).
 */
typedef struct li_kl_args {
    const void *q, *k, *q_rope, *k_rope;     /* bf16 main attention                          */
    const void *qi, *ki, *w;                 /* bf16 indexer query, key and weights          */
    const int32_t *sparse_indices;
    const float *softmax_max, *softmax_sum;
    float scale;
    int32_t batch, s1, s2;                   /* B, S1 (query rows per batch), S2 (keys)      */
    int32_t G, Dm, Dr, H, topk;
    int32_t reserved;                        /* must be 0                                    */
} li_kl_args;
li_status li_kl_grad_workspace_size(const li_kl_args *args, size_t *bytes);
li_status li_kl_grad(const li_kl_args *args, void *workspace, size_t workspace_bytes, float *loss,
                     float *d_qi, float *d_ki, float *d_w, void *stream);

/*
 * li_sparse_attention -- attention of every query row over the keys the indexer selected for it,
 * the indexer's consumer (aclnnLightningIndexerV2, main computation steps: the selected indices
 * are the attention's input; aclnnSparseFlashAttentionGrad, calculation formula: the selected keys
 * and values are gathered by the top-k indices, and value = key is the supported case). For query
 * row r of batch b, head g and the row's selected keys s:
 *     x[s]     = scale * (q[r,g,:] . k[s,:] + q_rope[r,g,:] . k_rope[s,:])
 *     o[r,g,:] = sum_s exp(x[s] - m) k[s,:] / l,   m = max_s x[s],   l = sum_s exp(x[s] - m)
 * [reading] the value rows are the key rows (all Dm dims; the rope dims only enter the scores).
 * The statistics m and l are the inputs li_kl_grad takes as softmax_max / softmax_sum.
 *
 * Layouts, all bf16: q (B,S1,G,Dm) and q_rope (B,S1,G,Dr); keys either dense, layout_k =
 * LI_LAYOUT_BSND: k (B,S2,1,Dm) and k_rope (B,S2,1,Dr), or paged, layout_k = LI_LAYOUT_PA_BSND
 * (lightning_indexer, "Prototype": block_table and the paged key cache): k (num_blocks,
 * block_size,1,Dm) and k_rope (num_blocks,block_size,1,Dr), key position v of batch b in cache
 * row block_table[b * block_table_stride + v / block_size] * block_size + v % block_size.
 * q_rope and k_rope are both NULL when Dr = 0. sparse_indices (B,S1,1,topk) int32, positions in
 * the row's batch (as li_indexer writes them without output_idx_offset; S2 bounds them for both
 * layouts); a negative entry selects nothing, an entry >= S2 selects nothing and sets
 * LI_DEVERR_LENGTHS, a block-table entry outside [0, num_blocks) selects nothing and sets
 * LI_DEVERR_TABLE. Entries may repeat (each counts).
 * Outputs, fp32: out (B,S1,G,Dm); softmax_max and softmax_sum (B,1,S1,G). A row that selects no
 * key gets out = 0, softmax_max = -inf, softmax_sum = 0.
 * Limits: G in [1, 32], Dm in {128, 256, 384, 512}, Dr in {0, 64}, topk in [1, 8192], S2 >= 1
 * when there are rows, scale > 0; q, k, q_rope, k_rope 16-byte aligned, the rest 4-byte aligned;
 * PA_BSND: block_size in [1, 1024], num_blocks >= 1, block_table_stride >= ceil(S2/block_size);
 * BSND: the block-table fields 0 / NULL. Argument errors return LI_ERR_INVALID_ARG before any
 * launch.
 * Numerics: products and sums in fp32 on the tensor cores; the softmax weights enter the value
 * product rounded to bf16 (the normaliser l is the fp32 sum of the unrounded weights).
 * The workspace (li_sparse_attention_workspace_size: 256 bytes) holds the device status word
 * (read it with li_check_status) and a row counter; its contents on entry are ignored.
 * Stream-ordered, no allocation, deterministic (bit-identical reruns).
 */
typedef struct li_attn_args {
    const void *q, *k, *q_rope, *k_rope;    /* bf16, see above                                   */
    const int32_t *sparse_indices;
    float scale;
    int32_t batch, s1, s2;                  /* B, S1 (query rows per batch), S2 (keys per batch) */
    int32_t G, Dm, Dr, topk;
    int32_t layout_k;                       /* LI_LAYOUT_BSND or LI_LAYOUT_PA_BSND               */
    const int32_t *block_table;             /* PA_BSND: (B, block_table_stride); else NULL       */
    int32_t block_table_stride;             /* PA_BSND: >= ceil(S2 / block_size); else 0         */
    int32_t num_blocks, block_size;         /* PA_BSND: >= 1 and 1..1024; else 0                 */
    int32_t reserved;                       /* must be 0                                         */
} li_attn_args;
li_status li_sparse_attention_workspace_size(const li_attn_args *args, size_t *bytes);
li_status li_sparse_attention(const li_attn_args *args, void *workspace, size_t workspace_bytes,
                              float *out, float *softmax_max, float *softmax_sum, void *stream);

/* Message of the last failing call on this host thread ("" if none). */
const char *li_last_error_string(void);

/* LI_ABI_VERSION of the loaded library. */
int32_t li_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LI_H_ */
