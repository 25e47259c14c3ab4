// Host side of the C ABI declared in include/li.h: argument validation, schedule choice,
// workspace sizing and the launch sequence. Mirrors the pages' two-phase convention
// (aclnnLightningIndexerV2: a first call validates the arguments and sizes the workspace, a
// second call runs on a stream) and their metadata-then-indexer order (lightning_indexer,
// "Prototype").
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "li_attn.cuh"
#include "li_internal.cuh"
#include "li_kl.cuh"
#include "li_merge.cuh"
#include "li_select.cuh"

namespace {

thread_local std::string g_err;

li_status fail(li_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

li_status ok() {
    g_err.clear();
    return LI_OK;
}

cudaEvent_t g_stage_events[6] = {};
bool g_stage_events_on = false;

void stage_mark(int i, cudaStream_t st) {
    if (g_stage_events_on && g_stage_events[i]) cudaEventRecord(g_stage_events[i], st);
}

// NVTX range around each entry point and each stage it enqueues, for timeline tools (Nsight
// Systems); without a tool attached a push/pop pair costs a few nanoseconds. Building with
// -DNVTX_DISABLE compiles them out.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Which score kernel runs: the tensor-core kernel unless LI_SCORE_KERNEL=simple selects the
// CUDA-core one (a debugging switch; both write the same score rows).
bool use_simple_kernel() {
    const char *e = std::getenv("LI_SCORE_KERNEL");
    return e && std::strcmp(e, "simple") == 0;
}

li_status validate(const li_args *a, li::Problem *p, li::Schedule *s) {
    if (!a) return fail(LI_ERR_INVALID_ARG, "args is NULL");
    if (a->num_heads_q < 1 || a->num_heads_q > li::kMaxHeads)
        return fail(LI_ERR_INVALID_ARG, "num_heads_q=%d outside [1, 64]", a->num_heads_q);
    if (a->num_heads_k != 1)
        return fail(LI_ERR_INVALID_ARG, "num_heads_k=%d, only 1 key head is supported",
                    a->num_heads_k);
    if (a->head_dim != li::kHeadDim)
        return fail(LI_ERR_INVALID_ARG, "head_dim=%d, only 128 is supported", a->head_dim);
    if (a->topk < 1 || a->topk > li::kMaxTopk)
        return fail(LI_ERR_INVALID_ARG, "topk=%d outside [1, 8192]", a->topk);
    if (a->mask_mode != 0 && a->mask_mode != 3)
        return fail(LI_ERR_INVALID_ARG, "mask_mode=%d, must be 0 or 3", a->mask_mode);
    // compressed keys: residuals are passed exactly when cmp_ratio > 1 under mask_mode 3
    // (lightning_indexer / aclnnLightningIndexerV2 constraints)
    if (a->cmp_ratio < 0)
        return fail(LI_ERR_INVALID_ARG, "cmp_ratio=%d < 0", a->cmp_ratio);
    if ((a->cmp_ratio > 1 && a->mask_mode == 3) != (a->cmp_residual_k != nullptr))
        return fail(LI_ERR_INVALID_ARG,
                    "cmp_residual_k is required with cmp_ratio > 1 and mask_mode 3, else absent");
    if (a->layout_q != LI_LAYOUT_BSND && a->layout_q != LI_LAYOUT_TND)
        return fail(LI_ERR_INVALID_ARG, "layout_q=%d, must be BSND or TND", a->layout_q);
    if (a->layout_k != LI_LAYOUT_BSND && a->layout_k != LI_LAYOUT_TND &&
        a->layout_k != LI_LAYOUT_PA_BSND)
        return fail(LI_ERR_INVALID_ARG, "layout_k=%d, must be BSND, TND or PA_BSND", a->layout_k);
    if (a->dtype_qk != LI_DTYPE_BF16 && a->dtype_qk != LI_DTYPE_FP16 &&
        a->dtype_qk != LI_DTYPE_FP8_E4M3)
        return fail(LI_ERR_INVALID_ARG, "dtype_qk=%d, must be bf16, fp16 or fp8 e4m3", a->dtype_qk);
    if ((a->dtype_qk == LI_DTYPE_FP8_E4M3) != (a->q_descale != nullptr) ||
        (a->dtype_qk == LI_DTYPE_FP8_E4M3) != (a->k_descale != nullptr))
        return fail(LI_ERR_INVALID_ARG, "q_descale and k_descale go with fp8 q/k, and only with it");
    if (!aligned(a->q_descale, 4) || !aligned(a->k_descale, 4))
        return fail(LI_ERR_INVALID_ARG, "q_descale and k_descale must be 4-byte aligned");
    if (a->dtype_w != LI_DTYPE_BF16 && a->dtype_w != LI_DTYPE_FP16 && a->dtype_w != LI_DTYPE_FP32)
        return fail(LI_ERR_INVALID_ARG, "dtype_w=%d, must be bf16, fp16 or fp32", a->dtype_w);
    if (a->return_value != 0 && a->return_value != 1)
        return fail(LI_ERR_INVALID_ARG, "return_value=%d, must be 0 or 1", a->return_value);
    if (a->batch < 0) return fail(LI_ERR_INVALID_ARG, "batch=%d < 0", a->batch);
    if (a->q_len < 0) return fail(LI_ERR_INVALID_ARG, "q_len=%d < 0", a->q_len);
    if (a->layout_k != LI_LAYOUT_PA_BSND && a->k_len < 0)
        return fail(LI_ERR_INVALID_ARG, "k_len=%d < 0", a->k_len);
    if (a->max_seqlen_k < 0) return fail(LI_ERR_INVALID_ARG, "max_seqlen_k=%d < 0", a->max_seqlen_k);
    if (a->max_seqlen_q < 0) return fail(LI_ERR_INVALID_ARG, "max_seqlen_q=%d < 0", a->max_seqlen_q);
    const int64_t rows0 = a->layout_q == LI_LAYOUT_TND ? (int64_t)a->q_len
                                                      : (int64_t)a->batch * a->q_len;
    const bool may_have_keys = a->layout_k == LI_LAYOUT_PA_BSND || a->k_len > 0;
    // Empty tensors may come with NULL data pointers: q and w are needed only when there are
    // query rows, k only when there can be keys.
    if (rows0 > 0 && (!a->q || !a->w)) return fail(LI_ERR_INVALID_ARG, "q and w are required");
    if (rows0 > 0 && may_have_keys && !a->k) return fail(LI_ERR_INVALID_ARG, "k is required");
    if (!aligned(a->q, 16) || !aligned(a->k, 16) ||
        !aligned(a->w, a->dtype_w == LI_DTYPE_FP32 ? 4 : 2))
        return fail(LI_ERR_INVALID_ARG, "q and k must be 16-byte aligned, w aligned to its type");
    if (a->layout_q == LI_LAYOUT_TND && !a->cu_seqlens_q)
        return fail(LI_ERR_INVALID_ARG, "layout_q TND requires cu_seqlens_q");
    if (a->layout_k == LI_LAYOUT_TND && !a->cu_seqlens_k)
        return fail(LI_ERR_INVALID_ARG, "layout_k TND requires cu_seqlens_k");
    if (a->layout_q == LI_LAYOUT_BSND && a->cu_seqlens_q)
        return fail(LI_ERR_INVALID_ARG, "cu_seqlens_q is only for layout_q TND");
    if (a->layout_k != LI_LAYOUT_TND && a->cu_seqlens_k)
        return fail(LI_ERR_INVALID_ARG, "cu_seqlens_k is only for layout_k TND");
    if (a->layout_k == LI_LAYOUT_PA_BSND) {
        if (!a->seqused_k) return fail(LI_ERR_INVALID_ARG, "layout_k PA_BSND requires seqused_k");
        if (!a->block_table) return fail(LI_ERR_INVALID_ARG, "layout_k PA_BSND requires block_table");
        if (a->block_size < 1 || a->block_size > 1024)
            return fail(LI_ERR_INVALID_ARG, "block_size=%d outside [1, 1024]", a->block_size);
        if (a->num_blocks < 1) return fail(LI_ERR_INVALID_ARG, "num_blocks=%d < 1", a->num_blocks);
        if (a->block_table_stride < 1)
            return fail(LI_ERR_INVALID_ARG, "block_table_stride=%lld < 1",
                        (long long)a->block_table_stride);
        // 32-byte block alignment (lightning_indexer, Constraints) holds for any block size:
        // one key is 128 bf16 = 256 bytes.
    } else if (a->block_table) {
        return fail(LI_ERR_INVALID_ARG, "block_table is only for layout_k PA_BSND");
    }
    if (a->layout_q == LI_LAYOUT_BSND && a->max_seqlen_q != 0 && a->max_seqlen_q != a->q_len)
        return fail(LI_ERR_INVALID_ARG, "BSND: max_seqlen_q=%d must equal S1=%d (or be 0)",
                    a->max_seqlen_q, a->q_len);
    const int64_t rows = a->layout_q == LI_LAYOUT_TND ? (int64_t)a->q_len
                                                     : (int64_t)a->batch * a->q_len;
    if (rows > INT32_MAX) return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 query rows");
    // the kernels address query-head rows and key-cache rows with 32-bit coordinates
    if (rows * a->num_heads_q > INT32_MAX)
        return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 query-head rows");
    const int64_t key_rows = a->layout_k == LI_LAYOUT_PA_BSND ? (int64_t)a->num_blocks * a->block_size
                             : a->layout_k == LI_LAYOUT_TND  ? (int64_t)a->k_len
                                                             : (int64_t)a->batch * a->k_len;
    if (key_rows > INT32_MAX) return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 key rows");

    li::Problem &P = *p;
    std::memset(&P, 0, sizeof P);
    P.q = static_cast<const uint16_t *>(a->q);
    P.k = static_cast<const uint16_t *>(a->k);
    P.w = static_cast<const uint16_t *>(a->w);
    P.cu_seqlens_q = a->cu_seqlens_q;
    P.cu_seqlens_k = a->cu_seqlens_k;
    P.seqused_q = a->seqused_q;
    P.seqused_k = a->seqused_k;
    P.block_table = a->block_table;
    P.output_idx_offset = a->output_idx_offset;
    P.bt_stride = a->block_table_stride;
    P.batch = a->batch;
    P.q_len = a->q_len;
    P.k_len = a->layout_k == LI_LAYOUT_PA_BSND ? 0 : a->k_len;
    P.max_seqlen_q = a->layout_q == LI_LAYOUT_BSND ? a->q_len : a->max_seqlen_q;
    int32_t mk = a->max_seqlen_k;
    if (a->layout_k == LI_LAYOUT_BSND) {
        if (mk == 0) mk = a->k_len;
        if (mk > a->k_len)
            return fail(LI_ERR_INVALID_ARG, "BSND: max_seqlen_k=%d > S2=%d", mk, a->k_len);
    }
    P.max_seqlen_k = mk;
    P.num_blocks = a->num_blocks;
    P.block_size = a->layout_k == LI_LAYOUT_PA_BSND ? a->block_size : 0;
    P.n_heads = a->num_heads_q;
    P.topk = a->topk;
    P.layout_q = a->layout_q;
    P.layout_k = a->layout_k;
    P.mask_mode = a->mask_mode;
    P.return_value = a->return_value;
    P.rows = (int32_t)rows;
    P.cmp_ratio = a->cmp_ratio > 1 ? a->cmp_ratio : 1;
    P.dtype_qk = a->dtype_qk;
    P.dtype_w = a->dtype_w;
    P.cmp_residual_k = a->cmp_residual_k;

    // Schedule: query blocks of tq rows (all N1 heads of tq rows fill one 256-column MMA tile),
    // split along the keys when there are too few blocks to fill the GPU.
    li::Schedule &S = *s;
    S.tq = li::kMaxHeads * 4 / P.n_heads;           // 256 / N1
    if (S.tq > 128) S.tq = 128;
    if (S.tq < 1) S.tq = 1;
    // a query block never spans batches, so it needs no more rows than the longest batch has
    // (decode: one row, MMA N = N1 instead of 256)
    if (P.max_seqlen_q > 0 && S.tq > P.max_seqlen_q) S.tq = P.max_seqlen_q;
    int64_t qblocks = (int64_t)P.batch * ((P.q_len + S.tq - 1) / S.tq);
    if (P.layout_q == LI_LAYOUT_TND) {
        qblocks = (rows + S.tq - 1) / S.tq + P.batch;
        if (qblocks > rows) qblocks = rows;
    }
    S.kc = 0;
    // too few query blocks to fill the GPU (decode): split the key ranges so that there are
    // about 32 items per SM, small enough for the dynamic scheduler to end all SMs together
    const int64_t target = 32LL * li::device_sm_count();
    if (qblocks < 2LL * li::device_sm_count() && P.max_seqlen_k >= 2048) {
        int64_t kc = ((int64_t)P.max_seqlen_k * (qblocks > 0 ? qblocks : 1) + target - 1) / target;
        kc = (kc + li::kKeyTile - 1) / li::kKeyTile * li::kKeyTile;
        if (kc < 512) kc = 512;
        if (kc < P.max_seqlen_k) S.kc = (int)kc;
    }
    // dense BSND with no seqused and no key split: the work list has a closed form
    S.dense = (P.layout_q == LI_LAYOUT_BSND && P.layout_k == LI_LAYOUT_BSND && !P.seqused_q &&
               !P.seqused_k && S.kc == 0 && P.max_seqlen_k == P.k_len) ? 1 : 0;
    // decode-shaped: one query block per batch, BSND or paged keys with per-batch lengths
    if (!S.dense && P.layout_q == LI_LAYOUT_BSND && !P.seqused_q && P.q_len <= S.tq &&
        (P.layout_k == LI_LAYOUT_BSND || P.layout_k == LI_LAYOUT_PA_BSND))
        S.dense = 2;
    // per-batch residuals of compressed keys are read and checked by the schedule kernel
    if (P.cmp_residual_k) S.dense = 0;
    const int64_t splits = S.kc > 0 ? ((int64_t)P.max_seqlen_k + S.kc - 1) / S.kc : 1;
    const int64_t max_items = qblocks * splits;
    if (max_items > INT32_MAX / 2) return fail(LI_ERR_UNSUPPORTED, "schedule too large");
    S.max_items = (int)(max_items > 0 ? max_items : 0);
    return LI_OK;
}

size_t scores_ld(const li::Problem &p) {
    return (size_t)li::scores_row_floats(p.max_seqlen_k, p.topk);
}

// Partial top-k lists of a row-split selection: [pieces][rows][topk] indices, then values.
size_t piece_bytes(const li::Problem &p, int pieces) {
    if (pieces <= 1) return 0;
    const size_t n = (size_t)pieces * (size_t)p.rows * (size_t)p.topk;
    return (n * sizeof(int32_t) + 255) / 256 * 256 + n * sizeof(float);
}

size_t scores_bytes(const li::Problem &p) {
    return ((size_t)p.rows * scores_ld(p) * sizeof(float) + 255) / 256 * 256;
}

size_t indexer_ws_bytes(const li::Problem &p, const li::Schedule &s) {
    return sizeof(li::WsHeader) + li::meta_bytes(p.batch, s.max_items) + scores_bytes(p) +
           piece_bytes(p, li::select_pieces(p));
}

}  // namespace

namespace li {
void set_last_error(const char *msg) { g_err = msg; }

int device_sm_count() {
    constexpr int kMaxDevices = 128;
    static std::atomic<int> cache[kMaxDevices];      // 0 = not looked up yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return 148;
    }
    const bool slot = dev >= 0 && dev < kMaxDevices;
    if (slot) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    if (slot) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}
}  // namespace li

extern "C" {

li_status li_metadata_workspace_size(const li_args *args, size_t *bytes) {
    li::Problem p;
    li::Schedule s;
    li_status st = validate(args, &p, &s);
    if (st != LI_OK) return st;
    if (!bytes) return fail(LI_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = li::meta_bytes(p.batch, s.max_items);
    return ok();
}

li_status li_metadata(const li_args *args, void *metadata, size_t bytes, void *stream) {
    NvtxRange range("li_metadata");
    li::Problem p;
    li::Schedule s;
    li_status st = validate(args, &p, &s);
    if (st != LI_OK) return st;
    if (!metadata || !aligned(metadata, 256))
        return fail(LI_ERR_WORKSPACE, "metadata must be a 256-byte aligned device buffer");
    const size_t need = li::meta_bytes(p.batch, s.max_items);
    if (bytes < need)
        return fail(LI_ERR_WORKSPACE, "metadata buffer of %zu bytes, %zu needed", bytes, need);
    cudaError_t e = li::launch_metadata(p, s, metadata, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "metadata launch: %s", cudaGetErrorString(e));
    return ok();
}

li_status li_plan(const li_args *args, li_plan_info *info) {
    li::Problem p;
    li::Schedule s;
    li_status st = validate(args, &p, &s);
    if (st != LI_OK) return st;
    if (!info) return fail(LI_ERR_INVALID_ARG, "info is NULL");
    info->tq = s.tq;
    info->kc = s.kc;
    info->max_items = s.max_items;
    info->dense = s.dense;
    const int pieces = li::select_pieces(p);
    info->kernels = p.rows > 0 ? (s.dense ? 2 : 3) + (pieces > 1 ? 1 : 0) : 0;
    info->select_pieces = pieces;
    info->score_tc = !use_simple_kernel() && li::score_tc_eligible(p, s) ? 1 : 0;
    return ok();
}

li_status li_indexer_workspace_size(const li_args *args, size_t *bytes) {
    li::Problem p;
    li::Schedule s;
    li_status st = validate(args, &p, &s);
    if (st != LI_OK) return st;
    if (!bytes) return fail(LI_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = indexer_ws_bytes(p, s);
    return ok();
}

li_status li_indexer(const li_args *args, const void *metadata, void *workspace,
                     size_t workspace_bytes, int32_t *sparse_indices, float *sparse_values,
                     void *stream) {
    NvtxRange range("li_indexer");
    li::Problem p;
    li::Schedule s;
    li_status st = validate(args, &p, &s);
    if (st != LI_OK) return st;
    // Outputs are needed only when there are rows (empty tensors may have NULL data).
    if (p.rows > 0 && (!sparse_indices || !aligned(sparse_indices, 4)))
        return fail(LI_ERR_INVALID_ARG, "sparse_indices must be a 4-byte aligned device buffer");
    if (p.rows > 0 && p.return_value && (!sparse_values || !aligned(sparse_values, 4)))
        return fail(LI_ERR_INVALID_ARG, "return_value=1 requires sparse_values");
    if (metadata && !aligned(metadata, 256))
        return fail(LI_ERR_WORKSPACE, "metadata must be 256-byte aligned");
    if (!workspace || !aligned(workspace, 256))
        return fail(LI_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
    const size_t need = indexer_ws_bytes(p, s);
    if (workspace_bytes < need)
        return fail(LI_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, need);

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    auto *ws = static_cast<li::WsHeader *>(workspace);
    char *base = static_cast<char *>(workspace);
    void *inline_meta = base + sizeof(li::WsHeader);
    float *scores = reinterpret_cast<float *>(base + sizeof(li::WsHeader) +
                                              li::meta_bytes(p.batch, s.max_items));
    const int64_t ld = (int64_t)scores_ld(p);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(li::WsHeader), cs);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "workspace clear: %s", cudaGetErrorString(e));
    if (p.rows == 0) return ok();
    const void *meta = metadata;
    if (!meta && s.dense) {
        stage_mark(0, cs);          // no schedule kernel: the stage is empty
        stage_mark(1, cs);
    }
    if (!meta && !s.dense) {
        NvtxRange r("li_indexer: schedule");
        stage_mark(0, cs);
        e = li::launch_metadata(p, s, inline_meta, cs);
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "metadata launch: %s", cudaGetErrorString(e));
        stage_mark(1, cs);
        meta = inline_meta;
    }
    bool launched = false;
    li::Quant quant;
    quant.q_descale = args->q_descale;
    quant.k_descale = args->k_descale;
    stage_mark(2, cs);
    {
    NvtxRange r("li_indexer: score");
    if (!use_simple_kernel()) {
        e = li::launch_score_tc(p, quant, s, meta, ws, scores, ld, cs, &launched);
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "score launch: %s", cudaGetErrorString(e));
    }
    if (!launched) {
        e = li::launch_score_simple(p, quant, s, meta, ws, scores, ld, cs);
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "score launch: %s", cudaGetErrorString(e));
    }
    }
    stage_mark(3, cs);
    NvtxRange rsel("li_indexer: select");
    stage_mark(4, cs);
    const int pieces = li::select_pieces(p);
    if (pieces > 1) {
        // few very long rows: one CTA per key piece, then the split merge of the pieces' lists
        const size_t n = (size_t)pieces * (size_t)p.rows * (size_t)p.topk;
        char *pbase = reinterpret_cast<char *>(scores) + scores_bytes(p);
        auto *part_idx = reinterpret_cast<int32_t *>(pbase);
        auto *part_val = reinterpret_cast<float *>(pbase + (n * sizeof(int32_t) + 255) / 256 * 256);
        e = li::launch_select_pieces(p, s, meta, ws, scores, ld, pieces, part_idx, part_val, cs);
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "select launch: %s", cudaGetErrorString(e));
        li_merge_args m{};
        const size_t list = (size_t)p.rows * (size_t)p.topk;
        for (int c = 0; c < pieces; ++c) {
            m.idx_in[c] = part_idx + c * list;
            m.val_in[c] = part_val + c * list;
        }
        m.idx_out = sparse_indices;
        m.val_out = p.return_value ? sparse_values : nullptr;
        m.device_status = &ws->status;
        m.rows = p.rows;
        m.n_lists = pieces;
        m.topk_in = m.topk_out = p.topk;
        e = li::launch_merge(m, cs, false);     // the pieces' lists are sorted by construction
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
    } else {
        e = li::launch_select(p, s, meta, ws, scores, ld, sparse_indices,
                              p.return_value ? sparse_values : nullptr, cs);
        if (e != cudaSuccess) return fail(LI_ERR_CUDA, "select launch: %s", cudaGetErrorString(e));
    }
    stage_mark(5, cs);
    return ok();
}

li_status li_check_status(const void *workspace, void *stream, uint32_t *device_bits) {
    if (!workspace) return fail(LI_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    uint32_t bits = 0;
    e = cudaMemcpy(&bits, workspace, sizeof bits, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (device_bits) *device_bits = bits;
    if (bits & LI_DEVERR_TIMEOUT) return fail(LI_ERR_DEVICE_TIMEOUT, "device wait timed out (bits 0x%x)", bits);
    if (bits) return fail(LI_ERR_DEVICE_DATA, "invalid device data (bits 0x%x)", bits);
    return ok();
}

li_status li_set_stage_events(void *const *events, int32_t n_events) {
    if (n_events == 0) {
        g_stage_events_on = false;
        for (auto &ev : g_stage_events) ev = nullptr;
        return ok();
    }
    if (n_events != 6 || !events) return fail(LI_ERR_INVALID_ARG, "li_set_stage_events wants 0 or 6 events");
    for (int i = 0; i < 6; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_events_on = true;
    return ok();
}

li_status li_merge_topk(const li_merge_args *a, void *stream) {
    NvtxRange range("li_merge_topk");
    if (!a) return fail(LI_ERR_INVALID_ARG, "args is NULL");
    if (a->n_lists < 1 || a->n_lists > LI_MERGE_MAX_LISTS)
        return fail(LI_ERR_INVALID_ARG, "n_lists=%d outside [1, %d]", a->n_lists, LI_MERGE_MAX_LISTS);
    if (a->rows < 0) return fail(LI_ERR_INVALID_ARG, "rows=%lld < 0", (long long)a->rows);
    if (a->topk_in < 1 || a->topk_in > 8192 || a->topk_out < 1 || a->topk_out > 8192)
        return fail(LI_ERR_INVALID_ARG, "topk_in=%d / topk_out=%d outside [1, 8192]", a->topk_in,
                    a->topk_out);
    if (a->reserved != 0) return fail(LI_ERR_INVALID_ARG, "reserved field must be 0");
    if (!a->idx_out) return fail(LI_ERR_INVALID_ARG, "idx_out is NULL");
    for (int l = 0; l < a->n_lists; ++l) {
        if (!a->idx_in[l] || !a->val_in[l])
            return fail(LI_ERR_INVALID_ARG, "list %d: idx_in / val_in is NULL", l);
        if (!aligned(a->idx_in[l], 4) || !aligned(a->val_in[l], 4))
            return fail(LI_ERR_INVALID_ARG, "list %d: pointers must be 4-byte aligned", l);
    }
    if (!aligned(a->idx_out, 4) || !aligned(a->val_out, 4) || !aligned(a->device_status, 4))
        return fail(LI_ERR_INVALID_ARG, "outputs and device_status must be 4-byte aligned");
    if (a->rows > INT32_MAX)
        return fail(LI_ERR_UNSUPPORTED, "rows=%lld above 2^31-1", (long long)a->rows);
    if (a->rows == 0) return ok();
    cudaError_t e = li::launch_merge(*a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
    return ok();
}

namespace {
li_status validate_kl(const li_kl_args *a) {
    if (!a) return fail(LI_ERR_INVALID_ARG, "args is NULL");
    if (a->reserved != 0) return fail(LI_ERR_INVALID_ARG, "reserved field must be 0");
    if (a->batch < 0 || a->s1 < 0 || a->s2 < 0)
        return fail(LI_ERR_INVALID_ARG, "batch / s1 / s2 must be >= 0");
    if (a->G < 1 || a->G > 128 || a->H < 1 || a->H > 64 || a->topk < 1 || a->topk > 2048)
        return fail(LI_ERR_INVALID_ARG, "G=%d (1..128), H=%d (1..64), topk=%d (1..2048)", a->G,
                    a->H, a->topk);
    if (a->Dm < 8 || a->Dm > 576 || a->Dm % 8 || a->Dr < 0 || a->Dr > 64 || a->Dr % 8)
        return fail(LI_ERR_INVALID_ARG, "Dm=%d (8..576) and Dr=%d (0..64) must be multiples of 8",
                    a->Dm, a->Dr);
    if ((int64_t)a->G * (a->Dm + a->Dr) > 40960)
        return fail(LI_ERR_INVALID_ARG, "G x (Dm + Dr) = %lld above 40960",
                    (long long)a->G * (a->Dm + a->Dr));
    if ((int64_t)a->batch * a->s1 > INT32_MAX || (int64_t)a->batch * a->s2 > INT32_MAX)
        return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 query or key rows");
    if (!a->q || !a->k || !a->qi || !a->ki || !a->w || !a->sparse_indices || !a->softmax_max ||
        !a->softmax_sum)
        return fail(LI_ERR_INVALID_ARG, "a required input is NULL");
    if ((a->Dr > 0) != (a->q_rope != nullptr) || (a->Dr > 0) != (a->k_rope != nullptr))
        return fail(LI_ERR_INVALID_ARG, "q_rope and k_rope go with Dr > 0, and only with it");

    if (!(a->scale > 0.0f)) return fail(LI_ERR_INVALID_ARG, "scale must be positive");
    const void *ptrs[] = {a->q, a->k, a->q_rope, a->k_rope, a->qi, a->ki, a->w, a->sparse_indices,
                          a->softmax_max, a->softmax_sum};
    for (const void *p : ptrs)
        if (!aligned(p, 4)) return fail(LI_ERR_INVALID_ARG, "inputs must be 4-byte aligned");
    return LI_OK;
}
// Which backward kernel runs: the tensor-core kernel when the shapes fit it, unless
// LI_KL_KERNEL=simple selects the CUDA-core one (a debugging switch).
bool kl_use_tc(const li_kl_args *a, li::KlTcPlan *plan) {
    const char *e = std::getenv("LI_KL_KERNEL");
    if (e && std::strcmp(e, "simple") == 0) return false;
    return li::kl_tc_plan(*a, plan);
}
size_t kl_row_loss_bytes(const li_kl_args *a) {
    return ((size_t)a->batch * a->s1 * sizeof(float) + 255) / 256 * 256;
}
// status word | row losses | tensor-core path: the partial d_ki slices
size_t kl_ws_bytes(const li_kl_args *a) {
    li::KlTcPlan plan;
    size_t n = 256 + kl_row_loss_bytes(a);
    if (kl_use_tc(a, &plan)) n += li::kl_tc_partial_floats(*a, li::kl_tc_chunks(*a)) * sizeof(float);
    return n;
}
}  // namespace

li_status li_kl_grad_workspace_size(const li_kl_args *args, size_t *bytes) {
    li_status st = validate_kl(args);
    if (st != LI_OK) return st;
    if (!bytes) return fail(LI_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = kl_ws_bytes(args);
    return ok();
}

li_status li_kl_grad(const li_kl_args *args, void *workspace, size_t workspace_bytes, float *loss,
                     float *d_qi, float *d_ki, float *d_w, void *stream) {
    NvtxRange range("li_kl_grad");
    li_status st = validate_kl(args);
    if (st != LI_OK) return st;
    if (!workspace || !aligned(workspace, 256))
        return fail(LI_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
    if (workspace_bytes < kl_ws_bytes(args))
        return fail(LI_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes,
                    kl_ws_bytes(args));
    const bool rows = (int64_t)args->batch * args->s1 > 0;
    if (!loss || !aligned(loss, 4) || (rows && (!d_qi || !d_w || !aligned(d_qi, 4) || !aligned(d_w, 4))) ||
        ((int64_t)args->batch * args->s2 > 0 && (!d_ki || !aligned(d_ki, 4))))
        return fail(LI_ERR_INVALID_ARG, "outputs must be 4-byte aligned device buffers");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, 256, cs);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "workspace clear: %s", cudaGetErrorString(e));
    auto *status = static_cast<uint32_t *>(workspace);
    auto *row_loss = reinterpret_cast<float *>(static_cast<char *>(workspace) + 256);
    li::KlTcPlan plan;
    if (kl_use_tc(args, &plan)) {
        auto *d_part = reinterpret_cast<float *>(static_cast<char *>(workspace) + 256 +
                                                 kl_row_loss_bytes(args));
        e = li::launch_kl_tc(*args, plan, row_loss, status, d_part, li::kl_tc_chunks(*args), d_qi,
                             d_ki, d_w, cs);
        if (e == cudaSuccess) e = li::launch_kl_loss(row_loss, (int64_t)args->batch * args->s1, loss, cs);
    } else {
        e = li::launch_kl_grad(*args, row_loss, status, loss, d_qi, d_ki, d_w, cs);
    }
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
    return ok();
}

namespace {
li_status validate_attn(const li_attn_args *a, li::AttnLayout *L) {
    if (!a) return fail(LI_ERR_INVALID_ARG, "args is NULL");
    if (a->reserved != 0) return fail(LI_ERR_INVALID_ARG, "reserved field must be 0");
    if (a->batch < 0 || a->s1 < 0 || a->s2 < 0)
        return fail(LI_ERR_INVALID_ARG, "batch / s1 / s2 must be >= 0");
    if (a->G < 1 || a->G > 32) return fail(LI_ERR_INVALID_ARG, "G=%d outside [1, 32]", a->G);
    if (a->Dm < 128 || a->Dm > 512 || a->Dm % 128)
        return fail(LI_ERR_INVALID_ARG, "Dm=%d must be 128, 256, 384 or 512", a->Dm);
    if (a->Dr != 0 && a->Dr != 64) return fail(LI_ERR_INVALID_ARG, "Dr=%d must be 0 or 64", a->Dr);
    if (a->topk < 1 || a->topk > li::kMaxTopk)
        return fail(LI_ERR_INVALID_ARG, "topk=%d outside [1, 8192]", a->topk);
    if (!(a->scale > 0.0f) || !(a->scale < 3.0e38f))
        return fail(LI_ERR_INVALID_ARG, "scale must be a positive finite number");
    const int64_t rows = (int64_t)a->batch * a->s1;
    if (rows > 0 && a->s2 < 1) return fail(LI_ERR_INVALID_ARG, "S2=0 with query rows");
    if (rows * a->G > INT32_MAX || (int64_t)a->batch * a->s2 > INT32_MAX)
        return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 query-head rows or key rows");
    if (rows > 0 && (!a->q || !a->k || !a->sparse_indices))
        return fail(LI_ERR_INVALID_ARG, "q, k and sparse_indices are required");
    if ((a->Dr > 0) != (a->q_rope != nullptr) || (a->Dr > 0) != (a->k_rope != nullptr))
        return fail(LI_ERR_INVALID_ARG, "q_rope and k_rope go with Dr > 0, and only with it");
    if (a->layout_k == LI_LAYOUT_PA_BSND) {
        if (a->block_size < 1 || a->block_size > 1024)
            return fail(LI_ERR_INVALID_ARG, "block_size=%d outside [1, 1024]", a->block_size);
        if (a->num_blocks < 1) return fail(LI_ERR_INVALID_ARG, "num_blocks must be >= 1");
        if ((int64_t)a->num_blocks * a->block_size > INT32_MAX)
            return fail(LI_ERR_UNSUPPORTED, "more than 2^31-1 cache rows");
        const int64_t need = ((int64_t)a->s2 + a->block_size - 1) / a->block_size;
        if (a->block_table_stride < need)
            return fail(LI_ERR_INVALID_ARG, "block_table_stride=%d below ceil(S2 / block_size)=%lld",
                        a->block_table_stride, (long long)need);
        if (rows > 0 && (!a->block_table || !aligned(a->block_table, 4)))
            return fail(LI_ERR_INVALID_ARG, "PA_BSND needs a 4-byte aligned block_table");
    } else if (a->layout_k == LI_LAYOUT_BSND) {
        if (a->block_table || a->block_table_stride || a->num_blocks || a->block_size)
            return fail(LI_ERR_INVALID_ARG, "block_table fields are for PA_BSND only");
    } else {
        return fail(LI_ERR_INVALID_ARG, "layout_k=%d must be BSND or PA_BSND", a->layout_k);
    }
    if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->q_rope, 16) ||
        !aligned(a->k_rope, 16) || !aligned(a->sparse_indices, 4))
        return fail(LI_ERR_INVALID_ARG, "q, k and the rope parts must be 16-byte aligned");
    if (!li::attn_layout(*a, L))
        return fail(LI_ERR_UNSUPPORTED, "G=%d with Dm=%d does not fit the kernel's shared memory",
                    a->G, a->Dm);
    return LI_OK;
}
}  // namespace

li_status li_sparse_attention_workspace_size(const li_attn_args *args, size_t *bytes) {
    li::AttnLayout L;
    li_status st = validate_attn(args, &L);
    if (st != LI_OK) return st;
    if (!bytes) return fail(LI_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = 256;
    return ok();
}

li_status li_sparse_attention(const li_attn_args *args, void *workspace, size_t workspace_bytes,
                              float *out, float *softmax_max, float *softmax_sum, void *stream) {
    NvtxRange range("li_sparse_attention");
    li::AttnLayout L;
    li_status st = validate_attn(args, &L);
    if (st != LI_OK) return st;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < 256)
        return fail(LI_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer of >= 256 bytes");
    const bool rows = (int64_t)args->batch * args->s1 > 0;
    if (rows && (!out || !softmax_max || !softmax_sum || !aligned(out, 4) ||
                 !aligned(softmax_max, 4) || !aligned(softmax_sum, 4)))
        return fail(LI_ERR_INVALID_ARG, "out, softmax_max and softmax_sum must be 4-byte aligned");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, 256, cs);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "workspace clear: %s", cudaGetErrorString(e));
    if (!rows) return ok();
    auto *hdr = static_cast<uint32_t *>(workspace);
    e = li::launch_sparse_attention(*args, hdr, reinterpret_cast<int32_t *>(hdr + 1), out,
                                    softmax_max, softmax_sum, cs);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
    return ok();
}

const char *li_last_error_string(void) { return g_err.c_str(); }

int32_t li_abi_version(void) { return LI_ABI_VERSION; }

}  // extern "C"
