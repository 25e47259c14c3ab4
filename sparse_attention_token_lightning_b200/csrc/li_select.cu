// Per-row top-k selection from the fp32 score rows (second pass of the two-pass design).
//
// For query row t with window [0, n): keep the m = min(topk, n) keys with the largest I[t, j],
// ordered by I descending and, on equal scores, by lower key index first; write their indices
// (+ output_idx_offset[b]) and scores, then pad with -1 / -inf up to topk (lightning_indexer and
// aclnnLightningIndexerV2, constraints on the invalid part; torch_npu.npu_sparse_lightning_
// indexer_grad_kl_loss, sparse_indices are sorted). Rows past seqused_q, rows of no batch and
// rows with an empty causal window are all padding. -0 and +0 are the same score.
//
// One CTA per row. Main path (value buckets):
//   1. min and max score of the row; if they are equal every key ties and the answer is keys
//      0..m-1 in order.
//   2. A monotone linear map of the score to ~n buckets (bucket 0 = highest scores), an
//      atomic histogram, and a warp-striped exclusive scan give each bucket its output range;
//      the bucket holding output position m-1 is the last one needed.
//   3. The keys of the needed buckets are scattered to their ranges as 64-bit composites
//      (score key << 32 | ~index), in any order; each key then counts the larger composites of
//      its bucket (about one or two keys) and lands in an output stage at its exact slot,
//      which fixes the order including ties; the stage is written out in slot order.
// Exact fallback, for rows whose needed buckets hold more than kBinCap keys (heavy exact ties)
// or whose score range overflows: radix select of the m-th key (most significant byte first),
// gather in index order, stable LSD radix sort.
// Rows of up to kRegKeys*kThreads keys are held in registers (one read of the row); longer rows
// take two streaming passes: a 12-bit key-digit histogram that bounds the selection, then a
// gather of the candidates into shared memory, which the bucket sort orders.
// Few very long rows (rows x 4 <= SMs, at least kPieceMinKeys keys) are cut into key pieces, one
// CTA each (select_piece_kernel), whose sorted lists the split merge joins into the row's output.
#include "li_internal.cuh"
#include "li_select.cuh"

namespace li {
namespace {

struct Params {
    Problem p;
    SchedView view;
    WsHeader *ws;
    const float *scores;
    int64_t ld;
    int32_t *out_idx;
    float *out_val;
    uint32_t signature;
    int32_t cand_cap;       // long-row candidates that fit in shared memory
};

struct PieceParams {
    int32_t *idx;           // [pieces][rows][topk] partial lists
    float *val;
    int32_t pieces;
    int32_t piece_len;
};

// Short rows: 256 threads per row, 16 keys per thread held in registers.
namespace sel256 {
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
#include "li_select_impl.cuh"
}  // namespace sel256

// Problems with rows longer than 4096 keys: 512 threads per row.
namespace sel512 {
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
#include "li_select_impl.cuh"
}  // namespace sel512

// Few long rows (fewer than two per SM, e.g. decode): 1024 threads per row shorten each row.
namespace sel1024 {
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
#include "li_select_impl.cuh"
}  // namespace sel1024

}  // namespace

// Launch on a problem's rows: the 256-thread kernel when no row can exceed 4096 keys, else the
// 512-thread kernel with the long-row path.
template <int NT, bool kLong, class Smem, class Kern>
static cudaError_t launch_one(const Problem &p, const Schedule &s, const void *meta, WsHeader *ws,
                              const float *scores, int64_t ld, int32_t *out_idx, float *out_val,
                              size_t smem, int32_t cand_cap, Kern kern, cudaStream_t st) {
    if (smem + sizeof(Smem) > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    Params sp{p, make_view(p, s, meta), ws, scores, ld, out_idx, out_val,
              problem_signature(p, s.tq, s.kc), cand_cap};
    kern<<<p.rows, NT, smem, st>>>(sp);
    return cudaGetLastError();
}

cudaError_t launch_select(const Problem &p, const Schedule &s, const void *meta, WsHeader *ws,
                          const float *scores, int64_t ld, int32_t *out_idx, float *out_val,
                          cudaStream_t st) {
    if (p.rows <= 0) return cudaSuccess;
    int32_t cand_cap = 0;
    if (p.max_seqlen_k <= 4096) {
        const size_t smem = sel256::select_work_bytes(p.topk, false, &cand_cap);
        return launch_one<256, false, sel256::Smem>(p, s, meta, ws, scores, ld, out_idx, out_val,
                                                    smem, cand_cap, sel256::select_kernel<false>, st);
    }
    const int sms = device_sm_count();
    if (p.rows < 2 * sms) {
        const size_t smem = sel1024::select_work_bytes(p.topk, true, &cand_cap);
        return launch_one<1024, true, sel1024::Smem>(p, s, meta, ws, scores, ld, out_idx, out_val,
                                                     smem, cand_cap, sel1024::select_kernel<true>,
                                                     st);
    }
    const size_t smem = sel512::select_work_bytes(p.topk, true, &cand_cap);
    return launch_one<512, true, sel512::Smem>(p, s, meta, ws, scores, ld, out_idx, out_val, smem,
                                               cand_cap, sel512::select_kernel<true>, st);
}

int select_pieces(const Problem &p) {
    const int sms = device_sm_count();
    // only rows long enough that one CTA streaming the whole row is the bottleneck, and few
    // enough rows that the GPU would otherwise sit mostly idle
    if (p.rows <= 0 || p.max_seqlen_k < kPieceMinKeys || p.rows * 4 > sms) return 1;
    int pieces = sms / (int)p.rows;
    const int by_len = (p.max_seqlen_k + kPieceMinKeys / 2 - 1) / (kPieceMinKeys / 2);
    if (pieces > by_len) pieces = by_len;
    if (pieces > kMaxPieces) pieces = kMaxPieces;
    while (pieces > 1 && !merge_fits_smem(pieces, p.topk, p.topk)) --pieces;
    return pieces < 2 ? 1 : pieces;
}

int32_t piece_len(const Problem &p, int pieces) {
    const int64_t len = ((int64_t)p.max_seqlen_k + pieces - 1) / pieces;
    return (int32_t)((len + 127) / 128 * 128);
}

cudaError_t launch_select_pieces(const Problem &p, const Schedule &s, const void *meta,
                                 WsHeader *ws, const float *scores, int64_t ld, int pieces,
                                 int32_t *part_idx, float *part_val, cudaStream_t st) {
    int32_t cand_cap = 0;
    const size_t smem = sel1024::select_work_bytes(p.topk, true, &cand_cap);
    if (smem + sizeof(sel1024::Smem) > 227 * 1024) return cudaErrorInvalidConfiguration;
    auto kern = sel1024::select_piece_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    Params sp{p, make_view(p, s, meta), ws, scores, ld, nullptr, nullptr,
              problem_signature(p, s.tq, s.kc), cand_cap};
    PieceParams pp{part_idx, part_val, pieces, piece_len(p, pieces)};
    kern<<<(unsigned)(p.rows * pieces), 1024, smem, st>>>(sp, pp);
    return cudaGetLastError();
}

}  // namespace li
