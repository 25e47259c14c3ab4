// Internal definitions shared by the library's kernels and host code (not part of the ABI).
//
// Device memory layout of the two caller-owned buffers:
//
//   metadata (li_metadata):   MetaHeader | BatchInfo[B] | WorkItem[max_items]
//   workspace (li_indexer):   WsHeader (256 B) | inline metadata | fp32 scores [rows][ld]
//
// The fp32 score rows hold I[t, j] for every key j of row t's window; the selection kernel reads
// them back. Rows are indexed by the global query row (B*S1 rows for BSND, T1 rows for TND).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "li.h"

namespace li {

constexpr int kHeadDim = 128;
constexpr int kMaxHeads = 64;
constexpr int kMaxTopk = 8192;
constexpr int kKeyTile = 128;          // keys per tile of the score kernels
constexpr uint32_t kMetaMagic = 0x4c494d31u;   // "LIM1"

// Device status bit used when metadata does not match the call it is used with.
constexpr uint32_t kDevErrMetadata = 0x10u;

struct MetaHeader {
    uint32_t magic;
    uint32_t status;       // LI_DEVERR_* bits found while building the schedule
    int32_t n_items;       // items written
    int32_t max_items;     // capacity
    int32_t batch;
    int32_t tq;            // query rows per work item
    int32_t kc;            // keys per work item (key-range split), 0 = whole window
    uint32_t signature;    // hash of the scalar arguments the schedule was built for
    int32_t pad[8];
};
static_assert(sizeof(MetaHeader) == 64, "MetaHeader size");

struct BatchInfo {
    int32_t L1;            // query rows allocated to the batch
    int32_t L1u;           // query rows in use (seqused_q), <= L1
    int32_t L2;            // keys of the batch
    int32_t q_row0;        // global query row of the batch's row 0
    int32_t k_row0;        // BSND: b*S2, TND: cu_seqlens_k[b], PA: 0
    int32_t pad[3];        // schedule kernel: [0] query blocks, [1] first block; [2] residual
                           // tokens of compressed keys (cmp_residual_k[b], else 0)
};
static_assert(sizeof(BatchInfo) == 32, "BatchInfo size");

// One unit of score work. It carries its batch's lengths and row bases too, so the kernels that
// take items need no second dependent load of the batch record.
struct alignas(16) WorkItem {
    int32_t b;             // batch
    int32_t q0;            // first query row (position inside the batch)
    int32_t nq;            // query rows (<= tq)
    int32_t j0;            // first key of the item's range
    int32_t j1;            // one past the last key any of its rows needs
    int32_t cost;          // key tiles, for ordering
    int32_t row0;          // global query row of q0 (the batch's q_row0 + q0)
    int32_t L1u;           // the batch's query rows in use
    int32_t L2;            // the batch's keys; compressed keys: j1 + L1u, so that the score
                           // kernel's plain right-down window reaches j1 for every row of the item
                           // (a superset of each row's window; the selection applies the exact one)
    int32_t k_row0;        // the batch's first key row
    int32_t pad[6];
};
static_assert(sizeof(WorkItem) == 64, "WorkItem size");

struct WsHeader {
    uint32_t status;       // LI_DEVERR_* bits of the last li_indexer on this workspace
    int32_t sched_next;    // dynamic scheduler ticket counter
    int32_t exact_rows;    // rows the selection finished on its exact (tie-heavy) fallback path
    int32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "WsHeader size");

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline size_t meta_bytes(int batch, int max_items) {
    return align_up(sizeof(MetaHeader) + sizeof(BatchInfo) * (size_t)batch +
                    sizeof(WorkItem) * (size_t)max_items, 256);
}

__host__ __device__ inline const BatchInfo *meta_batches(const void *meta) {
    return reinterpret_cast<const BatchInfo *>(static_cast<const char *>(meta) + sizeof(MetaHeader));
}
__host__ __device__ inline const WorkItem *meta_items(const void *meta, int batch) {
    return reinterpret_cast<const WorkItem *>(static_cast<const char *>(meta) + sizeof(MetaHeader) +
                                              sizeof(BatchInfo) * (size_t)batch);
}

// Window of row i of a batch: keys [0, hi). mask 0: hi = L2. mask 3 (right-down causal):
// hi = min(L2, i + L2 - L1u + 1), clipped at 0. Compressed keys (r > 1 original tokens each, res
// tokens past the last whole key) under mask 3: the keys whose last original token is visible,
// hi = floor((i + L2*r + res - L1u + 1) / r), clipped to [0, L2]. Rows past L1u have no window.
__host__ __device__ inline int32_t window_hi(int mask_mode, int32_t i, int32_t L1u, int32_t L2,
                                            int32_t r = 1, int32_t res = 0) {
    if (i >= L1u || L2 <= 0) return 0;
    if (mask_mode != 3) return L2;
    int64_t lim = r > 1 ? ((int64_t)i + (int64_t)L2 * r + res - L1u + 1) / r
                        : (int64_t)i + L2 - L1u + 1;     // negative numerators clip to 0 below
    if (lim > L2) lim = L2;
    return lim < 0 ? 0 : (int32_t)lim;
}

// Scalars every kernel needs, copied by value into kernel parameters.
struct Problem {
    const uint16_t *q, *k, *w;            // 16-bit patterns (dtype_qk / dtype_w); fp32 w is read
                                           // through a float pointer
    const int32_t *cu_seqlens_q, *cu_seqlens_k, *seqused_q, *seqused_k;
    const int32_t *block_table;
    const int32_t *output_idx_offset;
    int64_t bt_stride;
    int32_t batch, q_len, k_len, max_seqlen_q, max_seqlen_k;
    int32_t num_blocks, block_size;
    int32_t n_heads, topk;
    int32_t layout_q, layout_k, mask_mode;
    int32_t return_value;
    int32_t rows;                          // B*S1 or T1
    const int32_t *cmp_residual_k;         // compressed keys: [B] residual tokens, or null
    int32_t cmp_ratio;                     // original tokens per key (1: not compressed)
    int16_t dtype_qk, dtype_w;             // li_dtype of q/k (bf16, fp16) and w (also fp32)
};
// The tensor-core score kernel takes Problem inside its parameter block; growing it by 8 bytes
// (two int32 dtype fields) slowed that kernel by 6% on a 4096-token causal prefill, so new
// fields go into existing padding.
static_assert(sizeof(Problem) == 152, "Problem layout changed: re-measure the score kernel");

// fp32 elements per score row of the workspace (16-byte aligned rows).
__host__ __device__ inline int64_t scores_row_floats(int32_t max_seqlen_k, int32_t topk) {
    (void)topk;
    const int64_t ld = max_seqlen_k > 0 ? max_seqlen_k : 1;
    return (ld + 3) / 4 * 4;
}

// Signature of the scalar arguments a schedule depends on.
__host__ __device__ inline uint32_t problem_signature(const Problem &p, int tq, int kc) {
    uint32_t h = 2166136261u;
    auto mix = [&](uint32_t v) { h = (h ^ v) * 16777619u; };
    mix((uint32_t)p.batch); mix((uint32_t)p.q_len); mix((uint32_t)p.k_len);
    mix((uint32_t)p.max_seqlen_q); mix((uint32_t)p.max_seqlen_k); mix((uint32_t)p.n_heads);
    mix((uint32_t)p.layout_q); mix((uint32_t)p.layout_k); mix((uint32_t)p.mask_mode);
    mix((uint32_t)p.block_size); mix((uint32_t)tq); mix((uint32_t)kc);
    mix((uint32_t)p.cmp_ratio); mix(p.cmp_residual_k ? 1u : 0u);
    return h;
}

// Schedule parameters chosen on the host for a problem (shared by li_metadata and li_indexer).
struct Schedule {
    int tq;          // query rows per item
    int kc;          // key-range split (0 = none)
    int max_items;   // capacity of the item list
    int dense;       // work lists in closed form (no schedule kernel): 1 = dense BSND without
                     // seqused and without key split; 2 = BSND queries, no seqused_q, all of a
                     // batch's rows in one query block (decode), BSND or paged keys with
                     // per-batch lengths; 0 = the schedule kernel builds the list
};

// Keys of batch b from the device-resident lengths, clamped the way the schedule kernel clamps
// them (BSND or paged keys); sets LI_DEVERR_LENGTHS in *err when the stored length is out of
// range.
__device__ inline int32_t batch_keys(const Problem &p, int32_t b, uint32_t *err) {
    int64_t L2;
    if (p.layout_k == LI_LAYOUT_PA_BSND) {
        const int64_t u = p.seqused_k[b];
        const int64_t cap = p.bt_stride * (int64_t)p.block_size;
        if (u < 0 || u > cap) *err |= LI_DEVERR_LENGTHS;
        L2 = u < 0 ? 0 : (u > cap ? cap : u);
    } else {
        L2 = p.k_len;
        if (p.seqused_k) {
            const int64_t u = p.seqused_k[b];
            if (u < 0 || u > L2) *err |= LI_DEVERR_LENGTHS;
            L2 = u < 0 ? 0 : (u < L2 ? u : L2);
        }
    }
    if (L2 > p.max_seqlen_k) {
        *err |= LI_DEVERR_LENGTHS;
        L2 = p.max_seqlen_k;
    }
    return (int32_t)L2;
}

// Work list and per-batch lengths as the kernels see them: either the schedule built by
// li_metadata (a MetaHeader in device memory) or closed forms (Schedule::dense 1 or 2).
struct SchedView {
    const void *meta;      // nullptr: closed forms
    int32_t tq;
    int32_t n_items;
    int32_t nqb;           // dense: query blocks per batch
    int32_t mode;          // closed form: 1 dense BSND, 2 one query block per batch
    int32_t kc;            // mode 2: keys per item (0: the whole window)
    int32_t splits;        // mode 2: item slots per batch (ceil(max_seqlen_k / kc), or 1)

    __device__ BatchInfo batch(const Problem &p, int32_t b) const {
        if (meta) return meta_batches(meta)[b];
        BatchInfo bi;
        uint32_t err = 0;
        bi.L1 = bi.L1u = p.q_len;
        bi.L2 = mode == 2 ? batch_keys(p, b, &err) : p.k_len;
        bi.q_row0 = b * p.q_len;
        bi.k_row0 = p.layout_k == LI_LAYOUT_PA_BSND ? 0 : b * p.k_len;
        bi.pad[0] = bi.pad[1] = bi.pad[2] = 0;
        return bi;
    }
    // Item t of the list (0 <= t < n_items); an item whose window is empty has j1 <= j0 and is
    // skipped by the caller. Mode 1: query blocks last-to-first (for the causal mask that is
    // longest first), batches interleaved. Mode 2: key piece s = t / B of batch b = t % B, so
    // every batch's first pieces come first; pieces past a batch's keys are empty.
    __device__ WorkItem item(const Problem &p, int32_t t) const {
        const int32_t hb = meta ? reinterpret_cast<const MetaHeader *>(meta)->batch : 0;
        if (meta) return meta_items(meta, hb)[t];
        WorkItem it;
        if (mode == 2) {
            const int32_t sp = t / p.batch;
            uint32_t err = 0;
            it.b = t - sp * p.batch;
            it.q0 = 0;
            it.nq = p.q_len;
            it.L1u = p.q_len;
            it.L2 = batch_keys(p, it.b, &err);
            const int32_t jend = window_hi(p.mask_mode, p.q_len - 1, p.q_len, it.L2);
            const int32_t span = kc > 0 ? kc : jend;
            const int64_t j0 = (int64_t)sp * span;
            it.j0 = j0 < jend ? (int32_t)j0 : jend;
            it.j1 = j0 < jend ? min(jend, it.j0 + span) : jend;
            it.cost = 0;
            it.row0 = it.b * p.q_len;
            it.k_row0 = p.layout_k == LI_LAYOUT_PA_BSND ? 0 : it.b * p.k_len;
            for (int i = 0; i < 6; ++i) it.pad[i] = 0;
            return it;
        }
        const int32_t qb = nqb - 1 - t / p.batch;
        it.b = t % p.batch;
        it.q0 = qb * tq;
        it.nq = min(tq, p.q_len - it.q0);
        it.j0 = 0;
        it.j1 = window_hi(p.mask_mode, it.q0 + it.nq - 1, p.q_len, p.k_len);
        it.cost = 0;
        it.row0 = it.b * p.q_len + it.q0;
        it.L1u = p.q_len;
        it.L2 = p.k_len;
        it.k_row0 = it.b * p.k_len;
        for (int i = 0; i < 6; ++i) it.pad[i] = 0;
        return it;
    }
};

// Closed form with per-batch key lengths (mode 2) has no schedule kernel to check the stored
// lengths: threads tid0, tid0 + nthr, ... of one block check them and set the status bits.
__device__ inline void check_batch_keys(const Problem &p, const SchedView &v, uint32_t *status,
                                        int tid0, int nthr) {
    if (v.meta || v.mode != 2) return;
    uint32_t err = 0;
    for (int32_t b = tid0; b < p.batch; b += nthr) (void)batch_keys(p, b, &err);
    if (err) atomicOr(status, err);
}

// Builds the view for a kernel launch. meta == nullptr selects the dense closed forms.
inline SchedView make_view(const Problem &p, const Schedule &s, const void *meta) {
    SchedView v;
    v.meta = meta;
    v.tq = s.tq;
    v.nqb = p.q_len > 0 ? (p.q_len + s.tq - 1) / s.tq : 0;
    v.mode = s.dense;
    v.kc = s.kc;
    v.splits = s.kc > 0 ? (p.max_seqlen_k + s.kc - 1) / s.kc : 1;
    // with metadata the count is read on the device
    v.n_items = meta ? 0 : (s.dense == 2 ? p.batch * v.splits : p.batch * v.nqb);
    return v;
}

// Device-side: batch of a global query row (TND: binary search in cu_seqlens_q).
__device__ inline int32_t row_batch(const Problem &p, int32_t r, int32_t *pos) {
    if (p.layout_q != LI_LAYOUT_TND) {
        int32_t b = r / p.q_len;
        *pos = r - b * p.q_len;
        return b;
    }
    // largest b with cu[b] <= r and r < cu[b+1]; rows past cu[B] have no batch
    int32_t lo = 0, hi = p.batch;   // search in cu[0..B]
    if (p.batch <= 0 || r < p.cu_seqlens_q[0] || r >= p.cu_seqlens_q[p.batch]) { *pos = 0; return -1; }
    while (hi - lo > 1) {
        int32_t mid = (lo + hi) >> 1;
        if (p.cu_seqlens_q[mid] <= r) lo = mid; else hi = mid;
    }
    *pos = r - p.cu_seqlens_q[lo];
    return lo;
}

// Pointer to logical key j of batch b (paged: through the block table). Returns nullptr when
// the block table entry is out of range.
__device__ inline const uint16_t *key_ptr(const Problem &p, const BatchInfo &bi, int32_t b, int32_t j) {
    if (p.layout_k == LI_LAYOUT_PA_BSND) {
        int32_t blk = p.block_table[(int64_t)b * p.bt_stride + j / p.block_size];
        if (blk < 0 || blk >= p.num_blocks) return nullptr;
        return p.k + ((int64_t)blk * p.block_size + j % p.block_size) * kHeadDim;
    }
    return p.k + ((int64_t)bi.k_row0 + j) * kHeadDim;
}

// Row of the key cache holding key j of batch b (-1: block-table entry out of range).
__device__ inline int64_t key_row(const Problem &p, const BatchInfo &bi, int32_t b, int32_t j) {
    if (p.layout_k == LI_LAYOUT_PA_BSND) {
        int32_t blk = p.block_table[(int64_t)b * p.bt_stride + j / p.block_size];
        if (blk < 0 || blk >= p.num_blocks) return -1;
        return (int64_t)blk * p.block_size + j % p.block_size;
    }
    return (int64_t)bi.k_row0 + j;
}

// A scale of fp8 q/k is usable when it is a positive finite number.
__device__ inline bool good_scale(float x) { return x > 0.0f && x < __int_as_float(0x7f800000); }

__device__ inline float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ inline float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// A 16-bit q/k/w element to fp32: bf16 is the upper half of an fp32, fp16 is IEEE binary16.
__device__ inline float half16_to_f32(uint32_t bits16, bool fp16) {
    return fp16 ? __half2float(__ushort_as_half((unsigned short)bits16))
                : __uint_as_float(bits16 << 16);
}
// Weight idx of w in its type (kW = li_dtype), as fp32.
template <int kW>
__device__ __forceinline__ float weight_f32(const Problem &p, int64_t idx) {
    if constexpr (kW == LI_DTYPE_FP32) return reinterpret_cast<const float *>(p.w)[idx];
    else if constexpr (kW == LI_DTYPE_FP16) return __half2float(__ushort_as_half(p.w[idx]));
    else return __uint_as_float((uint32_t)p.w[idx] << 16);
}
__device__ inline float weight_f32(const Problem &p, int64_t idx) {
    return p.dtype_w == LI_DTYPE_FP32 ? weight_f32<LI_DTYPE_FP32>(p, idx)
         : p.dtype_w == LI_DTYPE_FP16 ? weight_f32<LI_DTYPE_FP16>(p, idx)
                                      : weight_f32<LI_DTYPE_BF16>(p, idx);
}

__device__ inline void set_status(uint32_t *status, uint32_t bits) {
    if (bits) atomicOr(status, bits);
}

// Bounds-checked build (-DLI_DEBUG): the kernels pass each computed shared- or global-memory
// index through in_bounds() before the access. A failing check sets LI_DEVERR_BOUNDS and the
// caller skips the access (no trap: the context stays usable). The release build compiles every
// check to `true`, so its code is unchanged.
#ifdef LI_DEBUG
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t *status) {
    if constexpr (kDebugBounds) {
        if (!ok) {
            if (status) atomicOr(status, LI_DEVERR_BOUNDS);
            return false;
        }
    }
    return true;
}
// Index i of a buffer of n elements.
__device__ __forceinline__ bool idx_ok(int64_t i, int64_t n, uint32_t *status) {
    return in_bounds(i >= 0 && i < n, status);
}

// Sets the message li_last_error_string() returns on this host thread.
void set_last_error(const char *msg);

// Streaming multiprocessors of the current device, looked up once per device (148, the B200's
// count, when the query fails).
int device_sm_count();

// fp8 q/k scales (li_args q_descale / k_descale), null for 16-bit q/k. Kept out of Problem so
// that the kernels' parameter blocks keep their layout.
struct Quant {
    const float *q_descale = nullptr;     // [rows * N1], laid out like w
    const float *k_descale = nullptr;     // one per key row
};

// ---- launchers implemented in the .cu files --------------------------------------------------
cudaError_t launch_metadata(const Problem &p, const Schedule &s, void *meta, cudaStream_t st);
cudaError_t launch_score_simple(const Problem &p, const Quant &qd, const Schedule &s,
                                const void *meta, WsHeader *ws, float *scores, int64_t ld,
                                cudaStream_t st);
// Tensor-core score kernel: whether the problem fits it, and its launcher (*launched = false
// when it does not, leaving the step to launch_score_simple).
bool score_tc_eligible(const Problem &p, const Schedule &s);
cudaError_t launch_score_tc(const Problem &p, const Quant &qd, const Schedule &s, const void *meta,
                            WsHeader *ws, float *scores, int64_t ld, cudaStream_t st,
                            bool *launched);
// (meta == nullptr in the score and select launchers selects the dense closed-form schedule)
cudaError_t launch_select(const Problem &p, const Schedule &s, const void *meta, WsHeader *ws,
                          const float *scores, int64_t ld, int32_t *out_idx, float *out_val,
                          cudaStream_t st);

}  // namespace li
