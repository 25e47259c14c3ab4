// Schedule builder (li_metadata). Replaces the pages' per-AI-core task list (lightning_indexer,
// "Function": lightning_indexer_metadata produces per-core tasks of batch, head and Q/K block
// ranges) with a list of work items for persistent CTAs:
//
//   item = (batch b, query rows [q0, q0+nq), key range [j0, j1))
//
// ordered by cost (key tiles) descending, so CTAs that pull items in order finish together.
// One CTA builds it: per-batch lengths first (validating the device-resident cu_seqlens, seqused
// and offsets), then a counting sort of the items by cost: a histogram pass, a descending scan of
// the histogram, and a placement pass. The order of equal-cost items may vary between runs; every
// item writes its own rows, so results do not depend on it.
#include "li_internal.cuh"

namespace li {
namespace {

constexpr int kMetaThreads = 1024;
constexpr int kCostBins = 1024;

struct MetaParams {
    Problem p;
    Schedule s;
    void *meta;
};

__device__ inline int item_cost(int32_t j0, int32_t j1) {
    int c = (j1 - j0 + kKeyTile - 1) / kKeyTile;
    return c < kCostBins ? c : kCostBins - 1;
}

// Block-wide inclusive scan of one value per thread (kMetaThreads threads): warp scans, then
// one warp scans the 32 warp totals.
__device__ inline int32_t block_inclusive_scan(int32_t x, int32_t *warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t ws = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += t;
        }
        warp_sums[lane] = ws;                       // inclusive prefix of the warp totals
    }
    __syncthreads();
    const int32_t before = warp > 0 ? warp_sums[warp - 1] : 0;
    __syncthreads();
    return before + incl;
}

// Writes one item as four 16-byte stores (items land at scattered slots; a warp's scalar
// stores to scattered slots cost one memory transaction per lane each).
__device__ inline void store_item(WorkItem *dst, const WorkItem &it) {
    const int4 *src = reinterpret_cast<const int4 *>(&it);
    int4 *d = reinterpret_cast<int4 *>(dst);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(WorkItem) / sizeof(int4)); ++i) d[i] = src[i];
}

constexpr int kSmemBatches = 1024;     // batches whose lengths and block prefix stay in smem

// Batch of global query block g: the last batch whose first block is <= g (qb0 holds each
// batch's first block, in shared memory when the batch count allows, else in global memory).
__device__ inline int32_t batch_of_block(const int32_t *qb0, int32_t batch, int32_t g) {
    int32_t lo = 0, hi = batch - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (qb0[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kMetaThreads) metadata_kernel(MetaParams mp) {
    const Problem &p = mp.p;
    const Schedule &s = mp.s;
    MetaHeader *hdr = reinterpret_cast<MetaHeader *>(mp.meta);
    BatchInfo *binfo = reinterpret_cast<BatchInfo *>(static_cast<char *>(mp.meta) + sizeof(MetaHeader));
    WorkItem *items = reinterpret_cast<WorkItem *>(binfo + p.batch);

    __shared__ int32_t hist[kCostBins];
    __shared__ uint32_t s_status;
    __shared__ int32_t s_total;
    // per-batch query rows in use, keys and first query block (B <= kSmemBatches)
    __shared__ int32_t s_L1u[kSmemBatches], s_L2[kSmemBatches], s_qb0[kSmemBatches];
    __shared__ int32_t s_qr0[kSmemBatches], s_kr0[kSmemBatches];   // first query / key rows
    __shared__ int32_t s_res[kSmemBatches];          // residual tokens of compressed keys
    const bool in_smem = p.batch <= kSmemBatches;
    const int tid = threadIdx.x;
    for (int i = tid; i < kCostBins; i += kMetaThreads) hist[i] = 0;
    if (tid == 0) { s_status = 0; s_total = 0; }
    __syncthreads();

    // ---- pass 0: per-batch lengths ------------------------------------------------------------
    for (int32_t b = tid; b < p.batch; b += kMetaThreads) {
        uint32_t err = 0;
        BatchInfo bi;
        int64_t L1, q0, L2, k0;
        if (p.layout_q == LI_LAYOUT_TND) {
            const int64_t c0 = p.cu_seqlens_q[b], c1 = p.cu_seqlens_q[b + 1];
            if (c0 < 0 || c1 < c0 || c1 > p.q_len) { err |= LI_DEVERR_LENGTHS; }
            L1 = (c1 >= c0 && c0 >= 0 && c1 <= p.q_len) ? c1 - c0 : 0;
            q0 = c0 < 0 ? 0 : c0;
        } else {
            L1 = p.q_len;
            q0 = (int64_t)b * p.q_len;
        }
        int64_t L1u = L1;
        if (p.seqused_q) {
            const int64_t u = p.seqused_q[b];
            if (u < 0 || u > L1) err |= LI_DEVERR_LENGTHS;
            L1u = u < 0 ? 0 : (u > L1 ? L1 : u);
        }
        if (p.layout_k == LI_LAYOUT_TND) {
            const int64_t c0 = p.cu_seqlens_k[b], c1 = p.cu_seqlens_k[b + 1];
            if (c0 < 0 || c1 < c0 || c1 > p.k_len) { err |= LI_DEVERR_LENGTHS; }
            L2 = (c1 >= c0 && c0 >= 0 && c1 <= p.k_len) ? c1 - c0 : 0;
            k0 = c0 < 0 ? 0 : c0;
        } else if (p.layout_k == LI_LAYOUT_PA_BSND) {
            const int64_t u = p.seqused_k[b];
            const int64_t cap = p.bt_stride * (int64_t)p.block_size;
            if (u < 0 || u > cap) err |= LI_DEVERR_LENGTHS;
            L2 = u < 0 ? 0 : (u > cap ? cap : u);
            k0 = 0;
        } else {
            L2 = p.k_len;
            k0 = (int64_t)b * p.k_len;
        }
        if (p.seqused_k && p.layout_k != LI_LAYOUT_PA_BSND) {
            const int64_t u = p.seqused_k[b];
            if (u < 0 || u > L2) err |= LI_DEVERR_LENGTHS;
            L2 = u < 0 ? 0 : (u < L2 ? u : L2);
        }
        if (L2 > p.max_seqlen_k) { err |= LI_DEVERR_LENGTHS; L2 = p.max_seqlen_k; }
        if (p.output_idx_offset) {
            const int64_t off = p.output_idx_offset[b];
            if (off < 0 || off + (L2 > 0 ? L2 - 1 : 0) > (int64_t)INT32_MAX) err |= LI_DEVERR_OFFSET;
        }
        int32_t res = 0;
        if (p.cmp_residual_k) {
            const int32_t u = p.cmp_residual_k[b];
            if (u < 0 || u >= p.cmp_ratio) err |= LI_DEVERR_LENGTHS;
            res = u < 0 ? 0 : (u >= p.cmp_ratio ? p.cmp_ratio - 1 : u);
        }
        bi.L1 = (int32_t)L1;
        bi.L1u = (int32_t)L1u;
        bi.L2 = (int32_t)L2;
        bi.q_row0 = (int32_t)q0;
        bi.k_row0 = (int32_t)k0;
        bi.pad[0] = bi.pad[1] = 0;
        bi.pad[2] = res;
        binfo[b] = bi;
        if (in_smem) {
            s_L1u[b] = bi.L1u;
            s_L2[b] = bi.L2;
            s_qr0[b] = bi.q_row0;
            s_kr0[b] = bi.k_row0;
            s_res[b] = res;
        }
        if (err) atomicOr(&s_status, err);
    }
    __syncthreads();

    // ---- query blocks per batch and their global numbering ------------------------------------
    __shared__ int32_t warp_sums[kMetaThreads / 32];
    int32_t carry = 0;
    for (int32_t b0 = 0; b0 < p.batch; b0 += kMetaThreads) {
        const int32_t b = b0 + tid;
        const int32_t l1u = b < p.batch ? (in_smem ? s_L1u[b] : binfo[b].L1u) : 0;
        const int32_t nqb = (l1u + s.tq - 1) / s.tq;
        const int32_t incl = block_inclusive_scan(nqb, warp_sums);
        if (b < p.batch) {
            binfo[b].pad[0] = nqb;
            binfo[b].pad[1] = carry + incl - nqb;
            if (in_smem) s_qb0[b] = carry + incl - nqb;
        }
        __syncthreads();
        if (tid == kMetaThreads - 1) warp_sums[0] = incl;       // block total
        __syncthreads();
        carry += warp_sums[0];
        __syncthreads();
    }
    const int32_t n_blocks = carry;
    __syncthreads();
    // batch lookups: shared memory when it holds every batch, else the global records
    const int32_t *qb0_arr = in_smem ? s_qb0 : nullptr;
    auto batch_info = [&](int32_t b) {
        BatchInfo bi;
        if (in_smem) {
            bi.L1u = s_L1u[b];
            bi.L2 = s_L2[b];
            bi.q_row0 = s_qr0[b];
            bi.k_row0 = s_kr0[b];
            bi.pad[1] = s_qb0[b];
            bi.pad[2] = s_res[b];
        } else {
            bi = binfo[b];
        }
        return bi;
    };
    auto block_batch = [&](int32_t gb) {
        if (qb0_arr) return batch_of_block(qb0_arr, p.batch, gb);
        int32_t lo = 0, hi = p.batch - 1;
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) >> 1;
            if (binfo[mid].pad[1] <= gb) lo = mid; else hi = mid - 1;
        }
        return lo;
    };

    // Items of query block gb: its window [0, jend) cut into n_s pieces of kc keys; every piece
    // but the last costs full_cost tiles, the last costs last_cost.
    struct BlockItems {
        int32_t b, q0, nq, jend, kc, n_s, full_cost, last_cost, row0, L1u, L2, k_row0;
    };
    auto block_items = [&](int32_t gb) {
        BlockItems r;
        r.b = block_batch(gb);
        const BatchInfo bi = batch_info(r.b);
        r.q0 = (gb - bi.pad[1]) * s.tq;
        r.nq = min(s.tq, bi.L1u - r.q0);
        // windows are prefixes [0, hi) growing with the row, so the block's last row has the widest
        r.jend = window_hi(p.mask_mode, r.q0 + r.nq - 1, bi.L1u, bi.L2, p.cmp_ratio, bi.pad[2]);
        r.kc = s.kc > 0 ? s.kc : r.jend;
        r.n_s = r.jend > 0 ? (r.jend + r.kc - 1) / r.kc : 0;
        r.full_cost = item_cost(0, r.kc);
        r.last_cost = r.n_s > 0 ? item_cost((r.n_s - 1) * r.kc, r.jend) : 0;
        r.row0 = bi.q_row0 + r.q0;
        r.L1u = bi.L1u;
        r.L2 = bi.L2;
        r.k_row0 = bi.k_row0;
        return r;
    };
    auto make_item = [&](const BlockItems &r, int32_t sp) {
        WorkItem it;
        it.b = r.b;
        it.q0 = r.q0;
        it.nq = r.nq;
        it.j0 = sp * r.kc;
        it.j1 = min(r.jend, it.j0 + r.kc);
        it.cost = sp + 1 < r.n_s ? r.full_cost : r.last_cost;
        it.row0 = r.row0;
        it.L1u = r.L1u;
        it.L2 = r.L2;
        it.k_row0 = r.k_row0;
        // compressed keys: a key count that makes the score kernel's plain window cover j1 for
        // every row (it clips at j1; the selection applies each row's exact window)
        if (p.cmp_residual_k) it.L2 = it.j1 + it.L1u;
        for (int i = 0; i < 6; ++i) it.pad[i] = 0;
        return it;
    };
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;

    // ---- pass 1: cost histogram, one or two adds per query block ------------------------------
    // Lanes of a warp whose last pieces cost the same add once, through their leader.
    int32_t mine = 0;
    for (int32_t g0 = 0; g0 < n_blocks; g0 += kMetaThreads) {
        const int32_t gb = g0 + tid;
        BlockItems r;
        r.n_s = 0;
        if (gb < n_blocks) r = block_items(gb);
        const bool ok = r.n_s > 0;
        if (ok && r.n_s > 1) atomicAdd(&hist[r.full_cost], r.n_s - 1);
        const int key = ok ? r.last_cost : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (ok && (peers & lt_mask) == 0) atomicAdd(&hist[key], __popc(peers));
        mine += r.n_s;
    }
    atomicAdd(&s_total, mine);
    __syncthreads();

    // ---- descending exclusive scan of the histogram: cursor[c] = items with cost > c ----------
    // thread t holds bin kCostBins - 1 - t, so an inclusive scan in thread order counts the bins
    // at or above each cost
    static_assert(kCostBins == kMetaThreads, "one histogram bin per thread");
    {
        const int bin = kCostBins - 1 - tid;
        const int32_t c = hist[bin];
        const int32_t incl = block_inclusive_scan(c, warp_sums);
        hist[bin] = incl - c;
    }
    __syncthreads();

    // ---- pass 2: placement -------------------------------------------------------------------
    const int32_t cap = s.max_items;
    if (s.kc == 0) {
        // one item per block: a thread per block, one atomic per equal-cost lane group
        for (int32_t g0 = 0; g0 < n_blocks; g0 += kMetaThreads) {
            const int32_t gb = g0 + tid;
            BlockItems r;
            r.n_s = 0;
            if (gb < n_blocks) r = block_items(gb);
            const bool ok = r.n_s > 0;
            const int key = ok ? r.last_cost : -1;
            const uint32_t peers = __match_any_sync(0xffffffffu, key);
            const int leader = __ffs(peers) - 1;
            int32_t base = 0;
            if (ok && lane == leader) base = atomicAdd(&hist[key], __popc(peers));
            base = __shfl_sync(0xffffffffu, base, leader);
            const int32_t slot = base + __popc(peers & lt_mask);
            if (ok && slot < cap) store_item(&items[slot], make_item(r, 0));
        }
    } else {
        // key splits (few query blocks, many pieces each): a warp per block; its lane 0 reserves
        // the block's full-cost pieces and its last piece, the lanes write the items
        for (int32_t gb = warp; gb < n_blocks; gb += kMetaThreads / 32) {
            const BlockItems r = block_items(gb);
            int32_t base_full = 0, base_last = 0;
            if (lane == 0 && r.n_s > 0) {
                if (r.n_s > 1) base_full = atomicAdd(&hist[r.full_cost], r.n_s - 1);
                base_last = atomicAdd(&hist[r.last_cost], 1);
            }
            base_full = __shfl_sync(0xffffffffu, base_full, 0);
            base_last = __shfl_sync(0xffffffffu, base_last, 0);
            for (int32_t sp = lane; sp < r.n_s; sp += 32) {
                const int32_t slot = sp + 1 < r.n_s ? base_full + sp : base_last;
                if (slot < cap) store_item(&items[slot], make_item(r, sp));
            }
        }
    }
    __syncthreads();

    if (tid == 0) {
        uint32_t st = s_status;
        int32_t n = s_total;
        if (n > cap) { st |= LI_DEVERR_LENGTHS; n = cap; }
        hdr->magic = kMetaMagic;
        hdr->status = st;
        hdr->n_items = n;
        hdr->max_items = cap;
        hdr->batch = p.batch;
        hdr->tq = s.tq;
        hdr->kc = s.kc;
        hdr->signature = problem_signature(p, s.tq, s.kc);
        for (int i = 0; i < 8; ++i) hdr->pad[i] = 0;
    }
}

}  // namespace

cudaError_t launch_metadata(const Problem &p, const Schedule &s, void *meta, cudaStream_t st) {
    MetaParams mp{p, s, meta};
    metadata_kernel<<<1, kMetaThreads, 0, st>>>(mp);
    return cudaGetLastError();
}

}  // namespace li
