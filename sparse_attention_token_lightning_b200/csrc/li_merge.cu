// Split merge: the top-k of the union of several per-row top-k lists (one per key range of a
// row), in the selection's order: score descending, then key index ascending.
//
// Every input row is already sorted, so the output slot of an entry is its rank in the union:
// its position in its own list plus, for every other list, the number of entries that come
// before it there. A thread takes a run of kChunk consecutive entries of one list, finds the
// first entry's place in every other list by binary search and walks forward from there for the
// rest of the run, so the ranks of a run cost one search and about one step per entry. Ranks
// are distinct (equal entries from two lists are ordered by list), so every output slot below
// the number of valid entries is written exactly once, and the rest is padded. Only the first
// topk_out entries of an input row can reach the output, so nothing past them is read.
//
// Two kernels. merge_tree_kernel (one CTA per row, the fast path) copies the row's lists into
// shared memory as 64-bit order keys with many loads in flight, then merges them pairwise, level
// by level, each result cut to topk_out entries; a pair's output positions are split evenly over
// its threads, each finding its start on the merge path by binary search. merge_kernel (one CTA
// per (row, list), the ranking scheme above) probes global memory and serves rows whose lists do
// not fit in shared memory.
//
// HBM traffic: every input entry that can reach the output is read once (8 B) and every output
// slot is written once (8 B, 4 B without values).
#include <cstdint>

#include "li_internal.cuh"
#include "li_merge.cuh"

namespace li {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 8;

struct MergeParams {
    const int32_t *idx[LI_MERGE_MAX_LISTS];
    const float *val[LI_MERGE_MAX_LISTS];
    int32_t *idx_out;
    float *val_out;
    uint32_t *status;
    int32_t n_lists, topk_in, topk_out;
    int32_t lim;          // entries of an input row that can reach the output: min(topk_in, topk_out)
    int32_t check;        // verify the input order (lists from outside the library)
};

// Larger key = earlier in the order. The score is mapped to an order-preserving unsigned
// integer (-0 as +0) and the index complemented, so a lower index wins among equal scores.
__device__ __forceinline__ uint64_t order_key(int32_t i, float v) {
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((uint64_t)b << 32) | (uint32_t)~(uint32_t)i;
}

__device__ __forceinline__ uint64_t key_at(const MergeParams &P, int l, int64_t at) {
    return order_key(__ldg(P.idx[l] + at), __ldg(P.val[l] + at));
}

// Number of leading valid entries (index >= 0) among the first lim of a row.
__device__ int32_t valid_prefix(const MergeParams &P, int l, int64_t base) {
    int32_t lo = 0, hi = P.lim;
    while (lo < hi) {
        const int32_t mid = (lo + hi) >> 1;
        if (__ldg(P.idx[l] + base + mid) >= 0) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// y comes before x in the union: strictly earlier, or equal and from a lower list.
__device__ __forceinline__ bool before(uint64_t y, uint64_t x, bool lower_list) {
    return lower_list ? y >= x : y > x;
}

__global__ void __launch_bounds__(kThreads) merge_kernel(const __grid_constant__ MergeParams P) {
    const int64_t r = blockIdx.x;
    const int a = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t base = r * (int64_t)P.topk_in;
    __shared__ int32_t s_len[LI_MERGE_MAX_LISTS];
    __shared__ int32_t s_bad;
    if (tid < P.n_lists) s_len[tid] = valid_prefix(P, tid, base);
    if (tid == 0) s_bad = 0;
    __syncthreads();

    const int32_t len_a = s_len[a];
    bool bad = false;
    for (int32_t e = len_a + tid; e < P.lim; e += kThreads)   // padding only after the prefix
        if (__ldg(P.idx[a] + base + e) >= 0) bad = true;
    for (int32_t e = tid; e + 1 < len_a; e += kThreads)       // strictly ordered prefix
        if (!(key_at(P, a, base + e) > key_at(P, a, base + e + 1))) bad = true;

    int32_t *oi = P.idx_out + r * (int64_t)P.topk_out;
    float *ov = P.val_out ? P.val_out + r * (int64_t)P.topk_out : nullptr;
    const int32_t n_runs = (len_a + kChunk - 1) / kChunk;
    for (int32_t c = tid; c < n_runs; c += kThreads) {
        const int32_t e0 = c * kChunk;
        const int32_t ne = min(kChunk, len_a - e0);
        uint64_t x[kChunk];
        int32_t rank[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            x[j] = j < ne ? key_at(P, a, base + e0 + j) : 0;
            rank[j] = e0 + j;
        }

        for (int b = 0; b < P.n_lists; ++b) {
            if (b == a) continue;
            const int32_t len_b = s_len[b];
            const bool lower = b < a;
            int32_t lo = 0, hi = len_b;
            while (lo < hi) {
                const int32_t mid = (lo + hi) >> 1;
                if (before(key_at(P, b, base + mid), x[0], lower)) lo = mid + 1;
                else hi = mid;
            }
            int32_t p = lo;
            rank[0] += p;
#pragma unroll
            for (int j = 1; j < kChunk; ++j) {
                if (j < ne) {
                    while (p < len_b && before(key_at(P, b, base + p), x[j], lower)) ++p;
                    rank[j] += p;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            if (j < ne && rank[j] < P.topk_out) {
                const int32_t i = (int32_t)~(uint32_t)x[j];
                oi[rank[j]] = i;
                if (ov) {
                    const float v = __ldg(P.val[a] + base + e0 + j);
                    ov[rank[j]] = v == 0.0f ? 0.0f : v;
                }
            }
        }
        if (rank[0] >= P.topk_out) break;   // the ranks of later runs of this list are larger
    }

    if (a == 0) {
        int32_t total = 0;
        for (int b = 0; b < P.n_lists; ++b) total += s_len[b];
        for (int32_t s = min(total, P.topk_out) + tid; s < P.topk_out; s += kThreads) {
            oi[s] = -1;
            if (ov) ov[s] = __int_as_float(0xff800000);
        }
    }
    if (bad) s_bad = 1;
    __syncthreads();
    if (tid == 0 && s_bad && P.status) atomicOr(P.status, (uint32_t)LI_DEVERR_MERGE_ORDER);
}

constexpr int kTreeThreads = 512;
constexpr int kStageUnroll = 16;                 // entries each thread has in flight while staging

__device__ __forceinline__ float key_value(uint64_t k) {
    const uint32_t u = (uint32_t)(k >> 32);
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// One CTA per row. The row's lists are staged in shared memory as order keys, then merged in a
// binary tree: at each level list 2p is merged with list 2p+1 (an odd last list is carried up by
// a merge with an empty list) and the result cut to topk_out entries, which keeps every entry of
// the final top-k. A pair's output positions are split evenly over its threads; each thread
// finds where its first position falls in the two inputs by binary search on the merge path and
// then takes its k positions one after the other. Equal keys take the lower list first. The
// last level writes the output row.
__global__ void __launch_bounds__(kTreeThreads) merge_tree_kernel(const __grid_constant__ MergeParams P,
                                                               int32_t y_off) {
    extern __shared__ uint64_t s_mem[];          // [0, G*lim): staged lists; [y_off, ...): odd levels
    __shared__ int32_t s_off[2][LI_MERGE_MAX_LISTS];
    __shared__ int32_t s_len[2][LI_MERGE_MAX_LISTS];
    __shared__ int32_t s_bad;
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const int G = P.n_lists, lim = P.lim;
    const int64_t base = r * (int64_t)P.topk_in;
    if (tid == 0) s_bad = 0;
    // flat position f = l * lim + e over all lists, kept as (l, e) and advanced by the block
    // size without a division; kStageUnroll independent loads per thread
    const int32_t total_in = G * lim;
    int sl = 0;
    int32_t se = tid;
    while (se >= lim && sl < G) { se -= lim; ++sl; }
    const int sl0 = sl;
    const int32_t se0 = se;
    for (int32_t f0 = 0; f0 < total_in; f0 += kTreeThreads * kStageUnroll) {
        // loads only in this loop (no branch on a loaded value), so all of them are in flight
        int32_t iv[kStageUnroll], fe[kStageUnroll];
        float vv[kStageUnroll];
#pragma unroll
        for (int u = 0; u < kStageUnroll; ++u) {
            iv[u] = -1;
            vv[u] = 0.0f;
            fe[u] = -1;
            if (sl < G) {
                const int64_t at = base + se;
                iv[u] = __ldg(P.idx[sl] + at);
                vv[u] = __ldg(P.val[sl] + at);
                fe[u] = sl * lim + se;
                se += kTreeThreads;
                while (se >= lim && sl < G) { se -= lim; ++sl; }
            }
        }
#pragma unroll
        for (int u = 0; u < kStageUnroll; ++u)
            if (fe[u] >= 0 && idx_ok(fe[u], total_in, P.status))
                s_mem[fe[u]] = iv[u] >= 0 ? order_key(iv[u], vv[u]) : 0ull;
    }
    __syncthreads();
    // input contract: within a list, keys strictly decrease until the padding (key 0) starts
    bool bad = false;
    for (sl = P.check ? sl0 : G, se = se0; sl < G;) {
        if (se + 1 < lim) {
            const uint64_t k0 = s_mem[sl * lim + se], k1 = s_mem[sl * lim + se + 1];
            if (k1 != 0 && !(k0 > k1)) bad = true;
        }
        se += kTreeThreads;
        while (se >= lim && sl < G) { se -= lim; ++sl; }
    }
    // valid prefix of each list
    if (tid < G) {
        const uint64_t *k = s_mem + tid * lim;
        int32_t lo = 0, hi = lim;
        while (lo < hi) {
            const int32_t mid = (lo + hi) >> 1;
            if (k[mid] != 0) lo = mid + 1;
            else hi = mid;
        }
        s_len[0][tid] = lo;
        s_off[0][tid] = tid * lim;
    }
    __syncthreads();

    int32_t *oi = P.idx_out + r * (int64_t)P.topk_out;
    float *ov = P.val_out ? P.val_out + r * (int64_t)P.topk_out : nullptr;
    int cur = 0, count = G;
    int32_t src = 0, dst = y_off;              // word offsets of this level's input and output
    for (;;) {
        const int pairs = (count + 1) >> 1;
        const bool last = pairs == 1;
        if (tid == 0) {
            int32_t o = 0;
            for (int q = 0; q < pairs; ++q) {
                const int32_t na = s_len[cur][2 * q];
                const int32_t nb = 2 * q + 1 < count ? s_len[cur][2 * q + 1] : 0;
                const int32_t n = min(na + nb, P.topk_out);
                s_off[cur ^ 1][q] = o;
                s_len[cur ^ 1][q] = n;
                o += n;
            }
        }
        __syncthreads();
        const int tpp = kTreeThreads / pairs;
        const int q = tid / tpp, tt = tid - q * tpp;
        if (q < pairs) {
            const uint64_t *A = s_mem + src + s_off[cur][2 * q];
            const int32_t na = s_len[cur][2 * q];
            const bool hasB = 2 * q + 1 < count;
            const uint64_t *B = hasB ? s_mem + src + s_off[cur][2 * q + 1] : A;
            const int32_t nb = hasB ? s_len[cur][2 * q + 1] : 0;
            const int32_t n_out = s_len[cur ^ 1][q];
            // an odd run length keeps the lanes of a warp (k entries apart) on different banks
            const int32_t k = ((n_out + tpp - 1) / tpp) | 1;
            const int32_t d = tt * k;
            if (d < n_out) {
                // merge path: i entries of A are among the first d outputs
                int32_t lo = max(0, d - nb), hi = min(d, na);
                while (lo < hi) {
                    const int32_t i = (lo + hi) >> 1;
                    if (A[i] >= B[d - i - 1]) lo = i + 1;
                    else hi = i;
                }
                int32_t i = lo, j = d - lo;
                uint64_t a = i < na ? A[i] : 0ull;
                uint64_t b = j < nb ? B[j] : 0ull;
                uint64_t *out = s_mem + dst + s_off[cur ^ 1][q];
                const int32_t end = min(d + k, n_out);
                for (int32_t pos = d; pos < end; ++pos) {
                    const bool takeA = j >= nb || (i < na && a >= b);
                    const uint64_t x = takeA ? a : b;
                    if (takeA) {
                        ++i;
                        a = i < na ? A[i] : 0ull;
                    } else {
                        ++j;
                        b = j < nb ? B[j] : 0ull;
                    }
                    if (last) {
                        if (!idx_ok(pos, P.topk_out, P.status)) break;
                        oi[pos] = (int32_t)~(uint32_t)x;
                        if (ov) ov[pos] = key_value(x);
                    } else {
                        out[pos] = x;
                    }
                }
            }
        }
        if (last) break;
        __syncthreads();
        const int32_t nsrc = dst;
        dst = src;
        src = nsrc;
        cur ^= 1;
        count = pairs;
    }

    const int32_t n_final = s_len[cur ^ 1][0];
    for (int32_t s = n_final + tid; s < P.topk_out; s += kTreeThreads) {
        oi[s] = -1;
        if (ov) ov[s] = __int_as_float(0xff800000);
    }
    if (bad) s_bad = 1;
    __syncthreads();
    if (tid == 0 && s_bad && P.status) atomicOr(P.status, (uint32_t)LI_DEVERR_MERGE_ORDER);
}

// Shared memory of merge_tree_kernel: the staged lists, then the largest odd-level output.
size_t tree_smem_words(int G, int lim, int topk_out, int32_t *y_off) {
    int64_t y = 0;
    int count = G;
    for (int level = 1; count > 1; ++level) {
        const int pairs = (count + 1) / 2;
        int64_t per = (int64_t)lim << level;
        if (per > topk_out) per = topk_out;
        if (level & 1) y = y > pairs * per ? y : pairs * per;
        count = pairs;
    }
    *y_off = G * lim;
    return (size_t)G * lim + (size_t)y;
}

constexpr size_t kSmemMergeMax = 200u * 1024u;   // dynamic shared memory of merge_smem_kernel

}  // namespace

bool merge_fits_smem(int n_lists, int topk_in, int topk_out) {
    int32_t y_off = 0;
    const int lim = topk_in < topk_out ? topk_in : topk_out;
    return tree_smem_words(n_lists, lim, topk_out, &y_off) * sizeof(uint64_t) <= kSmemMergeMax;
}

cudaError_t launch_merge(const li_merge_args &a, cudaStream_t stream, bool check) {
    MergeParams P{};
    for (int l = 0; l < a.n_lists; ++l) {
        P.idx[l] = a.idx_in[l];
        P.val[l] = a.val_in[l];
    }
    P.idx_out = a.idx_out;
    P.val_out = a.val_out;
    P.status = a.device_status;
    P.n_lists = a.n_lists;
    P.topk_in = a.topk_in;
    P.topk_out = a.topk_out;
    P.lim = a.topk_in < a.topk_out ? a.topk_in : a.topk_out;
    P.check = check ? 1 : 0;
    int32_t y_off = 0;
    const size_t smem = tree_smem_words(a.n_lists, P.lim, a.topk_out, &y_off) * sizeof(uint64_t);
    if (smem <= kSmemMergeMax) {
        cudaError_t e = cudaFuncSetAttribute(merge_tree_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMergeMax);
        if (e != cudaSuccess) return e;
        merge_tree_kernel<<<(unsigned)a.rows, kTreeThreads, smem, stream>>>(P, y_off);
        return cudaGetLastError();
    }
    const dim3 grid((unsigned)a.rows, (unsigned)a.n_lists);
    merge_kernel<<<grid, kThreads, 0, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace li
