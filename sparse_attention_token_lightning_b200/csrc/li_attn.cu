// Sparse attention over the keys the indexer selected (the indexer's consumer), sm_100a.
//
// For query row r (batch b), head g < G and the row's selected keys s (sparse_indices: positions
// in batch b's key sequence, negative = no key) -- aclnnLightningIndexerV2, main computation steps
// (the selected indices are the attention's input); aclnnSparseFlashAttentionGrad, calculation
// formula (the selected keys and values are gathered by the top-k indices; value = key is the
// supported case):
//     x[s]     = scale * (q[r,g,:] . k[s,:] + q_rope[r,g,:] . k_rope[s,:])
//     m        = max_s x[s],     l = sum_s exp(x[s] - m)
//     o[r,g,:] = sum_s exp(x[s] - m) / l * k[s,:]          (the value rows are the key rows)
// and the forward statistics softmax_max = m, softmax_sum = l (the inputs of the indexer's
// backward). A row with no selected key gets o = 0, m = -inf, l = 0.
//
// One persistent CTA per SM takes query rows from a ticket counter. Per row the selected keys are
// processed in tiles of 64:
//   warp 8      scheduler: takes a ticket, finds the row's last selected position (the tile
//               count), publishes the row, and loads the row's Q tile (all heads, Dm + Dr dims)
//               with TMA into a 128-byte swizzled buffer
//   warps 11-14 gather: each tile's 64 key rows (dense keys at the batch's row plus the index, or
//               paged keys through the batch's block-table row; the paged instantiations carry
//               that lookup) are copied with cp.async (16 bytes per thread and copy, eight
//               threads per 128-byte segment) into 128-byte swizzled chunks of 64 dims;
//               two chunks form a 16 KB pair slot, the rope dims an 8 KB rope slot; one barrier
//               per tile signals its arrival
//   warp 9      allocates TMEM; one thread issues the scores S = sum over chunks K_chunk Q_chunk^T
//               (keys on M = 64, heads on N; row m of S sits in TMEM lane m % 16 + 32 (m / 16))
//   warp 10     one thread issues the values O_g^T += V^T P^T per pair of chunks (dims on M = 128,
//               keys on K; the key tile read MN-major, P from shared memory); a tcgen05.mma
//               costs about the same to issue whatever its N, so the two products are issued
//               from two threads
//   warps 0-7   softmax, two groups of four warps: group g takes the row's tiles j = g, g + 2, ...
//               with its own S and P buffers, its own O accumulator and its own online softmax,
//               so the two groups work on consecutive tiles at once; lanes 0-15 of a warp hold
//               the first half of a key's heads, lanes 16-31 the second half. The reference max
//               of a group moves only when a tile max exceeds it by more than ln(256) (so every
//               p <= 256; O and the sums are rescaled then); p goes to shared memory as bf16 for
//               the MMA and the sums stay in fp32. At the end of the row group 1 hands its
//               statistics to group 0, which combines the two partial outputs and writes the
//               output rows and the statistics.
// Every wait is bounded in time; on expiry the kernel records LI_DEVERR_TIMEOUT and returns.
#include <cuda_bf16.h>

#include "li_attn.cuh"
#include "li_internal.cuh"
#include "li_sm100.cuh"

namespace li {
namespace {

using namespace sm100;

constexpr int kKeys = 64;                           // keys per tile (MMA M of S = K Q^T)
constexpr uint32_t kChunk = kKeys * 128;            // 64 dims of 64 keys: 8 KB
constexpr uint32_t kPair = 2 * kChunk;              // 128 dims: 16 KB
// warps 0-7 softmax (group = warp / 4 takes the row's tiles j with j % 2 == group; quarter =
// warp % 4), 8 scheduler, 9 scores MMA (and TMEM), 10 values MMA, 11-14 gather
constexpr int kSoftWarps = 8, kSchedWarp = 8, kQkWarp = 9, kPvWarp = 10, kGatherWarp0 = 11;
constexpr int kGatherWarps = 4;
constexpr int kThreads = 32 * 15;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kGroupThreads = 128;
constexpr uint32_t kSmemBytes = 232448;
constexpr int kMaxPairSlots = 16, kMaxRopeSlots = 2, kTileRing = 8;
constexpr int kMaxHeads = 32;
constexpr float kLog2e = 1.4426950408889634f;
// the reference max moves when a tile max exceeds it by more than this (natural log units):
// every p = exp(x - ref) stays <= 256
constexpr float kSlack = 5.545177444479562f;        // ln 256
constexpr uint32_t kDevErrInternal = 0x20u;

struct RowSlot {
    int32_t row, tiles, n_eff, pad;
    int64_t key_base;
    int64_t pad2;
};

// Barrier layout in the shared-memory tail.
struct Bars {
    uint32_t base;
    __device__ uint32_t at(int i) const { return base + 8 * i; }
    __device__ uint32_t rs_full(int i) const { return at(0 + i); }
    __device__ uint32_t rs_empty(int i) const { return at(2 + i); }
    __device__ uint32_t q_full(int i) const { return at(4 + i); }
    __device__ uint32_t q_empty(int i) const { return at(6 + i); }
    __device__ uint32_t s_full(int g) const { return at(8 + g); }          // per softmax group
    __device__ uint32_t s_empty(int g) const { return at(10 + g); }
    __device__ uint32_t p_full(int g) const { return at(12 + g); }
    __device__ uint32_t p_empty(int g) const { return at(14 + g); }
    __device__ uint32_t o_done(int g) const { return at(16 + g); }
    __device__ uint32_t o_full() const { return at(18); }
    __device__ uint32_t o_empty() const { return at(19); }
    __device__ uint32_t stat_full(int i) const { return at(20 + i); }
    __device__ uint32_t stat_empty(int i) const { return at(22 + i); }
    __device__ uint32_t red_full(int g, int b) const { return at(24 + 2 * g + b); }
    __device__ uint32_t sum_full(int g, int b) const { return at(28 + 2 * g + b); }
    __device__ uint32_t tile_full(int i) const { return at(32 + i); }
    __device__ uint32_t rope_empty(int i) const { return at(32 + kTileRing + i); }
    __device__ uint32_t pair_empty(int i) const { return at(32 + kTileRing + kMaxRopeSlots + i); }
};
constexpr int kNumBars = 32 + kTileRing + kMaxRopeSlots + kMaxPairSlots;
// tail: barriers | row slots | per group: tile-max and row-sum exchange [2 groups][2][32 heads]
// [4 warps] floats | group-1 statistics [2][3][32] | TMEM slot, abort flag
constexpr uint32_t kTailBytes = 6144;
constexpr uint32_t kTailOff = kSmemBytes - kTailBytes;
constexpr uint32_t kRowSlotOff = kTailOff + 8 * kNumBars;
constexpr uint32_t kRedOff = (kRowSlotOff + 2 * sizeof(RowSlot) + 15) / 16 * 16;
constexpr uint32_t kSumOff = kRedOff + 2 * 2 * kMaxHeads * 4 * 4;
constexpr uint32_t kStatOff = kSumOff + 2 * 2 * kMaxHeads * 4 * 4;
constexpr uint32_t kFlagOff = kStatOff + 2 * 3 * kMaxHeads * 4;
static_assert(kFlagOff + 16 <= kSmemBytes, "shared memory tail");
static_assert(kTailOff % 1024 == 0, "tail alignment");

struct AttnParams {
    const uint16_t *k, *k_rope;          // key rows (Dm) and their rope dims (Dr), bf16
    const int32_t *indices;              // [rows][topk]
    const int32_t *block_table;          // paged keys: [B][bt_stride]; null for dense keys
    int64_t key_rows;                    // rows of k: B * S2, or num_blocks * block_size
    int32_t bt_stride, block_size, num_blocks, pad0;
    float *out, *smax, *ssum;            // [rows][G][Dm], [rows][G], [rows][G]
    uint32_t *status;
    int32_t *ticket;
    float scale;
    int32_t rows, s1, s2, G, N, Dm, Dr, topk;
    int32_t npairs, q_bufs, pair_slots, rope_slots;
    uint32_t q_bytes;                    // one Q buffer: (2 npairs + rope) chunks of N x 128 B
    uint32_t q_off, p_off, pair_off, rope_off;
    uint32_t idesc_qk, idesc_pv;
    uint32_t tmem_cols;
};

// Position in a ring of n buffers with its phase parity.
struct Ring {
    int idx = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++idx == n) { idx = 0; phase ^= 1u; }
    }
};

__device__ __forceinline__ bool wait_(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return mbar_wait(bar, parity, abort_flag);
}
// The same wait taken by a whole warp, with one answer for all lanes (a lane that saw the phase
// complete and one that gave up on the abort flag at the same moment agree on giving up).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// TMEM columns: S of group g at g N; O of group g, pair b at 2 N + (g npairs + b) N.
__device__ __forceinline__ uint32_t o_col(const AttnParams &P, int g, int b) {
    return (uint32_t)(2 * P.N + (g * P.npairs + b) * P.N);
}

// ---- scheduler: rows and their Q tiles --------------------------------------------------------
__device__ void scheduler_role(const AttnParams &P, const CUtensorMap *tmq, const CUtensorMap *tmr,
                               uint8_t *smem, const Bars &bars, volatile int *abort_flag) {
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    RowSlot *slots = reinterpret_cast<RowSlot *>(smem + kRowSlotOff);
    const int nqc = 2 * P.npairs + (P.Dr > 0 ? 1 : 0);
    Ring qr;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        int row = 0;
        if (lane == 0) row = atomicAdd(P.ticket, 1);
        row = __shfl_sync(0xffffffffu, row, 0);
        if (row >= P.rows) row = -1;
        int last = -1;
        if (row >= 0) {
            const int32_t *ir = P.indices + (int64_t)row * P.topk;
#pragma unroll 4
            for (int pos = lane; pos < P.topk; pos += 32)
                if (__ldg(ir + pos) >= 0) last = pos;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        }
        const int n_eff = last + 1;
        const int tiles = (n_eff + kKeys - 1) / kKeys;
        const int sl = it & 1;
        if (!wait_warp(bars.rs_empty(sl), ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (lane == 0) {
            RowSlot &S = slots[sl];
            S.row = row;
            S.tiles = tiles;
            S.n_eff = n_eff;
            // dense keys: the batch's first key row; paged keys: the batch (its block-table row)
            S.key_base = row < 0 ? 0 : P.block_table ? (int64_t)(row / P.s1) : (int64_t)(row / P.s1) * P.s2;
            mbar_arrive(bars.rs_full(sl));
        }
        __syncwarp();
        if (row < 0) break;
        if (tiles == 0) continue;
        if (!wait_warp(bars.q_empty(qr.idx), qr.phase ^ 1u, abort_flag)) { ok = false; break; }
        if (lane == 0) {
            const uint32_t dst = sbase + P.q_off + qr.idx * P.q_bytes;
            const uint32_t cb = (uint32_t)P.N * 128u;
            mbar_arrive_expect_tx(bars.q_full(qr.idx), (uint32_t)nqc * P.G * 128u);
            for (int c = 0; c < 2 * P.npairs; ++c)
                tma_load_2d(dst + c * cb, tmq, bars.q_full(qr.idx), 64 * c, row * P.G);
            if (P.Dr > 0)
                tma_load_2d(dst + 2 * P.npairs * cb, tmr, bars.q_full(qr.idx), 0, row * P.G);
        }
        __syncwarp();
        qr.next(P.q_bufs);
    }
    if (!ok) *abort_flag = 1;
}

// ---- gather: the selected key rows of each tile into the pair and rope slots -------------------
template <bool kPaged>
__device__ void gather_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                            volatile int *abort_flag) {
    const int t = threadIdx.x - 32 * kGatherWarp0;      // 0..127
    const int lane = t & 31;
    const int key0 = t >> 3, piece = t & 7;              // keys key0 + 16 i (i < 4), 16-byte piece
    const uint32_t sbase = smem_u32(smem);
    const uint32_t swz = (uint32_t)((piece ^ (key0 & 7)) << 4);   // (key0 + 16 i) & 7 == key0 & 7
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    Ring pr, rr, tr;
    uint32_t err = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_warp(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        const int64_t key_base = slots[sl].key_base;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        const int32_t *ir = P.indices + (int64_t)row * P.topk;
        for (int j = 0; j < tiles && ok; ++j, tr.next(kTileRing)) {
            const uint16_t *krow[4];
            const uint16_t *rrow[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pos = kKeys * j + key0 + 16 * i;
                const int32_t v = pos < P.topk ? __ldg(ir + pos) : -1;
                if (v >= P.s2) err |= LI_DEVERR_LENGTHS;
                // an unselected slot copies an in-bounds row (the batch's first key, or cache row
                // 0); its p is 0
                int64_t kr;
                if constexpr (kPaged) {
                    // paged keys: the row of position v through the batch's block table
                    kr = 0;
                    if (v >= 0 && v < P.s2) {
                        const int32_t blk = __ldg(P.block_table + key_base * P.bt_stride + v / P.block_size);
                        if (blk >= 0 && blk < P.num_blocks) kr = (int64_t)blk * P.block_size + v % P.block_size;
                        else err |= LI_DEVERR_TABLE;
                    }
                } else {
                    kr = key_base + (v >= 0 && v < P.s2 ? v : 0);
                }
                if (!idx_ok(kr, P.key_rows, P.status)) kr = 0;
                krow[i] = P.k + kr * P.Dm + 8 * piece;
                rrow[i] = P.Dr > 0 ? P.k_rope + kr * P.Dr + 8 * piece : nullptr;
            }
            for (int b = 0; b < P.npairs; ++b, pr.next(P.pair_slots)) {
                if (!wait_warp(bars.pair_empty(pr.idx), pr.phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t base = sbase + P.pair_off + pr.idx * kPair + key0 * 128u + swz;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        cp_async16(base + h * kChunk + i * 16u * 128u, krow[i] + 64 * (2 * b + h));
            }
            if (!ok) break;
            if (P.Dr > 0) {
                if (!wait_warp(bars.rope_empty(rr.idx), rr.phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t base = sbase + P.rope_off + rr.idx * kChunk + key0 * 128u + swz;
#pragma unroll
                for (int i = 0; i < 4; ++i) cp_async16(base + i * 16u * 128u, rrow[i]);
                rr.next(P.rope_slots);
            }
            // one arrival per thread once every copy of the tile has landed
            cp_async_arrive(bars.tile_full(tr.idx));
        }
    }
    // no copy may still be writing shared memory when the CTA leaves
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) *abort_flag = 1;
    if (err) atomicOr(P.status, err);
}

// ---- scores MMA: S(j) = K(j) Q^T into the S buffer of tile j's softmax group -------------------
__device__ void qk_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                        volatile int *abort_flag, uint32_t tmem) {
    const uint32_t sbase = smem_u32(smem);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const uint32_t N = (uint32_t)P.N;
    const uint32_t cb = N * 128u;
    Ring qr, pq, rr, tr;
    uint32_t kg[2] = {0u, 0u};                           // tiles of each group so far
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        if (tiles == 0) continue;
        if (!wait_(bars.q_full(qr.idx), qr.phase, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qa = sbase + P.q_off + qr.idx * P.q_bytes;
        for (int j = 0; j < tiles; ++j, tr.next(kTileRing)) {
            const int g = j & 1;
            if (!wait_(bars.s_empty(g), (kg[g] & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            if (!wait_(bars.tile_full(tr.idx), tr.phase, abort_flag)) { ok = false; break; }
            fence_async_smem();                  // the gathered rows, for the async proxy
            tc_fence_after();
            const uint32_t d_s = tmem + g * N;
            for (int b = 0; b < P.npairs; ++b, pq.next(P.pair_slots)) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint64_t a = sw128_desc(sbase + P.pair_off + pq.idx * kPair + h * kChunk);
                    const uint64_t bq = sw128_desc(qa + (2 * b + h) * cb);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(d_s, a + 2 * kk, bq + 2 * kk, P.idesc_qk, (b | h | kk) != 0);
                }
            }
            if (P.Dr > 0) {
                const uint64_t a = sw128_desc(sbase + P.rope_off + rr.idx * kChunk);
                const uint64_t bq = sw128_desc(qa + 2 * P.npairs * cb);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) umma_f16(d_s, a + 2 * kk, bq + 2 * kk, P.idesc_qk, 1u);
                umma_commit(bars.rope_empty(rr.idx));
                rr.next(P.rope_slots);
            }
            umma_commit(bars.s_full(g));
            ++kg[g];
        }
        if (!ok) break;
        umma_commit(bars.q_empty(qr.idx));
        qr.next(P.q_bufs);
    }
    if (!ok) *abort_flag = 1;
}

// ---- values MMA: O_g^T += V(j)^T P(j)^T for tile j of group g --------------------------------
__device__ void pv_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                        volatile int *abort_flag, uint32_t tmem) {
    const uint32_t sbase = smem_u32(smem);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const uint32_t N = (uint32_t)P.N;
    const uint32_t cb = N * 128u;
    Ring pv;
    uint32_t kg[2] = {0u, 0u};
    uint32_t nrow = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        const uint32_t this_row = nrow++;
        for (int j = 0; j < tiles; ++j) {
            const int g = j & 1;
            // both groups' O are overwritten by the row's first two tiles: the previous row's
            // output must have been read out of TMEM (one o_empty phase per row, in order)
            if (j == 0 && this_row > 0 && !wait_(bars.o_empty(), (this_row - 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (!wait_(bars.p_full(g), kg[g] & 1u, abort_flag)) { ok = false; break; }
            fence_async_smem();
            tc_fence_after();
            const uint32_t pa = sbase + P.p_off + g * cb;
            for (int b = 0; b < P.npairs; ++b, pv.next(P.pair_slots)) {
                const uint32_t va = sbase + P.pair_off + pv.idx * kPair;
                const uint32_t d_o = tmem + o_col(P, g, b);
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint64_t a = sw128_desc_mn(va + kk * 16u * 128u, kChunk);
                    umma_f16(d_o, a, sw128_desc(pa) + 2 * kk, P.idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bars.pair_empty(pv.idx));
            }
            umma_commit(bars.p_empty(g));
            umma_commit(bars.o_done(g));
            ++kg[g];
        }
        if (!ok) break;
        umma_commit(bars.o_full());
    }
    if (!ok) *abort_flag = 1;
}

// ---- softmax and output ----------------------------------------------------------------------
// Per-head reduction of HH values over the 16 lanes of a half-warp, transposed: afterwards lane l
// holds the result for head (l >> 4) * HH + half_head<HH>(l) (with HH = 8, lanes l and l ^ 1
// share a head).
template <int HH>
__device__ __forceinline__ int half_head(int lane) {
    if constexpr (HH == 16)
        return ((lane >> 3) & 1) * 8 + ((lane >> 2) & 1) * 4 + ((lane >> 1) & 1) * 2 + (lane & 1);
    else
        return ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}
template <int HH, bool kMax>
__device__ __forceinline__ float half_reduce(const float (&v)[HH], int lane) {
    float a[HH];
#pragma unroll
    for (int i = 0; i < HH; ++i) a[i] = v[i];
    // step s halves the values held: lanes with bit (8 >> s) set keep the upper half
    constexpr int kSteps = HH == 16 ? 4 : 3;
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
        const int bit = 8 >> s;
        const int half = HH >> (s + 1);
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < HH / 2; ++i) {
            if (i < half) {
                const float keep = up ? a[i + half] : a[i];
                const float send = up ? a[i] : a[i + half];
                const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
                a[i] = kMax ? fmaxf(keep, recv) : keep + recv;
            }
        }
    }
    if constexpr (HH == 8) {
        const float o = __shfl_xor_sync(0xffffffffu, a[0], 1);
        a[0] = kMax ? fmaxf(a[0], o) : a[0] + o;
    }
    return a[0];
}

// bf16 bits of x, round to nearest even (x is finite and non-negative here)
__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Softmax group g (warps 4 g .. 4 g + 3) over the row's tiles j = g, g + 2, ...: each thread owns
// key 16 q + (lane % 16) of the tile (q = warp % 4, the TMEM lanes of M = 64 scores) and heads
// (lane / 16) HH .. + HH - 1 of it. Group 1 hands its statistics to group 0, which combines the
// two partial outputs and writes the row.
template <int NH, bool kPaged>
__device__ void softmax_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                             volatile int *abort_flag, uint32_t tmem) {
    constexpr int HH = NH / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 2, q = warp & 3;
    const int key = 16 * q + (lane & 15);
    const int half = lane >> 4;
    const int hb = half * HH;
    const int dlane = 32 * q + lane;                     // dim of a 128-dim block of O
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const uint32_t N = (uint32_t)P.N;
    const uint32_t cb = N * 128u;
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    float *red = reinterpret_cast<float *>(smem + kRedOff) + g * 2 * kMaxHeads * 4;
    float *sumx = reinterpret_cast<float *>(smem + kSumOff) + g * 2 * kMaxHeads * 4;
    float *stat = reinterpret_cast<float *>(smem + kStatOff);    // [2][3][kMaxHeads]
    const float kInf = __int_as_float(0x7f800000);
    const int my_head = hb + half_head<HH>(lane);
    const bool writer = HH == 16 || (lane & 1) == 0;
    // P element (head h, this key) in the K-major 128-byte swizzled tile of N rows x 64 keys:
    // row h, 16-byte chunk (key / 8) ^ (h % 8)
    const uint32_t p_key = (uint32_t)((key & 7) << 1);
    const uint32_t p_chunk = (uint32_t)(key >> 3);
    uint32_t kg = 0, nrow = 0;                           // this group's tiles, rows
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_warp(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        const int32_t *ir = P.indices + (int64_t)row * P.topk;
        // references and true maxima of this thread's heads hb .. hb + HH - 1
        float mr[HH], mt[HH], l_part[HH];
#pragma unroll
        for (int i = 0; i < HH; ++i) { mr[i] = -kInf; mt[i] = -kInf; }
#pragma unroll
        for (int i = 0; i < HH; ++i) l_part[i] = 0.f;
        int mine = 0;                                    // tiles of this group in the row
        for (int j = g; j < tiles; j += 2, ++kg, ++mine) {
            const int pos = kKeys * j + key;
            const int32_t v = pos < P.topk ? __ldg(ir + pos) : -1;
            bool valid = v >= 0 && v < P.s2;
            if (kPaged && valid) {
                // paged keys: a block-table entry out of range selects nothing (the gather
                // reported it)
                const int32_t blk = __ldg(P.block_table + (int64_t)(row / P.s1) * P.bt_stride + v / P.block_size);
                valid = blk >= 0 && blk < P.num_blocks;
            }
            if (!wait_warp(bars.s_full(g), kg & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float x[16];
            float y[HH];
            tmem_ld16(tmem + lane_addr + g * N, x);      // lanes 0-15: heads 0-15 of the key
            if constexpr (NH == 16) {
#pragma unroll
                for (int i = 0; i < HH; ++i) {
                    const float up = __shfl_sync(0xffffffffu, x[HH + i], lane & 15);
                    y[i] = half ? up : x[i];
                }
            } else {
                float x2[16];
                tmem_ld16(tmem + lane_addr + g * N + 16, x2);
#pragma unroll
                for (int i = 0; i < HH; ++i) {
                    const float up = __shfl_sync(0xffffffffu, x2[i], lane & 15);
                    y[i] = half ? up : x[i];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_empty(g));
#pragma unroll
            for (int i = 0; i < HH; ++i) y[i] = valid ? y[i] * P.scale : -kInf;
            // tile max per head over the group's 64 keys
            float *rb = red + (kg & 1) * kMaxHeads * 4;
            const float wm = half_reduce<HH, true>(y, lane);
            if (writer) rb[my_head * 4 + q] = wm;
            mbar_arrive(bars.red_full(g, kg & 1));
            if (!wait_warp(bars.red_full(g, kg & 1), (kg >> 1) & 1u, abort_flag)) { ok = false; break; }
            // this thread's heads only; the other half of the warp holds the rest
            bool moved = false;
            float alpha[HH];
#pragma unroll
            for (int i = 0; i < HH; ++i) {
                const float4 r4 = *reinterpret_cast<const float4 *>(rb + (hb + i) * 4);
                const float tm = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
                mt[i] = fmaxf(mt[i], tm);
                const float ref = tm - mr[i] > kSlack ? tm : mr[i];
                alpha[i] = ref != mr[i] ? exp2f((mr[i] - ref) * kLog2e) : 1.f;
                moved |= ref != mr[i];
                mr[i] = ref;
            }
            // every warp of the group sees the same tile maxima, so the vote is group-wide
            const bool rescale = __any_sync(0xffffffffu, moved);
            float p[HH];
#pragma unroll
            for (int i = 0; i < HH; ++i) {
                p[i] = valid ? exp2f((y[i] - mr[i]) * kLog2e) : 0.f;
                l_part[i] = l_part[i] * alpha[i] + p[i];
            }
            // this group's O (accumulated up to its previous tile) follows a moved reference
            if (rescale && mine > 0) {
                if (!wait_warp(bars.o_done(g), (kg - 1) & 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // every head's factor: own half and the other half's, from lane ^ 16
                float af[NH];
#pragma unroll
                for (int i = 0; i < HH; ++i) {
                    const float other = __shfl_xor_sync(0xffffffffu, alpha[i], 16);
                    af[i] = half ? other : alpha[i];
                    af[HH + i] = half ? alpha[i] : other;
                }
                for (int b = 0; b < P.npairs; ++b) {
#pragma unroll
                    for (int c = 0; c < NH; c += 16) {
                        const uint32_t ta = tmem + lane_addr + o_col(P, g, b) + c;
                        float o[16];
                        tmem_ld16(ta, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= af[c + i];
                        tmem_st16(ta, o);
                    }
                }
                tc_fence_before();
            }
            // p as bf16 into the group's P buffer once the MMA has finished with it
            if (!wait_warp(bars.p_empty(g), (kg & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            {
                uint8_t *pb = smem + P.p_off + g * cb + p_key;
#pragma unroll
                for (int i = 0; i < HH; ++i) {
                    const int h = hb + i;
                    *reinterpret_cast<uint16_t *>(pb + (h >> 3) * 1024 + (h & 7) * 128 +
                                                  ((p_chunk ^ (uint32_t)(h & 7)) << 4)) =
                        bf16_bits(p[i]);
                }
            }
            fence_async_smem();
            mbar_arrive(bars.p_full(g));
        }
        if (!ok) break;
        // row totals of this group's fp32 sums (exchange buffers alternate by row)
        float *sb = sumx + (nrow & 1) * kMaxHeads * 4;
        {
            const float ws = half_reduce<HH, false>(l_part, lane);
            if (writer) sb[my_head * 4 + q] = ws;
            mbar_arrive(bars.sum_full(g, nrow & 1));
            if (!wait_warp(bars.sum_full(g, nrow & 1), (nrow >> 1) & 1u, abort_flag)) { ok = false; break; }
        }
        // every head's reference and true maximum (own half and the other half's)
        float m_ref[NH], m_true[NH];
#pragma unroll
        for (int i = 0; i < HH; ++i) {
            const float orr = __shfl_xor_sync(0xffffffffu, mr[i], 16);
            const float ort = __shfl_xor_sync(0xffffffffu, mt[i], 16);
            m_ref[i] = half ? orr : mr[i];
            m_ref[HH + i] = half ? mr[i] : orr;
            m_true[i] = half ? ort : mt[i];
            m_true[HH + i] = half ? mt[i] : ort;
        }
        float l_tot[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float4 s4 = *reinterpret_cast<const float4 *>(sb + h * 4);
            l_tot[h] = (s4.x + s4.y) + (s4.z + s4.w);
        }
        float *st = stat + (nrow & 1) * 3 * kMaxHeads;
        if (g == 1) {
            // hand the statistics to group 0
            if (!wait_warp(bars.stat_empty(nrow & 1), ((nrow >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            if (warp == 4 && lane == 0) {
                for (int h = 0; h < NH; ++h) {
                    st[h] = m_ref[h];
                    st[kMaxHeads + h] = m_true[h];
                    st[2 * kMaxHeads + h] = l_tot[h];
                }
                mbar_arrive(bars.stat_full(nrow & 1));
            }
            __syncwarp();
            ++nrow;
            continue;
        }
        if (!wait_warp(bars.stat_full(nrow & 1), (nrow >> 1) & 1u, abort_flag)) { ok = false; break; }
        // combine: c = the larger reference; weights of the two partial sums
        const bool two = tiles >= 2;
        float wa[NH], wb[NH], inv[NH];
        float smx[NH], ssm[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float rb_ = st[h], tb = st[kMaxHeads + h], lb = st[2 * kMaxHeads + h];
            const float c = two ? fmaxf(m_ref[h], rb_) : m_ref[h];
            wa[h] = m_ref[h] > -kInf ? exp2f((m_ref[h] - c) * kLog2e) : 0.f;
            wb[h] = two && rb_ > -kInf ? exp2f((rb_ - c) * kLog2e) : 0.f;
            const float L = l_tot[h] * wa[h] + (two ? lb * wb[h] : 0.f);
            inv[h] = L > 0.f ? 1.f / L : 0.f;
            const float mt = two ? fmaxf(m_true[h], tb) : m_true[h];
            smx[h] = mt;
            ssm[h] = mt > -kInf ? L * exp2f((c - mt) * kLog2e) : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.stat_empty(nrow & 1));
        if (!wait_warp(bars.o_full(), nrow & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int G = P.G;
        const bool row_ok = idx_ok(row, P.rows, P.status);
        float *orow = P.out + (int64_t)row * G * P.Dm;
        for (int b = 0; b < P.npairs; ++b) {
#pragma unroll
            for (int c = 0; c < NH; c += 16) {
                float oa[16], ob[16];
                if (tiles > 0) tmem_ld16(tmem + lane_addr + o_col(P, 0, b) + c, oa);
                if (two) tmem_ld16(tmem + lane_addr + o_col(P, 1, b) + c, ob);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int h = c + i;
                    if (h < G && row_ok) {
                        float o = 0.f;
                        if (tiles > 0) o = oa[i] * wa[h];
                        if (two) o += ob[i] * wb[h];
                        orow[(int64_t)h * P.Dm + 128 * b + dlane] = o * inv[h];
                    }
                }
            }
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            if (h == dlane && h < G && row_ok) {
                P.smax[(int64_t)row * G + h] = smx[h];
                P.ssum[(int64_t)row * G + h] = ssm[h];
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.o_empty());
        ++nrow;
    }
    if (!ok) *abort_flag = 1;
}

template <int NH, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_qr,
                   const AttnParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) atomicOr(P.status, kDevErrInternal);
        return;
    }
    Bars bars{sbase + kTailOff};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kFlagOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kFlagOff + 4);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.rs_full(i), 1);
            mbar_init(bars.rs_empty(i), 2 + kSoftWarps + kGatherWarps);
            mbar_init(bars.q_full(i), 1);
            mbar_init(bars.q_empty(i), 1);
            mbar_init(bars.s_full(i), 1);
            mbar_init(bars.s_empty(i), 4);
            mbar_init(bars.p_full(i), kGroupThreads);
            mbar_init(bars.p_empty(i), 1);
            mbar_init(bars.o_done(i), 1);
            mbar_init(bars.stat_full(i), 1);
            mbar_init(bars.stat_empty(i), 4);
            for (int b = 0; b < 2; ++b) {
                mbar_init(bars.red_full(i, b), kGroupThreads);
                mbar_init(bars.sum_full(i, b), kGroupThreads);
            }
        }
        mbar_init(bars.o_full(), 1);
        mbar_init(bars.o_empty(), 4);
        for (int i = 0; i < kTileRing; ++i) mbar_init(bars.tile_full(i), kGatherThreads);
        for (int i = 0; i < kMaxRopeSlots; ++i) mbar_init(bars.rope_empty(i), 1);
        for (int i = 0; i < kMaxPairSlots; ++i) mbar_init(bars.pair_empty(i), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // heads G..N-1 of the Q buffers are never loaded: zero them once so their columns stay finite
    {
        const int nqc = 2 * P.npairs + (P.Dr > 0 ? 1 : 0);
        const int pad_rows = P.N - P.G;
        const int per_chunk = pad_rows * 8;              // 16-byte words
        const int total = P.q_bufs * nqc * per_chunk;
        for (int i = threadIdx.x; i < total; i += kThreads) {
            const int c = i / per_chunk, r = i % per_chunk;
            uint8_t *dst = smem + P.q_off + c * P.N * 128 + (P.G + r / 8) * 128 + (r % 8) * 16;
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
    }
    if (warp == kSchedWarp && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)) : "memory");
        if (P.Dr > 0)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_qr)) : "memory");
    }
    if (warp == kQkWarp) {
        tmem_alloc(smem_u32(tmem_slot), P.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kSoftWarps) {
        softmax_role<NH, kPaged>(P, smem, bars, abort_flag, tmem);
    } else if (warp == kSchedWarp) {
        scheduler_role(P, &tmap_q, &tmap_qr, smem, bars, abort_flag);
    } else if (warp == kQkWarp) {
        if (lane == 0) qk_role(P, smem, bars, abort_flag, tmem);
        __syncwarp();
    } else if (warp == kPvWarp) {
        if (lane == 0) pv_role(P, smem, bars, abort_flag, tmem);
        __syncwarp();
    } else {
        gather_role<kPaged>(P, smem, bars, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(P.status, LI_DEVERR_TIMEOUT);
    if (warp == kQkWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, P.tmem_cols);
    }
}

// 2-D bf16 tensor map over [rows, cols] (cols contiguous), box {64, box_rows}, 128-byte swizzle.
bool make_map_bf16(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn || rows == 0) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_layout(const li_attn_args &a, AttnLayout *L) {
    const int N = (a.G + 15) / 16 * 16;
    const int npairs = a.Dm / 128;
    const int nqc = 2 * npairs + (a.Dr > 0 ? 1 : 0);
    L->N = N;
    L->npairs = npairs;
    L->q_bytes = (uint32_t)nqc * N * 128u;
    const uint32_t p_bytes = 2u * N * 128u;                 // one N x 64-key bf16 tile per group
    const int rope = a.Dr > 0 ? kMaxRopeSlots : 0;
    // the MMA order keeps two tiles resident: at least 2 npairs pair slots; two Q buffers when
    // they leave room for one more pair
    for (int q_bufs = 2; q_bufs >= 1; --q_bufs) {
        const uint32_t q_end = q_bufs * L->q_bytes;
        const uint32_t pair_off = (q_end + p_bytes + 1023u) / 1024u * 1024u;
        const uint32_t need = (uint32_t)rope * kChunk;
        if (pair_off + need >= kTailOff) continue;
        int pairs = (int)((kTailOff - pair_off - need) / kPair);
        if (pairs > kMaxPairSlots) pairs = kMaxPairSlots;
        // the gather may run at most this many tiles ahead of the scores (tile barrier ring)
        if (pairs > (kTileRing - 2) * npairs) pairs = (kTileRing - 2) * npairs;
        if (q_bufs == 2 && pairs < 2 * npairs + 1) continue;
        if (pairs < 2 * npairs) return false;
        L->q_bufs = q_bufs;
        L->q_off = 0;
        L->p_off = q_end;
        L->pair_off = pair_off;
        L->pair_slots = pairs;
        L->rope_off = pair_off + pairs * kPair;
        L->rope_slots = rope;
        uint32_t cols = 32;
        while (cols < (uint32_t)(2 * N + 2 * npairs * N)) cols <<= 1;
        L->tmem_cols = cols;
        return true;
    }
    return false;
}

cudaError_t launch_sparse_attention(const li_attn_args &a, uint32_t *status, int32_t *ticket,
                                    float *out, float *smax, float *ssum, cudaStream_t st) {
    AttnLayout L;
    if (!attn_layout(a, &L)) return cudaErrorInvalidConfiguration;
    const int64_t rows = (int64_t)a.batch * a.s1;
    if (rows == 0) return cudaSuccess;
    AttnParams P{};
    P.k = static_cast<const uint16_t *>(a.k);
    P.k_rope = static_cast<const uint16_t *>(a.k_rope);
    P.indices = a.sparse_indices;
    if (a.layout_k == LI_LAYOUT_PA_BSND) {
        P.block_table = a.block_table;
        P.bt_stride = a.block_table_stride;
        P.block_size = a.block_size;
        P.num_blocks = a.num_blocks;
        P.key_rows = (int64_t)a.num_blocks * a.block_size;
    } else {
        P.key_rows = (int64_t)a.batch * a.s2;
    }
    P.out = out;
    P.smax = smax;
    P.ssum = ssum;
    P.status = status;
    P.ticket = ticket;
    P.scale = a.scale;
    P.rows = (int32_t)rows;
    P.s1 = a.s1;
    P.s2 = a.s2;
    P.G = a.G;
    P.N = L.N;
    P.Dm = a.Dm;
    P.Dr = a.Dr;
    P.topk = a.topk;
    P.npairs = L.npairs;
    P.q_bufs = L.q_bufs;
    P.pair_slots = L.pair_slots;
    P.rope_slots = L.rope_slots > 0 ? L.rope_slots : 1;
    P.q_bytes = L.q_bytes;
    P.q_off = L.q_off;
    P.p_off = L.p_off;
    P.pair_off = L.pair_off;
    P.rope_off = L.rope_off;
    // D fp32, A and B bf16, N; S = K Q^T: K-major A and B, M = 64; O^T = V^T P^T: MN-major A,
    // M = 128
    const uint32_t base = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(L.N >> 3) << 17);
    P.idesc_qk = base | ((uint32_t)(kKeys >> 4) << 24);
    P.idesc_pv = base | (1u << 15) | ((uint32_t)(128 >> 4) << 24);
    P.tmem_cols = L.tmem_cols;
    CUtensorMap mq, mr;
    if (!make_map_bf16(&mq, a.q, (uint64_t)rows * a.G, (uint64_t)a.Dm, (uint32_t)a.G))
        return cudaErrorInvalidValue;
    if (a.Dr > 0) {
        if (!make_map_bf16(&mr, a.q_rope, (uint64_t)rows * a.G, (uint64_t)a.Dr, (uint32_t)a.G))
            return cudaErrorInvalidValue;
    } else {
        mr = mq;
    }
    // paged keys have instantiations of their own, so the dense kernels carry no paged code
    const bool paged = a.layout_k == LI_LAYOUT_PA_BSND;
    auto kern = L.N <= 16 ? (paged ? sparse_attn_kernel<16, true> : sparse_attn_kernel<16, false>)
                          : (paged ? sparse_attn_kernel<32, true> : sparse_attn_kernel<32, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    int grid = device_sm_count();
    if (rows < grid) grid = (int)rows;
    kern<<<grid, kThreads, kSmemBytes, st>>>(mq, mr, P);
    return cudaGetLastError();
}

}  // namespace li
