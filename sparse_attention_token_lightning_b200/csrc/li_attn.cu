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
// processed in tiles of 128:
//   warp 4      scheduler: takes a ticket, finds the row's last selected position (the tile
//               count), publishes the row, and loads the row's Q tile (all heads, Dm + Dr dims)
//               with TMA into a 128-byte swizzled buffer
//   warps 6-9   gather: each tile's 128 key rows are copied with cp.async (16 bytes per thread and
//               copy, eight threads per 128-byte segment) into 128-byte swizzled chunks of 64 dims;
//               two chunks form a 32 KB pair slot, the rope dims a 16 KB rope slot
//   warp 5      allocates TMEM; one thread issues tcgen05.mma:
//                 S[key, g]  = sum over chunks  K_chunk . Q_chunk^T   (keys on M = 128, heads on N)
//                 O^T[d, g] += V^T . P^T       per pair of chunks (dims on M, keys on K; the key
//                                              tile is read MN-major, P from shared memory)
//   warps 0-3   softmax (thread = key = TMEM lane): S from TMEM, per-head tile max over the 128
//               keys, an online softmax against a reference max that moves only when the tile max
//               exceeds it by more than ln(256) (so every p <= 256; O and the sums are rescaled
//               then), p to shared memory as bf16 for the MMA, fp32 sums kept per thread; at the
//               end of the row the output rows O / l and the statistics
// Every wait is bounded in time; on expiry the kernel records LI_DEVERR_TIMEOUT and returns.
#include <cuda_bf16.h>

#include "li_attn.cuh"
#include "li_internal.cuh"
#include "li_sm100.cuh"

namespace li {
namespace {

using namespace sm100;

constexpr int kKeys = 128;                          // keys per tile (MMA M of S = K Q^T)
constexpr uint32_t kChunk = kKeys * 128;            // 64 dims of 128 keys: 16 KB
constexpr uint32_t kPair = 2 * kChunk;              // 128 dims: 32 KB
constexpr int kSoftWarps = 4, kSchedWarp = 4, kMmaWarp = 5, kGatherWarp0 = 6, kGatherWarps = 4;
constexpr int kThreads = 32 * 10;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr uint32_t kSmemBytes = 232448;
constexpr int kMaxPairSlots = 8, kMaxRopeSlots = 2;
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
    __device__ uint32_t rs_full(int i) const { return base + 8 * (0 + i); }
    __device__ uint32_t rs_empty(int i) const { return base + 8 * (2 + i); }
    __device__ uint32_t q_full(int i) const { return base + 8 * (4 + i); }
    __device__ uint32_t q_empty(int i) const { return base + 8 * (6 + i); }
    __device__ uint32_t s_full(int i) const { return base + 8 * (8 + i); }
    __device__ uint32_t s_empty(int i) const { return base + 8 * (10 + i); }
    __device__ uint32_t p_full(int i) const { return base + 8 * (12 + i); }
    __device__ uint32_t p_empty(int i) const { return base + 8 * (14 + i); }
    __device__ uint32_t o_done() const { return base + 8 * 16; }
    __device__ uint32_t o_full() const { return base + 8 * 17; }
    __device__ uint32_t o_empty() const { return base + 8 * 18; }
    __device__ uint32_t pair_full(int i) const { return base + 8 * (19 + i); }
    __device__ uint32_t pair_empty(int i) const { return base + 8 * (19 + kMaxPairSlots + i); }
    __device__ uint32_t rope_full(int i) const { return base + 8 * (19 + 2 * kMaxPairSlots + i); }
    __device__ uint32_t rope_empty(int i) const {
        return base + 8 * (19 + 2 * kMaxPairSlots + kMaxRopeSlots + i);
    }
    // exchange of the softmax warps' per-head partial results (tile max, row sums)
    __device__ uint32_t red_full(int i) const { return base + 8 * (19 + 2 * kMaxPairSlots + 2 * kMaxRopeSlots + i); }
    __device__ uint32_t sum_full(int i) const { return base + 8 * (21 + 2 * kMaxPairSlots + 2 * kMaxRopeSlots + i); }
};
constexpr int kNumBars = 23 + 2 * kMaxPairSlots + 2 * kMaxRopeSlots;
// tail: barriers | row slots | max and sum exchange, [2][4 warps][32] floats each | TMEM slot,
// abort flag
constexpr uint32_t kTailBytes = 3072;
constexpr uint32_t kTailOff = kSmemBytes - kTailBytes;
constexpr uint32_t kRowSlotOff = kTailOff + 8 * kNumBars;
constexpr uint32_t kRedOff = (kRowSlotOff + 2 * sizeof(RowSlot) + 15) / 16 * 16;
constexpr uint32_t kSumOff = kRedOff + 2 * 4 * 32 * 4;
constexpr uint32_t kFlagOff = kSumOff + 2 * 4 * 32 * 4;
static_assert(kFlagOff + 16 <= kSmemBytes, "shared memory tail");
static_assert(kTailOff % 1024 == 0, "tail alignment");

struct AttnParams {
    const uint16_t *k, *k_rope;          // key rows (Dm) and their rope dims (Dr), bf16
    const int32_t *indices;              // [rows][topk]
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
            S.key_base = row >= 0 ? (int64_t)(row / P.s1) * P.s2 : 0;
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
__device__ void gather_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                            volatile int *abort_flag) {
    const int t = threadIdx.x - 32 * kGatherWarp0;      // 0..127
    const int lane = t & 31;
    const int key0 = t >> 3, piece = t & 7;              // keys key0 + 16 i, 16-byte piece
    const uint32_t sbase = smem_u32(smem);
    const uint32_t swz = (uint32_t)((piece ^ (key0 & 7)) << 4);   // (key0 + 16 i) & 7 == key0 & 7
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    Ring pr, rr;
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
        for (int j = 0; j < tiles && ok; ++j) {
            const uint16_t *krow[8];
            const uint16_t *rrow[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pos = kKeys * j + key0 + 16 * i;
                const int32_t v = pos < P.topk ? __ldg(ir + pos) : -1;
                if (v >= P.s2) err |= LI_DEVERR_LENGTHS;
                // an unselected slot copies the batch's first key row (in bounds); its p is 0
                const int64_t kr = key_base + (v >= 0 && v < P.s2 ? v : 0);
                krow[i] = P.k + kr * P.Dm + 8 * piece;
                rrow[i] = P.Dr > 0 ? P.k_rope + kr * P.Dr + 8 * piece : nullptr;
            }
            for (int b = 0; b < P.npairs; ++b, pr.next(P.pair_slots)) {
                if (!wait_warp(bars.pair_empty(pr.idx), pr.phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t base = sbase + P.pair_off + pr.idx * kPair + key0 * 128u + swz;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        cp_async16(base + h * kChunk + i * 16u * 128u, krow[i] + 64 * (2 * b + h));
                cp_async_arrive(bars.pair_full(pr.idx));
            }
            if (!ok) break;
            if (P.Dr > 0) {
                if (!wait_warp(bars.rope_empty(rr.idx), rr.phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t base = sbase + P.rope_off + rr.idx * kChunk + key0 * 128u + swz;
#pragma unroll
                for (int i = 0; i < 8; ++i) cp_async16(base + i * 16u * 128u, rrow[i]);
                cp_async_arrive(bars.rope_full(rr.idx));
                rr.next(P.rope_slots);
            }
        }
    }
    // no copy may still be writing shared memory when the CTA leaves
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) *abort_flag = 1;
    if (err) atomicOr(P.status, err);
}

// ---- MMA issuer ----------------------------------------------------------------------------
__device__ void mma_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                         volatile int *abort_flag, uint32_t tmem) {
    const uint32_t sbase = smem_u32(smem);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const uint32_t N = (uint32_t)P.N;
    const uint32_t cb = N * 128u;                        // one Q chunk / one P atom column
    Ring qr, pr, rr, sr;
    uint32_t tile = 0, nrow = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        const uint32_t this_row = nrow++;
        if (tiles > 0) {
            if (!wait_(bars.q_full(qr.idx), qr.phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t qa = sbase + P.q_off + qr.idx * P.q_bytes;
            for (int j = 0; j < tiles; ++j, ++tile, sr.next(2)) {
                if (!wait_(bars.s_empty(sr.idx), sr.phase ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_s = tmem + sr.idx * N;
                Ring p0 = pr;
                for (int b = 0; b < P.npairs; ++b, p0.next(P.pair_slots)) {
                    if (!wait_(bars.pair_full(p0.idx), p0.phase, abort_flag)) { ok = false; break; }
                    fence_async_smem();
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t a = sw128_desc(sbase + P.pair_off + p0.idx * kPair + h * kChunk);
                        const uint64_t bq = sw128_desc(qa + (2 * b + h) * cb);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(d_s, a + 2 * kk, bq + 2 * kk, P.idesc_qk, (b | h | kk) != 0);
                    }
                }
                if (!ok) break;
                if (P.Dr > 0) {
                    if (!wait_(bars.rope_full(rr.idx), rr.phase, abort_flag)) { ok = false; break; }
                    fence_async_smem();
                    tc_fence_after();
                    const uint64_t a = sw128_desc(sbase + P.rope_off + rr.idx * kChunk);
                    const uint64_t bq = sw128_desc(qa + 2 * P.npairs * cb);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) umma_f16(d_s, a + 2 * kk, bq + 2 * kk, P.idesc_qk, 1u);
                    umma_commit(bars.rope_empty(rr.idx));
                    rr.next(P.rope_slots);
                }
                umma_commit(bars.s_full(sr.idx));
                // O is overwritten by the row's first tile: the previous row's output must have been
                // read out of TMEM (one o_empty phase per row, completed in order)
                if (j == 0 && this_row > 0 &&
                    !wait_(bars.o_empty(), (this_row - 1) & 1u, abort_flag)) { ok = false; break; }
                // P of this tile, then O^T += V^T P^T pair by pair
                if (!wait_(bars.p_full(sr.idx), sr.phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t pa = sbase + P.p_off + sr.idx * 2u * cb;
                for (int b = 0; b < P.npairs; ++b, pr.next(P.pair_slots)) {
                    const uint32_t va = sbase + P.pair_off + pr.idx * kPair;
                    const uint32_t d_o = tmem + 2u * N + b * N;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t a = sw128_desc_mn(va + kk * 16u * 128u, kChunk);
                        const uint64_t bp = sw128_desc(pa + (kk >> 2) * cb) + 2 * (kk & 3);
                        umma_f16(d_o, a, bp, P.idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bars.pair_empty(pr.idx));
                }
                umma_commit(bars.p_empty(sr.idx));
                umma_commit(bars.o_done());
            }
            if (!ok) break;
            umma_commit(bars.q_empty(qr.idx));
            qr.next(P.q_bufs);
        }
        umma_commit(bars.o_full());
    }
    if (!ok) *abort_flag = 1;
}

// ---- softmax and output ----------------------------------------------------------------------
// Per-head reduction of NH values over the 32 lanes of a warp, transposed: afterwards lane l
// holds the result for head head_of_lane<NH>(l) (lanes l and l ^ 1 share a head when NH = 16).
template <int NH>
__device__ __forceinline__ int head_of_lane(int lane) {
    // the halving steps keep the upper half on lanes whose bit (16, 8, 4, 2[, 1]) is set
    if constexpr (NH == 32)
        return ((lane >> 4) & 1) * 16 + ((lane >> 3) & 1) * 8 + ((lane >> 2) & 1) * 4 +
               ((lane >> 1) & 1) * 2 + (lane & 1);
    else
        return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
               ((lane >> 1) & 1);
}
template <int NH, bool kMax>
__device__ __forceinline__ float warp_reduce_heads(const float (&v)[NH], int lane) {
    float a[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) a[i] = v[i];
    // step s halves the values held: lanes with bit (16 >> s) set keep the upper half
    constexpr int kSteps = NH == 32 ? 5 : 4;
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
        const int bit = 16 >> s;
        const int half = NH >> (s + 1);
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < NH / 2; ++i) {
            if (i < half) {
                const float keep = up ? a[i + half] : a[i];
                const float send = up ? a[i] : a[i + half];
                const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
                a[i] = kMax ? fmaxf(keep, recv) : keep + recv;
            }
        }
    }
    // NH = 16 leaves lane bit 0 unreduced
    if constexpr (NH == 16) {
        const float o = __shfl_xor_sync(0xffffffffu, a[0], 1);
        a[0] = kMax ? fmaxf(a[0], o) : a[0] + o;
    }
    return a[0];
}

// S of this thread's key: NH columns of its TMEM lane.
template <int NH>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[NH]) {
    float a[16];
    tmem_ld16(taddr, a);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = a[i];
    if constexpr (NH == 32) {
        tmem_ld16(taddr + 16, a);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 + i] = a[i];
    }
}

// bf16 bits of x, round to nearest even (x is finite and non-negative here)
__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

template <int NH>
__device__ void softmax_role(const AttnParams &P, uint8_t *smem, const Bars &bars,
                             volatile int *abort_flag, uint32_t tmem) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int key = 32 * w + lane;                        // TMEM lane: key of the tile / dim of O
    const uint32_t lane_addr = (uint32_t)(32 * w) << 16;
    const uint32_t N = (uint32_t)P.N;
    const uint32_t cb = N * 128u;
    const uint32_t sbase = smem_u32(smem);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    float *red = reinterpret_cast<float *>(smem + kRedOff);      // [2][4 warps][32]
    float *sumx = reinterpret_cast<float *>(smem + kSumOff);     // [2][4 warps][32]
    const float kInf = __int_as_float(0x7f800000);
    const int my_head = head_of_lane<NH>(lane);
    // P element (head h, this key) in the K-major 128-byte swizzled tile: atom column key / 64,
    // row h, 16-byte chunk ((key % 64) / 8) ^ (h % 8)
    const uint32_t p_key = (uint32_t)(key >> 6) * cb + (uint32_t)((key & 7) << 1);
    const uint32_t p_chunk = (uint32_t)((key & 63) >> 3);
    Ring sr;
    uint32_t tile = 0, nrow = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_warp(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        const int32_t *ir = P.indices + (int64_t)row * P.topk;
        float m_ref[NH], m_true[NH], l_part[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) { m_ref[h] = -kInf; m_true[h] = -kInf; l_part[h] = 0.f; }
        for (int j = 0; j < tiles; ++j, ++tile, sr.next(2)) {
            const int pos = kKeys * j + key;
            const int32_t v = pos < P.topk ? __ldg(ir + pos) : -1;
            const bool valid = v >= 0 && v < P.s2;
            if (!wait_warp(bars.s_full(sr.idx), sr.phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float x[NH];
            tmem_ld_row<NH>(tmem + lane_addr + sr.idx * N, x);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_empty(sr.idx));
#pragma unroll
            for (int h = 0; h < NH; ++h) x[h] = valid ? x[h] * P.scale : -kInf;
            // tile max per head over the 128 keys
            float *rb = red + (tile & 1) * 4 * 32;
            const float wm = warp_reduce_heads<NH, true>(x, lane);
            if (NH == 32 || (lane & 1) == 0) rb[w * 32 + my_head] = wm;
            mbar_arrive(bars.red_full(tile & 1));
            if (!wait_warp(bars.red_full(tile & 1), (tile >> 1) & 1u, abort_flag)) { ok = false; break; }
            bool rescale = false;
            float alpha[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float tm = fmaxf(fmaxf(rb[h], rb[32 + h]), fmaxf(rb[64 + h], rb[96 + h]));
                m_true[h] = fmaxf(m_true[h], tm);
                const float ref = tm - m_ref[h] > kSlack ? tm : m_ref[h];
                alpha[h] = ref != m_ref[h] ? exp2f((m_ref[h] - ref) * kLog2e) : 1.f;
                rescale |= ref != m_ref[h];
                m_ref[h] = ref;
                l_part[h] *= alpha[h];
            }
            float p[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                p[h] = valid ? exp2f((x[h] - m_ref[h]) * kLog2e) : 0.f;
                l_part[h] += p[h];
            }
            // O (accumulated up to the previous tile) follows a moved reference
            if (rescale && j > 0) {
                if (!wait_warp(bars.o_done(), (tile - 1) & 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int b = 0; b < P.npairs; ++b) {
#pragma unroll
                    for (int c = 0; c < NH; c += 16) {
                        const uint32_t ta = tmem + lane_addr + 2u * N + b * N + c;
                        float o[16];
                        tmem_ld16(ta, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= alpha[c + i];
                        tmem_st16(ta, o);
                    }
                }
                tc_fence_before();
            }
            // p as bf16 into this tile's P buffer once the MMA has finished with it
            if (!wait_warp(bars.p_empty(sr.idx), sr.phase ^ 1u, abort_flag)) { ok = false; break; }
            uint8_t *pb = smem + P.p_off + sr.idx * 2u * cb + p_key;
#pragma unroll
            for (int h = 0; h < NH; ++h)
                *reinterpret_cast<uint16_t *>(pb + (h >> 3) * 1024 + (h & 7) * 128 +
                                              ((p_chunk ^ (uint32_t)(h & 7)) << 4)) = bf16_bits(p[h]);
            fence_async_smem();
            mbar_arrive(bars.p_full(sr.idx));
        }
        if (!ok) break;
        // row totals of the fp32 sums (exchange buffers alternate by row)
        float *sb = sumx + (nrow & 1) * 4 * 32;
        {
            const float ws = warp_reduce_heads<NH, false>(l_part, lane);
            if (NH == 32 || (lane & 1) == 0) sb[w * 32 + my_head] = ws;
            mbar_arrive(bars.sum_full(nrow & 1));
            if (!wait_warp(bars.sum_full(nrow & 1), (nrow >> 1) & 1u, abort_flag)) { ok = false; break; }
        }
        float l_tot[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) l_tot[h] = (sb[h] + sb[32 + h]) + (sb[64 + h] + sb[96 + h]);
        if (!wait_warp(bars.o_full(), nrow & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int G = P.G;
        float *orow = P.out + (int64_t)row * G * P.Dm;
        if (tiles > 0) {
            for (int b = 0; b < P.npairs; ++b) {
#pragma unroll
                for (int c = 0; c < NH; c += 16) {
                    float o[16];
                    tmem_ld16(tmem + lane_addr + 2u * N + b * N + c, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c + i < G)
                            orow[(int64_t)(c + i) * P.Dm + 128 * b + key] =
                                l_tot[c + i] > 0.f ? o[i] / l_tot[c + i] : 0.f;
                }
            }
        } else {
            for (int b = 0; b < P.npairs; ++b)
                for (int h = 0; h < G; ++h) orow[(int64_t)h * P.Dm + 128 * b + key] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            if (h == key && h < G) {
                const bool any = m_true[h] > -kInf;
                P.smax[(int64_t)row * G + h] = m_true[h];
                P.ssum[(int64_t)row * G + h] = any ? l_tot[h] * exp2f((m_ref[h] - m_true[h]) * kLog2e) : 0.f;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.o_empty());
        ++nrow;
    }
    if (!ok) *abort_flag = 1;
}

template <int NH>
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
            mbar_init(bars.rs_empty(i), 1 + kSoftWarps + kGatherWarps);
            mbar_init(bars.q_full(i), 1);
            mbar_init(bars.q_empty(i), 1);
            mbar_init(bars.s_full(i), 1);
            mbar_init(bars.s_empty(i), kSoftWarps);
            mbar_init(bars.p_full(i), 32 * kSoftWarps);
            mbar_init(bars.p_empty(i), 1);
        }
        mbar_init(bars.o_done(), 1);
        mbar_init(bars.o_full(), 1);
        mbar_init(bars.o_empty(), kSoftWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.red_full(i), 32 * kSoftWarps);
            mbar_init(bars.sum_full(i), 32 * kSoftWarps);
        }
        for (int i = 0; i < kMaxPairSlots; ++i) {
            mbar_init(bars.pair_full(i), kGatherThreads);
            mbar_init(bars.pair_empty(i), 1);
        }
        for (int i = 0; i < kMaxRopeSlots; ++i) {
            mbar_init(bars.rope_full(i), kGatherThreads);
            mbar_init(bars.rope_empty(i), 1);
        }
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
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), P.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kSoftWarps) {
        softmax_role<NH>(P, smem, bars, abort_flag, tmem);
    } else if (warp == kSchedWarp) {
        scheduler_role(P, &tmap_q, &tmap_qr, smem, bars, abort_flag);
    } else if (warp == kMmaWarp) {
        if (lane == 0) mma_role(P, smem, bars, abort_flag, tmem);
        __syncwarp();
    } else {
        gather_role(P, smem, bars, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(P.status, LI_DEVERR_TIMEOUT);
    if (warp == kMmaWarp) {
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
    const uint32_t p_bytes = 2u * 2u * N * 128u;           // two buffers of N x 128 keys bf16
    for (int q_bufs = 2; q_bufs >= 1; --q_bufs) {
        const uint32_t q_end = q_bufs * L->q_bytes;
        const uint32_t pair_off = (q_end + p_bytes + 1023u) / 1024u * 1024u;
        const uint32_t avail = kTailOff > pair_off ? kTailOff - pair_off : 0;
        int rope = a.Dr > 0 ? kMaxRopeSlots : 0;
        int pairs = 0;
        for (; rope >= (a.Dr > 0 ? 1 : 0); --rope) {
            const uint32_t left = avail > rope * kChunk ? avail - rope * kChunk : 0;
            pairs = (int)(left / kPair);
            if (pairs > kMaxPairSlots) pairs = kMaxPairSlots;
            if (pairs >= npairs + 1) break;                 // one pair of prefetch
            if (rope == (a.Dr > 0 ? 1 : 0)) break;
        }
        // two Q buffers only when a pair of prefetch remains
        if (q_bufs == 2 && pairs < npairs + 1) continue;
        if (pairs < npairs) return false;
        L->q_bufs = q_bufs;
        L->q_off = 0;
        L->p_off = q_end;
        L->pair_off = pair_off;
        L->pair_slots = pairs;
        L->rope_off = pair_off + pairs * kPair;
        L->rope_slots = rope;
        uint32_t cols = 32;
        while (cols < (uint32_t)(2 * N + npairs * N)) cols <<= 1;
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
    // D fp32, A and B bf16, K-major A and B (S = K Q^T) / MN-major A (O^T = V^T P^T); N, M = 128
    const uint32_t base = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(L.N >> 3) << 17) |
                          ((uint32_t)(128 >> 4) << 24);
    P.idesc_qk = base;
    P.idesc_pv = base | (1u << 15);
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
    auto kern = L.N <= 16 ? sparse_attn_kernel<16> : sparse_attn_kernel<32>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    int grid = device_sm_count();
    if (rows < grid) grid = (int)rows;
    kern<<<grid, kThreads, kSmemBytes, st>>>(mq, mr, P);
    return cudaGetLastError();
}

}  // namespace li
