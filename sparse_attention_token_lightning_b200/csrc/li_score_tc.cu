// Score kernel on the 5th-generation tensor cores (tcgen05 + TMA + TMEM), sm_100a.
//
// Computes, for every work item (batch b, query rows [q0, q0+nq), keys [j0, j1)), the index score
//     I[t, j] = sum_h w[t,h] * ReLU(q[t,h,:] . k[j,:])
// (custom_pypto.npu_lightning_indexer_pto, function description formula; lightning_indexer,
// "Function" steps 1-3) and writes it to the fp32 score rows of the workspace for the keys of
// each row's window (right-down causal or none, custom_pypto.npu_lightning_indexer_pto,
// sparse_mode). The head-by-key score tensor never leaves the SM.
//
// Orientation: keys on the MMA M axis (128 TMEM lanes), query rows x heads on N:
//     D[key, t*N1 + h] = k_key . q[t, h]          M = 128, N = tq*N1 (<= 256), K = 128
// so every epilogue thread owns one key (one TMEM lane) and reduces the heads of a row in
// registers; no cross-lane reduction is needed and w is a per-row broadcast.
//
// Warp roles (one CTA per SM, persistent, work items pulled from a global ticket counter):
//   warp 18     scheduler: takes tickets, stages each item's header, weights and paged cache rows
//   warp 0      TMA producer: the item's Q tile (double buffered), its K tiles through a ring of
//               as many stages as fit; paged keys piece by piece through the staged rows
//   warp 1      allocates TMEM (512 columns); one thread issues the tcgen05.mma chain per tile
//               (8 x kind::f16 K16 for bf16/fp16, 4 x kind::f8f6f4 K32 for fp8) and commits
//   warps 2-17  epilogue: four warps per TMEM lane quarter, warp group g taking rows g, g+4, ..;
//               tcgen05.ld of a row's N1 columns, ReLU, weight, head sum (fp8: times the key's
//               scale), causal mask, coalesced fp32 stores
// Instantiated per w type and for fp8 q/k. Every wait on an mbarrier is bounded in time; on
// expiry the kernel records LI_DEVERR_TIMEOUT, the roles leave their loops, TMEM is freed and the
// kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "li_internal.cuh"
#include "li_sm100.cuh"

namespace li {
namespace {

using namespace sm100;

#ifndef LI_EPI_WARPS
#define LI_EPI_WARPS 16
#endif
constexpr int kEpiWarps = LI_EPI_WARPS;                 // multiple of 4 (one per TMEM lane quarter)
constexpr int kEpiGroups = kEpiWarps / 4;               // warps sharing a lane quarter split the rows
constexpr int kSchedWarp = 2 + kEpiWarps;
constexpr int kThreads = 32 * (3 + kEpiWarps);
constexpr int kMaxStages = 8;
constexpr int kSlots = 2;
constexpr int kNmax = 256;
constexpr uint32_t kKHalfBytes = kKeyTile * 128;         // 128 keys x 64 bf16
constexpr uint32_t kKStageBytes = 2 * kKHalfBytes;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxAcc = 8;                               // TMEM accumulators (512 / stride)
constexpr uint32_t kDevErrInternal = 0x20u;
// The producer issues no TMA load in the test build (LI_TEST_NO_LOADS), so the MMA warp's first
// wait runs out with no bulk copy in flight (see li_sm100.cuh on the wait limit).
#ifdef LI_TEST_NO_LOADS
constexpr bool kIssueLoads = false;
#else
constexpr bool kIssueLoads = true;
#endif

struct Slot {
    int32_t valid, b, q0, nq, j0, j1, row0, L1u, L2, k_row0;
    int32_t pad[6];
    int32_t prow[32];     // paged: cache row of each of the item's first 32 key pieces
                          // (-1: past the item's keys, -2: block-table entry out of range)
    float w[kNmax];       // weights of the item's columns, even columns halved (see epilogue)
};
static_assert(sizeof(Slot) == 64 + 128 + 4 * kNmax, "Slot size");

// Shared memory: [Q buffers x2 | K stages][tail: slots, barriers, flags]. The Q buffers take
// 2 x (2 halves x N x 128 B); the K ring gets as many 32 KB stages as fit before the tail, so
// small N (decode) gets a deeper key pipeline.
constexpr uint32_t kSmemBytes = 232448;
constexpr int kNumBars = 2 * kMaxStages + 2 * 2 + 2 * kMaxAcc + 2 * kSlots;
constexpr uint32_t kTailBytes = 2816;
constexpr uint32_t kTailOff = kSmemBytes - kTailBytes;
constexpr uint32_t kSlotOff = kTailOff;
constexpr uint32_t kBarOff = kSlotOff + kSlots * sizeof(Slot);
constexpr uint32_t kFlagOff = kBarOff + 8 * kNumBars;
static_assert(kFlagOff + 16 <= kSmemBytes, "shared memory tail");
static_assert(kTailOff % 16 == 0, "tail alignment");

struct TcParams {
    Problem p;
    SchedView view;
    WsHeader *ws;
    float *scores;
    int64_t ld;
    uint32_t signature;
    int32_t N;            // MMA N
    int32_t tq;           // query rows per item
    uint32_t idesc;       // tcgen05 instruction descriptor
    int32_t piece_rows;   // paged keys: > 0, keys per TMA load (the largest power of two dividing
                          // block_size, at most 128); < 0, -(that power) below 8, the key rows
                          // copied one by one (cp.async); 0 for dense keys
    int32_t stages;       // K ring depth
    int32_t n_acc;        // TMEM accumulators in use
    uint32_t acc_stride;  // TMEM columns per accumulator (power of two >= N)
    uint32_t q_half;      // bytes of one 64-wide half of a Q buffer (N x 128)
    uint32_t k_off;       // start of the K ring (after the two Q buffers)
    Quant qd;             // fp8 q/k: the scales (null otherwise)
};

struct Bars {
    uint32_t base;
    __device__ uint32_t k_full(int s) const { return base + 8 * s; }
    __device__ uint32_t k_empty(int s) const { return base + 8 * (kMaxStages + s); }
    __device__ uint32_t q_full(int i) const { return base + 8 * (2 * kMaxStages + i); }
    __device__ uint32_t q_empty(int i) const { return base + 8 * (2 * kMaxStages + 2 + i); }
    __device__ uint32_t acc_full(int i) const { return base + 8 * (2 * kMaxStages + 4 + i); }
    __device__ uint32_t acc_empty(int i) const { return base + 8 * (2 * kMaxStages + 4 + kMaxAcc + i); }
    __device__ uint32_t sl_full(int i) const { return base + 8 * (2 * kMaxStages + 4 + 2 * kMaxAcc + i); }
    __device__ uint32_t sl_empty(int i) const {
        return base + 8 * (2 * kMaxStages + 4 + 2 * kMaxAcc + kSlots + i);
    }
};

// Position in a ring of n buffers: index and phase parity, advanced without division.
struct RingPos {
    int idx = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++idx == n) { idx = 0; phase ^= 1u; }
    }
};

__device__ __forceinline__ int32_t n_tiles_of(int32_t j0, int32_t j1) {
    return (j1 - j0 + kKeyTile - 1) / kKeyTile;
}

// Paged keys: row in the key cache of piece pi of an item whose keys start at j0 (pieces of
// piece_rows keys; j0 is a multiple of them). -1 past j1, -2 when the block-table entry is out
// of range.
__device__ __forceinline__ int32_t piece_len(const TcParams &P) {
    return P.piece_rows < 0 ? -P.piece_rows : P.piece_rows;
}
__device__ __forceinline__ int32_t piece_row(const TcParams &P, int32_t b, int32_t j0, int32_t j1,
                                             int32_t pi) {
    const int32_t jp = j0 + pi * piece_len(P);
    if (jp >= j1) return -1;
    const int32_t bs = P.p.block_size;
    const int32_t blk = P.p.block_table[(int64_t)b * P.p.bt_stride + jp / bs];
    if (blk < 0 || blk >= P.p.num_blocks) return -2;
    return blk * bs + jp % bs;
}

// ---- roles ---------------------------------------------------------------------------------
// Scheduler warp: takes tickets and stages each non-empty item (header, w, cache rows of its
// first 32 key pieces) in the slot ring ahead of the producer. The next item's loads go to
// registers right after a slot is filled, so they complete while the warp waits for the next
// free slot, and a ticket is taken only when the ring has moved on by one item.
template <int kW, bool kQ8>
__device__ void scheduler(const TcParams &P, uint8_t *smem, const Bars &bars,
                          volatile int *abort_flag, int n_items) {
    constexpr int kWPerLane = kNmax / 32;
    const int lane = threadIdx.x & 31;
    Slot *slots = reinterpret_cast<Slot *>(smem + kSlotOff);
    const int N1 = P.p.n_heads;
    WorkItem cur{};
    float wv[kWPerLane];
    int32_t tv = -1;
    bool scale_err = false;
    // takes tickets up to the next item with a non-empty window (the dense closed forms can yield
    // empty ones) and loads its weights (lane l holds entries l, l + 32, ...) and the cache row
    // of its key piece l; false at the end of the list
    auto fetch = [&]() -> bool {
        for (;;) {
            int ticket = 0;
            if (lane == 0) ticket = atomicAdd(&P.ws->sched_next, 1);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            if (ticket >= n_items) return false;
            cur = P.view.item(P.p, ticket);
            if (cur.j1 > cur.j0) break;
        }
        const int64_t wbase = (int64_t)cur.row0 * N1;
        const int nw = cur.nq * N1;
#pragma unroll
        for (int i = 0; i < kWPerLane; ++i) {
            const int e = lane + 32 * i;
            // even columns are staged halved: the epilogue takes their ReLU as x + |x|
            float we = e < nw ? weight_f32<kW>(P.p, wbase + e) : 0.0f;
            if constexpr (kQ8) {
                // a positive q scale passes through the ReLU: w ReLU(s q) = (w s) ReLU(q)
                const float sc = e < nw ? P.qd.q_descale[wbase + e] : 1.0f;
                if (!good_scale(sc)) scale_err = true;
                we *= sc;
            }
            wv[i] = (e & 1) ? we : 0.5f * we;
        }
        if (P.piece_rows) tv = piece_row(P, cur.b, cur.j0, cur.j1, lane);
        return true;
    };
    bool have = fetch();
    bool ok = true;
    for (int it = 0;; ++it) {
        const int sl = it % kSlots;
        if (!mbar_wait(bars.sl_empty(sl), ((it / kSlots) & 1) ^ 1, abort_flag)) { ok = false; break; }
        Slot &S = slots[sl];
        if (have) {
#pragma unroll
            for (int i = 0; i < kWPerLane; ++i) S.w[lane + 32 * i] = wv[i];
            if (P.piece_rows) S.prow[lane] = tv;
            if (lane == 0) {
                S.b = cur.b; S.q0 = cur.q0; S.nq = cur.nq; S.j0 = cur.j0; S.j1 = cur.j1;
                S.row0 = cur.row0; S.L1u = cur.L1u; S.L2 = cur.L2; S.k_row0 = cur.k_row0;
            }
        }
        if (lane == 0) S.valid = have ? 1 : 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.sl_full(sl));
        if (!have) break;
        have = fetch();
    }
    if (!ok) *abort_flag = 1;
    if constexpr (kQ8) {
        if (__any_sync(0xffffffffu, scale_err) && lane == 0) set_status(&P.ws->status, LI_DEVERR_DESCALE);
    }
}

// TMA producer warp: per staged item, the Q tile (double buffered) and the K tiles of its key
// range through the ring; paged keys block by block through the block table.
// kQ8: fp8 q/k, whose 128-element rows are one 128-byte box (two 64-element halves for 16-bit
// types), so a Q tile and a K stage are half as many bytes and loads.
template <bool kQ8, bool kRows>
__device__ void producer(const TcParams &P, const CUtensorMap *tmq, const CUtensorMap *tmk,
                         uint8_t *smem, const Bars &bars, volatile int *abort_flag) {
    constexpr uint32_t kStage = kQ8 ? kKHalfBytes : kKStageBytes;
    constexpr uint32_t kRowBytes = kQ8 ? 128u : 256u;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    Slot *slots = reinterpret_cast<Slot *>(smem + kSlotOff);
    const int N1 = P.p.n_heads;
    uint32_t err = 0;
    RingPos kr;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it % kSlots;
        if (!mbar_wait(bars.sl_full(sl), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const Slot &S = slots[sl];
        const int valid = S.valid;
        const int32_t b = S.b, q0 = S.q0, j0 = S.j0, j1 = S.j1, row0 = S.row0, k_row0 = S.k_row0;
        int32_t pv = S.prow[lane];          // row of piece pbase + lane
        int32_t pbase = 0;
        __syncwarp();
        if (!valid) {
            if (lane == 0) mbar_arrive(bars.sl_empty(sl));
            break;
        }
        (void)q0;
        // Q tile of the item (all heads of tq rows): two TMA loads, one per 64-wide K half.
        const int qb = it & 1;
        if (!mbar_wait(bars.q_empty(qb), ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (kIssueLoads && lane == 0 &&
            !in_bounds((qb + 1) * 2u * P.q_half <= P.k_off, &P.ws->status)) {
            mbar_arrive(bars.q_full(qb));            // bounds-checked build: skip the load
        } else if (kIssueLoads && lane == 0) {
            const uint32_t qdst = sbase + qb * 2u * P.q_half;
            const int32_t y = row0 * N1;
            if constexpr (kQ8) {
                mbar_arrive_expect_tx(bars.q_full(qb), P.q_half);
                tma_load_2d(qdst, tmq, bars.q_full(qb), 0, y);
            } else {
                mbar_arrive_expect_tx(bars.q_full(qb), 2u * P.q_half);
                tma_load_2d(qdst, tmq, bars.q_full(qb), 0, y);
                tma_load_2d(qdst + P.q_half, tmq, bars.q_full(qb), 64, y);
            }
        }
        // K tiles of the item's key range. Paged keys: lane l holds the cache row of piece
        // pbase + l (the first 32 staged by the scheduler, later ones refilled 32 at a time) and
        // lanes 0..pieces-1 each load one piece of the tile.
        const int32_t nt = n_tiles_of(j0, j1);
        const int pr = P.piece_rows;
        const int pieces = pr > 0 ? kKeyTile / pr : 0;
        int prev_st = -1;                   // row-copy mode: the stage whose arrival is pending
        for (int32_t tile = 0; tile < nt; ++tile, kr.next(P.stages)) {
            const int st = kr.idx;
            if (!mbar_wait(bars.k_empty(st), kr.phase ^ 1u, abort_flag)) { ok = false; break; }
            const int32_t jt = j0 + tile * kKeyTile;
            const uint32_t kdst = sbase + P.k_off + st * kStage;
            if (!kIssueLoads) {
                // test build: no load and no arrive; the MMA warp's wait on k_full runs out
            } else if (!in_bounds(P.k_off + (st + 1) * kStage <= kTailOff, &P.ws->status)) {
                if (lane == 0) mbar_arrive(bars.k_full(st));   // bounds-checked build: skip
            } else if constexpr (kRows) {
                // block sizes that are not a multiple of 8: the key rows are copied one by one
                // (cp.async, eight lanes per 128-byte half row) into the same 128-byte swizzled
                // layout the TMA writes; lane l copies chunk l % 8 of keys l / 8 + 4 i. Each
                // lane arrives on a stage's full barrier (32 arrivals) once its copies of that
                // stage have landed and are fenced for the tensor cores, one tile later, so two
                // tiles' copies are in flight.
                const int32_t g = -pr;
                const int kq = lane >> 3, ch = lane & 7;
                const char *kbase = reinterpret_cast<const char *>(P.p.k);
                const int64_t cache_rows = (int64_t)P.p.num_blocks * P.p.block_size;
#pragma unroll 4
                for (int i = 0; i < kKeyTile / 4; ++i) {
                    const int key = kq + 4 * i;
                    const int32_t j = jt + key;
                    int32_t row = -1;
                    if (j < j1) {
                        const int32_t q = j - j0;
                        row = piece_row(P, b, j0, j1, q / g);
                        if (row >= 0) row += q % g;
                    }
                    if (row == -2) err |= LI_DEVERR_TABLE;
                    if (row >= 0 && idx_ok(row, cache_rows, &P.ws->status)) {
                        const char *src = kbase + (int64_t)row * kRowBytes + ch * 16;
                        const uint32_t dst = kdst + (uint32_t)key * 128u + (uint32_t)((ch ^ (key & 7)) << 4);
                        cp_async16(dst, src);
                        if constexpr (!kQ8) cp_async16(dst + kKHalfBytes, src + 128);
                    }
                }
                cp_async_commit();
                if (prev_st >= 0) {
                    cp_async_wait<1>();
                    fence_async_smem();
                    mbar_arrive(bars.k_full(prev_st));
                }
                prev_st = st;
            } else if (pr == 0) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(bars.k_full(st), kStage);
                    tma_load_2d(kdst, tmk, bars.k_full(st), 0, k_row0 + jt);
                    if constexpr (!kQ8)
                        tma_load_2d(kdst + kKHalfBytes, tmk, bars.k_full(st), 64, k_row0 + jt);
                }
            } else {
                const int32_t p0 = tile * pieces;
                if (p0 + pieces > pbase + 32) {
                    pbase = p0;
                    pv = piece_row(P, b, j0, j1, pbase + lane);
                }
                const int32_t row = __shfl_sync(0xffffffffu, pv, (p0 - pbase + lane) & 31);
                const bool mine = lane < pieces && row >= 0 &&
                                  in_bounds((int64_t)row + pr <= (int64_t)P.p.num_blocks * P.p.block_size,
                                            &P.ws->status);
                const uint32_t loads = __ballot_sync(0xffffffffu, mine);
                if (__ballot_sync(0xffffffffu, lane < pieces && row == -2)) err |= LI_DEVERR_TABLE;
                if (lane == 0)
                    mbar_arrive_expect_tx(bars.k_full(st), (uint32_t)__popc(loads) * pr * kRowBytes);
                __syncwarp();
                if (mine) {
                    const uint32_t off = (uint32_t)lane * pr * 128u;
                    tma_load_2d(kdst + off, tmk, bars.k_full(st), 0, row);
                    if constexpr (!kQ8)
                        tma_load_2d(kdst + kKHalfBytes + off, tmk, bars.k_full(st), 64, row);
                }
            }
            __syncwarp();
        }
        if (kRows && prev_st >= 0) {        // row-copy mode: the item's last stage
            cp_async_wait<0>();
            fence_async_smem();
            mbar_arrive(bars.k_full(prev_st));
        }
        if (!ok) break;
        if (lane == 0) mbar_arrive(bars.sl_empty(sl));
    }
    // no copy may still be writing shared memory when the CTA leaves
    if constexpr (kRows) asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) *abort_flag = 1;
    if (lane == 0 && err) set_status(&P.ws->status, err);
}

template <bool kQ8>
__device__ void mma_issuer(const TcParams &P, uint8_t *smem, const Bars &bars,
                           volatile int *abort_flag, uint32_t tmem_base) {
    constexpr uint32_t kStage = kQ8 ? kKHalfBytes : kKStageBytes;
    const uint32_t sbase = smem_u32(smem);
    Slot *slots = reinterpret_cast<Slot *>(smem + kSlotOff);
    RingPos kr, ar;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int sl = it % kSlots;
        if (!mbar_wait(bars.sl_full(sl), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const Slot &S = slots[sl];
        const int valid = S.valid;
        const int32_t j0 = S.j0, j1 = S.j1;
        mbar_arrive(bars.sl_empty(sl));
        if (!valid) break;
        const int qb = it & 1;
        if (!mbar_wait(bars.q_full(qb), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const uint32_t qsm = sbase + qb * 2u * P.q_half;
        const uint64_t b0 = sw128_desc(qsm);
        const uint64_t b_half16 = P.q_half >> 4;
        const int32_t nt = n_tiles_of(j0, j1);
        for (int32_t tile = 0; tile < nt; ++tile, kr.next(P.stages), ar.next(P.n_acc)) {
            const int st = kr.idx;
            const int ab = ar.idx;
            if (!mbar_wait(bars.k_full(st), kr.phase, abort_flag)) { ok = false; break; }
            if (!mbar_wait(bars.acc_empty(ab), ar.phase ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            // descriptors advance by the byte offset / 16 in their address field (no carry:
            // shared addresses stay below 2^18 bytes)
            const uint64_t a0 = sw128_desc(sbase + P.k_off + st * kStage);
            const uint32_t d = tmem_base + ab * P.acc_stride;
            if constexpr (kQ8) {
                // one 128-byte row holds all 128 elements: four K = 32 steps of 32 bytes
                umma_f8_c<false>(d, a0, b0, P.idesc);
#pragma unroll
                for (int kk = 1; kk < kHeadDim / 32; ++kk)
                    umma_f8_c<true>(d, a0 + 2 * kk, b0 + 2 * kk, P.idesc);
            } else {
                umma_bf16_c<false>(d, a0, b0, P.idesc);
#pragma unroll
                for (int kk = 1; kk < kHeadDim / 16; ++kk) {
                    const uint64_t a_off = ((kk >> 2) * kKHalfBytes + (kk & 3) * 32u) >> 4;
                    const uint64_t b_off = ((uint64_t)(kk >> 2) * b_half16) + (uint64_t)((kk & 3) * 2);
                    umma_bf16_c<true>(d, a0 + a_off, b0 + b_off, P.idesc);
                }
            }
            umma_commit(bars.k_empty(st));
            umma_commit(bars.acc_full(ab));
        }
        if (!ok) break;
        umma_commit(bars.q_empty(qb));
    }
    if (!ok) *abort_flag = 1;
}

// Score of one key for one query row from its 64 head columns v (N1 = 64) and the row's staged
// weights w: the sum over heads of w * ReLU(v). Even heads take the ReLU on the FMA pipe as
// x + |x| = 2 max(x, 0) with a halved weight ((w/2)(2x) = w x exactly, so each FMA rounds the same
// value); odd heads take max(x, 0) on the ALU pipe. The four partial sums (heads = 0, 1, 2, 3
// mod 4) are two packed pairs; a packed FMA is two round-to-nearest fp32 FMAs.
__device__ __forceinline__ float head_sum64(const float (&v)[64], const float *w) {
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
    float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
    for (int h4 = 0; h4 < 16; ++h4) {
        const float4 ww = w4[h4];
        const float x0 = v[4 * h4 + 0], x2 = v[4 * h4 + 2];
        a01 = __ffma2_rn(make_float2(ww.x, ww.y),
                         make_float2(x0 + fabsf(x0), fmaxf(v[4 * h4 + 1], 0.f)), a01);
        a23 = __ffma2_rn(make_float2(ww.z, ww.w),
                         make_float2(x2 + fabsf(x2), fmaxf(v[4 * h4 + 3], 0.f)), a23);
    }
    return (a01.x + a01.y) + (a23.x + a23.y);
}

// The same sum with the 64 columns read from TMEM in two halves of 32: fewer live registers,
// the same additions in the same order. The fp8 instantiations take it (with one 64-column
// load their key-scale registers spill at the kernel's 96-register budget); the 16-bit ones
// keep the single load, which measures faster there.
__device__ __forceinline__ float head_sum64_tmem(uint32_t taddr, const float *w) {
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
    float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(taddr + 32u * half, v);
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
            const float4 ww = w4[8 * half + h4];
            const float x0 = v[4 * h4 + 0], x2 = v[4 * h4 + 2];
            a01 = __ffma2_rn(make_float2(ww.x, ww.y),
                             make_float2(x0 + fabsf(x0), fmaxf(v[4 * h4 + 1], 0.f)), a01);
            a23 = __ffma2_rn(make_float2(ww.z, ww.w),
                             make_float2(x2 + fabsf(x2), fmaxf(v[4 * h4 + 3], 0.f)), a23);
        }
    }
    return (a01.x + a01.y) + (a23.x + a23.y);
}

// The same sum for any N1: row t's columns [t*N1, (t+1)*N1) of the accumulator at acc, read 16
// columns at a time; even columns carry halved weights.
__device__ __forceinline__ float head_sum(uint32_t acc, const float *w, int t, int N1) {
    const int c_lo = t * N1, c_hi = c_lo + N1;
    float a = 0.f;
    for (int ch = c_lo & ~15; ch < c_hi; ch += 16) {
        float v[16];
        tmem_ld16(acc + ch, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = ch + i;
            if (c >= c_lo && c < c_hi)
                a = fmaf(w[c], (c & 1) ? fmaxf(v[i], 0.f) : v[i] + fabsf(v[i]), a);
        }
    }
    return a;
}

// kQ8: fp8 q/k. The q scales were folded into the staged weights; a key's positive scale passes
// through the ReLU of every head, so each key's sum is multiplied by its k scale.
template <bool kQ8>
__device__ void epilogue(const TcParams &P, uint8_t *smem, const Bars &bars,
                         volatile int *abort_flag, uint32_t tmem_base) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int group = (warp - 2) >> 2;     // which rows of the item: t = group (mod kEpiGroups)
    Slot *slots = reinterpret_cast<Slot *>(smem + kSlotOff);
    const int N1 = P.p.n_heads;
    const int mask_mode = P.p.mask_mode;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    RingPos ar;
    bool ok = true;
    bool scale_err = false;
    for (int it = 0; ok; ++it) {
        const int sl = it % kSlots;
        if (!mbar_wait(bars.sl_full(sl), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const Slot &S = slots[sl];
        const int valid = S.valid;
        if (!valid) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.sl_empty(sl));
            break;
        }
        const int32_t q0 = S.q0, nq = S.nq, j0 = S.j0, j1 = S.j1, row0 = S.row0, L1u = S.L1u,
                      L2 = S.L2;
        const int32_t nt = n_tiles_of(j0, j1);
        // At most one row per warp group (N1 >= 64): the row, its window end and its output
        // row are fixed for the whole item.
        const bool one_row = nq <= kEpiGroups;
        const int32_t hi1 = one_row && group < nq ? min(window_hi(mask_mode, q0 + group, L1u, L2), j1) : 0;
        float *const out1 = P.scores + (int64_t)(row0 + (one_row && group < nq ? group : 0)) * P.ld;
        // fp8: this thread's key scale of tile t (-1 row: none), loaded kKdAhead tiles early and
        // carried in registers so the load is in flight while earlier tiles are summed; paged
        // rows come from the rows the scheduler staged
        constexpr int kKdAhead = 3;
        auto kd_load = [&](int32_t t, bool &has) -> float {
            has = false;
            const int32_t jj = j0 + t * kKeyTile + 32 * quarter + lane;
            if (t >= nt || jj >= j1) return 0.0f;
            int64_t kr = (int64_t)S.k_row0 + jj;
            if (P.piece_rows) {
                const int32_t pl = piece_len(P);
                const int32_t pc = (jj - j0) / pl;
                int32_t prow = pc < 32 ? S.prow[pc] : -1;
                if (pc >= 32) {
                    const int32_t bs = P.p.block_size;
                    const int32_t blk = P.p.block_table[(int64_t)S.b * P.p.bt_stride + jj / bs];
                    prow = blk >= 0 && blk < P.p.num_blocks ? blk * bs + (jj - jj % pl) % bs
                                                            : -2;
                }
                if (prow < 0) return 0.0f;
                kr = (int64_t)prow + (jj - j0) % pl;
            }
            has = true;
            return __ldg(P.qd.k_descale + kr);
        };
        float kq0 = 0.f, kq1 = 0.f, kq2 = 0.f;
        bool hq0 = false, hq1 = false, hq2 = false;
        if constexpr (kQ8) {
            static_assert(kKdAhead == 3, "three scales in flight");
            kq0 = kd_load(0, hq0);
            kq1 = kd_load(1, hq1);
            kq2 = kd_load(2, hq2);
        }
        for (int32_t tile = 0; tile < nt; ++tile, ar.next(P.n_acc)) {
            const int ab = ar.idx;
            const int32_t jt = j0 + tile * kKeyTile;
            const int32_t j = jt + 32 * quarter + lane;
            float kd = 1.0f;
            if constexpr (kQ8) {
                bool hn = false;
                const float kn = kd_load(tile + kKdAhead, hn);
                kd = kq0;
                if (hq0 && !good_scale(kd)) scale_err = true;
                kq0 = kq1; hq0 = hq1;
                kq1 = kq2; hq1 = hq2;
                kq2 = kn; hq2 = hn;
            }
            if (!mbar_wait(bars.acc_full(ab), ar.phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t acc = tmem_base + lane_addr + ab * P.acc_stride;
            if (one_row) {
                if (N1 == 64 && jt < hi1) {
                    float I;
                    if constexpr (kQ8) {
                        I = head_sum64_tmem(acc + group * 64, S.w + group * 64);
                    } else {
                        float v[64];
                        tmem_ld64(acc + group * 64, v);
                        I = head_sum64(v, S.w + group * 64);
                    }
                    if constexpr (kQ8) I *= kd;
                    if (j < hi1 && in_bounds(row0 + group < P.p.rows && j < P.ld, &P.ws->status))
                        out1[j] = I;
                } else if (jt < hi1) {
                    float I = head_sum(acc, S.w, group, N1);
                    if constexpr (kQ8) I *= kd;
                    if (j < hi1 && in_bounds(row0 + group < P.p.rows && j < P.ld, &P.ws->status))
                        out1[j] = I;
                }
            } else {
                for (int t = group; t < nq; t += kEpiGroups) {
                    const int32_t hi = min(window_hi(mask_mode, q0 + t, L1u, L2), j1);
                    if (jt >= hi) continue;                       // tile past this row's window
                    float I;
                    if (N1 == 64) {
                        if constexpr (kQ8) {
                            I = head_sum64_tmem(acc + t * 64, S.w + t * 64);
                        } else {
                            float v[64];
                            tmem_ld64(acc + t * 64, v);
                            I = head_sum64(v, S.w + t * 64);
                        }
                    } else {
                        I = head_sum(acc, S.w, t, N1);
                    }
                    if constexpr (kQ8) I *= kd;
                    if (j < hi && in_bounds(row0 + t < P.p.rows && j < P.ld, &P.ws->status))
                        P.scores[(int64_t)(row0 + t) * P.ld + j] = I;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.acc_empty(ab));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.sl_empty(sl));
    }
    if (!ok) *abort_flag = 1;
    if constexpr (kQ8) {
        if (__any_sync(0xffffffffu, scale_err) && lane == 0) set_status(&P.ws->status, LI_DEVERR_DESCALE);
    }
}

// kW: li_dtype of w (the weights are staged as fp32; q and k go to the MMA as they are);
// kQ8: fp8 q/k with scales.
template <int kW, bool kQ8, bool kRows>
__global__ void __launch_bounds__(kThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const TcParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {                              // the swizzled tiles need 1 KB alignment
        if (threadIdx.x == 0) set_status(&P.ws->status, kDevErrInternal);
        return;
    }
    int n_items = P.view.n_items;
    if (P.view.meta) {
        const MetaHeader *hdr = reinterpret_cast<const MetaHeader *>(P.view.meta);
        if (hdr->magic != kMetaMagic || hdr->signature != P.signature) {
            if (threadIdx.x == 0 && blockIdx.x == 0) set_status(&P.ws->status, kDevErrMetadata);
            return;
        }
        n_items = hdr->n_items;
    }

    Bars bars{sbase + kBarOff};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kFlagOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kFlagOff + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(bars.k_full(s), kRows ? 32 : 1);   // row copies: one arrival per lane
            mbar_init(bars.k_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.q_full(i), 1);
            mbar_init(bars.q_empty(i), 1);
        }
        for (int i = 0; i < kMaxAcc; ++i) {
            mbar_init(bars.acc_full(i), 1);
            mbar_init(bars.acc_empty(i), kEpiWarps);
        }
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(bars.sl_full(i), 1);
            mbar_init(bars.sl_empty(i), 2 + kEpiWarps);   // producer, MMA, epilogue warps
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        producer<kQ8, kRows>(P, &tmap_q, &tmap_k, smem, bars, abort_flag);
    } else if (warp == kSchedWarp) {
        if (blockIdx.x == 0) check_batch_keys(P.p, P.view, &P.ws->status, lane, 32);
        scheduler<kW, kQ8>(P, smem, bars, abort_flag, n_items);
    } else if (warp == 1) {
        if (lane == 0) mma_issuer<kQ8>(P, smem, bars, abort_flag, tmem_base);
        __syncwarp();
    } else {
        epilogue<kQ8>(P, smem, bars, abort_flag, tmem_base);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(&P.ws->status, LI_DEVERR_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---- host ----------------------------------------------------------------------------------
// Rows of 128 elements; 16-bit types are loaded as two 64-element (128-byte) boxes, fp8 as one.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint32_t box_rows, int dtype) {
    auto fn = encode_fn();
    if (!fn || rows == 0) return false;
    const bool b8 = dtype == LI_DTYPE_FP8_E4M3;
    cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * (b8 ? 1 : 2)};
    cuuint32_t box[2] = {b8 ? 128u : 64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType t = b8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                  : dtype == LI_DTYPE_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = fn(m, t, 2, const_cast<void *>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

// Shape checks of the tensor-core kernel: MMA width 16..256, at least two key stages in shared
// memory and 16-byte aligned q and k for the tensor maps. Every paged block size is taken: TMA
// pieces of the largest power of two dividing it (capped at 128) when that is 8 or more, row
// copies otherwise.
bool score_tc_eligible(const Problem &p, const Schedule &s) {
    if (s.max_items <= 0 || p.rows <= 0) return false;
    const int N = (s.tq * p.n_heads + 15) / 16 * 16;
    if (N > kNmax || N < 16) return false;
    if ((kTailOff - 4u * (uint32_t)N * 128u) / kKStageBytes < 2) return false;
    return (reinterpret_cast<uintptr_t>(p.q) & 15) == 0 && (reinterpret_cast<uintptr_t>(p.k) & 15) == 0;
}

// Launches the tensor-core kernel when the problem fits it; *launched = false leaves the call
// to the CUDA-core kernel (see score_tc_eligible, and a tensor map the driver refuses).
cudaError_t launch_score_tc(const Problem &p, const Quant &qd, const Schedule &s, const void *meta,
                            WsHeader *ws, float *scores, int64_t ld, cudaStream_t st,
                            bool *launched) {
    *launched = false;
    if (!score_tc_eligible(p, s)) return cudaSuccess;
    TcParams P{};
    P.p = p;
    P.view = make_view(p, s, meta);
    P.ws = ws;
    P.scores = scores;
    P.ld = ld;
    P.signature = problem_signature(p, s.tq, s.kc);
    P.tq = s.tq;
    P.N = (s.tq * p.n_heads + 15) / 16 * 16;
    if (P.N > kNmax || P.N < 16) return cudaSuccess;
    const bool q8 = p.dtype_qk == LI_DTYPE_FP8_E4M3;
    P.qd = qd;
    // D fp32; A and B both bf16 (format 1) or both fp16 (format 0) for kind::f16, both E4M3
    // (format 0) for kind::f8f6f4; N, M
    const uint32_t ab_format = p.dtype_qk == LI_DTYPE_BF16 ? 1u : 0u;
    P.idesc = (1u << 4) | (ab_format << 7) | (ab_format << 10) | ((uint32_t)(P.N >> 3) << 17) |
              ((uint32_t)(128 >> 4) << 24);
    P.q_half = (uint32_t)P.N * 128u;               // N is a multiple of 16: 1 KB aligned halves
    P.k_off = 4u * P.q_half;
    P.acc_stride = 32;
    while (P.acc_stride < (uint32_t)P.N) P.acc_stride <<= 1;
    P.n_acc = (int)(kTmemCols / P.acc_stride);
    if (P.n_acc > kMaxAcc) P.n_acc = kMaxAcc;
    P.stages = (int)((kTailOff - P.k_off) / (q8 ? kKHalfBytes : kKStageBytes));
    if (P.stages > kMaxStages) P.stages = kMaxStages;
    if (P.stages < 2) return cudaSuccess;
    uint64_t k_rows = 0;
    if (p.layout_k == LI_LAYOUT_PA_BSND) {
        // pieces: the largest power of two dividing the block size, at most a tile; each piece
        // lies inside one block and one tile. TMA loads pieces of 8 rows or more (whole
        // 1024-byte swizzle atoms); smaller ones are copied row by row.
        const int bs = p.block_size;
        const int low = bs & -bs;
        const int piece = low < kKeyTile ? low : kKeyTile;
        P.piece_rows = piece >= 8 ? piece : -piece;
        k_rows = (uint64_t)p.num_blocks * bs;
    } else {
        P.piece_rows = 0;
        k_rows = p.layout_k == LI_LAYOUT_TND ? (uint64_t)p.k_len : (uint64_t)p.batch * p.k_len;
    }
    const uint64_t q_rows = (uint64_t)(p.layout_q == LI_LAYOUT_TND ? p.q_len : p.batch * p.q_len) *
                            p.n_heads;
    CUtensorMap mq, mk;
    if (!make_map(&mq, p.q, q_rows, (uint32_t)P.N, p.dtype_qk)) return cudaSuccess;
    if (!make_map(&mk, p.k, k_rows,
                  P.piece_rows > 0 ? (uint32_t)P.piece_rows : P.piece_rows < 0 ? 1u : (uint32_t)kKeyTile,
                  p.dtype_qk))
        return cudaSuccess;
    // row-copy mode (block sizes that are not a multiple of 8) has instantiations of its own,
    // so the TMA kernels' code is unchanged by it
    const bool rows = P.piece_rows < 0;
    auto pick = [&](auto q8c, auto rowsc) {
        constexpr bool Q8 = decltype(q8c)::value, R = decltype(rowsc)::value;
        return p.dtype_w == LI_DTYPE_FP32   ? score_tc_kernel<LI_DTYPE_FP32, Q8, R>
             : p.dtype_w == LI_DTYPE_FP16 ? score_tc_kernel<LI_DTYPE_FP16, Q8, R>
                                          : score_tc_kernel<LI_DTYPE_BF16, Q8, R>;
    };
    using T = std::true_type;
    using F = std::false_type;
    auto kern = q8 ? (rows ? pick(T{}, T{}) : pick(T{}, F{})) : (rows ? pick(F{}, T{}) : pick(F{}, F{}));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    int grid = device_sm_count();
    if (s.max_items < grid) grid = s.max_items;
    kern<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, P);
    e = cudaGetLastError();
    if (e == cudaSuccess) *launched = true;
    return e;
}

}  // namespace li
