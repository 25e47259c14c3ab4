// The indexer's backward with the KL loss (torch_npu.npu_sparse_lightning_indexer_grad_kl_loss,
// formulas 1-4) on the tensor cores (tcgen05 + TMEM), sm_100a. For query row r and its selected
// keys s (64 per tile):
//   pass 1, per tile   S_main[s, g] = q[r, g] . k[s] (+ rope)          (keys on M = 64, heads on N)
//                      S~[s, h]     = qi[r, h] . ki[s]                 (keys on M = 64, heads on N)
//                      p^[s] = sum_g exp(scale S_main - softmax_max_g) / softmax_sum_g,
//                      I[s]  = sum_h w_h ReLU(S~[s, h])                 (kept in shared memory)
//   row statistics     p = p^ / sum p^, softmax(I), loss = sum_s p log(p / softmax(I)) with
//                      0 log 0 = 0, dI = softmax(I) - p                 (fixed-order reductions)
//   pass 2, per tile   S~ again; dS[s, h] = dI[s] w_h [S~ > 0] as bf16 hi + lo (the pair carries
//                      16 significant bits); d_w[h] += sum_s dI[s] ReLU(S~[s, h]);
//                      d_qi[h, :] += sum_s dS[s, h] ki[s, :]            (heads on M = 64, dims
//                                                                         on N = 128, keys on K)
//                      dK[s, :]    = sum_h dS[s, h] qi[r, h, :]         (keys on M = 64, dims on
//                                                                         N = 128, heads on K)
// One CTA per SM owns the rows r = c, c + C, c + 2 C, ... (C = the grid). Its dK rows are added,
// in its row order, into its own slice c of a partial buffer [C][key rows][128]; a second kernel
// sums the C slices of every key in slice order, so d_key_index is bit-reproducible (no atomics).
//
// Warp roles: 0-7 epilogue (thread = key or head of the M = 64 TMEM layouts: lanes 0-15 of each
// quarter; warps q and q + 4 share quarter q and split each key's heads and dK dims in halves),
// 8 MMA (and TMEM), 9 scheduler (row slots, Q tiles by TMA), 10-13 gather (cp.async of the
// selected key rows into 128-byte swizzled 64-dim chunks). Every wait is bounded in time.
#include <cuda_bf16.h>

#include <type_traits>

#include "li_internal.cuh"
#include "li_kl.cuh"
#include "li_sm100.cuh"

namespace li {
namespace {

using namespace sm100;

constexpr int kKeys = 64;
constexpr uint32_t kChunk = kKeys * 128;            // 64 keys x 64 dims bf16: 8 KB
constexpr int kDi = 128;
constexpr int kEpiWarps = 8, kMmaWarp = 8, kSchedWarp = 9, kGatherWarp0 = 10, kGatherWarps = 4;
constexpr int kThreads = 32 * 14;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr uint32_t kSmemBytes = 232448;
constexpr int kMaxMainSlots = 16, kMaxKiSlots = 4, kTileRing = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// TMEM columns: S_main (<= 32), S~ (<= 64), d_qi (128, heads on lanes), dK (128, keys on lanes)
constexpr uint32_t kColSm = 0, kColSi = 32, kColDq = 96, kColDk = 224, kTmemCols = 512;

struct RowSlot {
    int32_t row, tiles, pad0, pad1;
    int64_t key_base;
    int64_t pad2;
};

struct Bars {
    uint32_t base;
    __device__ uint32_t at(int i) const { return base + 8 * i; }
    __device__ uint32_t rs_full(int i) const { return at(0 + i); }
    __device__ uint32_t rs_empty(int i) const { return at(2 + i); }
    __device__ uint32_t q_full() const { return at(4); }
    __device__ uint32_t q_empty() const { return at(5); }
    __device__ uint32_t s_full() const { return at(6); }
    __device__ uint32_t s_empty() const { return at(7); }
    __device__ uint32_t ds_full() const { return at(8); }
    __device__ uint32_t ds_empty() const { return at(9); }
    __device__ uint32_t dk_full() const { return at(10); }
    __device__ uint32_t dk_empty() const { return at(11); }
    __device__ uint32_t dq_full() const { return at(12); }
    __device__ uint32_t dq_empty() const { return at(13); }
    __device__ uint32_t xch(int i) const { return at(14 + i); }
    __device__ uint32_t tile_full(int i) const { return at(16 + i); }
    __device__ uint32_t ki_empty(int i) const { return at(16 + kTileRing + i); }
    __device__ uint32_t main_empty(int i) const { return at(16 + kTileRing + kMaxKiSlots + i); }
};
constexpr int kNumBars = 16 + kTileRing + kMaxKiSlots + kMaxMainSlots;
// tail: barriers | row slots | scalar exchange [2][8 warps] | d_w sums [64][4] | w, max, sum of
// the row [64 + 32 + 32] | TMEM slot, abort flag
constexpr uint32_t kTailBytes = 4096;
constexpr uint32_t kTailOff = kSmemBytes - kTailBytes;
constexpr uint32_t kRowSlotOff = kTailOff + 8 * kNumBars;
constexpr uint32_t kXchOff = (kRowSlotOff + 2 * sizeof(RowSlot) + 15) / 16 * 16;
constexpr uint32_t kDwOff = kXchOff + 2 * kEpiWarps * 4;
constexpr uint32_t kRowDataOff = kDwOff + 64 * 4 * 4;
constexpr uint32_t kFlagOff = kRowDataOff + (64 + 32 + 32) * 4;
static_assert(kFlagOff + 16 <= kSmemBytes, "shared memory tail");
static_assert(kTailOff % 1024 == 0, "tail alignment");

struct KlTcParams {
    const uint16_t *k, *k_rope, *ki, *w;
    const int32_t *indices;
    const float *smax, *ssum;
    float *row_loss, *d_qi, *d_w, *d_part;
    uint32_t *status;
    float scale;
    int32_t rows, s1, s2, G, Ng, Dm, Dr, H, Nh, topk, nmc, chunks;
    int64_t key_rows;                    // B * S2: rows of one slice of d_part
    uint32_t qm_off, qi_off, ds_off, parr_off, iarr_off, main_off, ki_off;
    int32_t main_slots, ki_slots;
    uint32_t idesc_sm, idesc_si, idesc_dq, idesc_dk;
};

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
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

// The CTA's k-th row (k >= 0), or -1 past its last.
__device__ __forceinline__ int cta_row(const KlTcParams &P, int k) {
    const int64_t r = (int64_t)blockIdx.x + (int64_t)k * P.chunks;
    return r < P.rows ? (int)r : -1;
}

// ---- scheduler: row slots and the row's Q tiles ---------------------------------------------
__device__ void scheduler_role(const KlTcParams &P, const CUtensorMap *tmq, const CUtensorMap *tmr,
                               const CUtensorMap *tmi, uint8_t *smem, const Bars &bars,
                               volatile int *abort_flag) {
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    RowSlot *slots = reinterpret_cast<RowSlot *>(smem + kRowSlotOff);
    const int nmain = P.Dm / 64;
    uint32_t qph = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
        const int row = cta_row(P, it);
        int last = -1;
        if (row >= 0) {
            const int32_t *ir = P.indices + (int64_t)row * P.topk;
#pragma unroll 4
            for (int pos = lane; pos < P.topk; pos += 32)
                if (__ldg(ir + pos) >= 0) last = pos;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        }
        const int tiles = (last + 1 + kKeys - 1) / kKeys;
        const int sl = it & 1;
        if (!wait_warp(bars.rs_empty(sl), ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (lane == 0) {
            RowSlot &S = slots[sl];
            S.row = row;
            S.tiles = tiles;
            S.key_base = row >= 0 ? (int64_t)(row / P.s1) * P.s2 : 0;
            mbar_arrive(bars.rs_full(sl));
        }
        __syncwarp();
        if (row < 0) break;
        if (tiles == 0) continue;
        if (!wait_warp(bars.q_empty(), qph ^ 1u, abort_flag)) { ok = false; break; }
        if (lane == 0) {
            const uint32_t cbm = (uint32_t)P.Ng * 128u, cbi = (uint32_t)P.Nh * 128u;
            mbar_arrive_expect_tx(bars.q_full(), (uint32_t)(P.nmc * P.G + 2 * P.H) * 128u);
            for (int c = 0; c < nmain; ++c)
                tma_load_2d(sbase + P.qm_off + c * cbm, tmq, bars.q_full(), 64 * c, row * P.G);
            if (P.Dr > 0)
                tma_load_2d(sbase + P.qm_off + nmain * cbm, tmr, bars.q_full(), 0, row * P.G);
            for (int c = 0; c < 2; ++c)
                tma_load_2d(sbase + P.qi_off + c * cbi, tmi, bars.q_full(), 64 * c, row * P.H);
        }
        __syncwarp();
        qph ^= 1u;
    }
    if (!ok) *abort_flag = 1;
}

// ---- gather: pass 1 tiles (main key chunks + indexer key pair), pass 2 tiles (pair only) -------
__device__ void gather_role(const KlTcParams &P, uint8_t *smem, const Bars &bars,
                            volatile int *abort_flag) {
    const int t = threadIdx.x - 32 * kGatherWarp0;
    const int lane = t & 31;
    const int key0 = t >> 3, piece = t & 7;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t swz = (uint32_t)((piece ^ (key0 & 7)) << 4);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const int nmain = P.Dm / 64;
    Ring mr, kr, tr;
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
        for (int pass = 0; pass < 2 && ok; ++pass) {
            for (int j = 0; j < tiles && ok; ++j, tr.next(kTileRing)) {
                int64_t kr_[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pos = kKeys * j + key0 + 16 * i;
                    const int32_t v = pos < P.topk ? __ldg(ir + pos) : -1;
                    if (pass == 0 && v >= P.s2) err |= LI_DEVERR_LENGTHS;
                    kr_[i] = key_base + (v >= 0 && v < P.s2 ? v : 0);
                    if (!idx_ok(kr_[i], P.key_rows, P.status)) kr_[i] = 0;
                }
                if (pass == 0) {
                    for (int c = 0; c < P.nmc; ++c, mr.next(P.main_slots)) {
                        if (!wait_warp(bars.main_empty(mr.idx), mr.phase ^ 1u, abort_flag)) { ok = false; break; }
                        const uint32_t base = sbase + P.main_off + mr.idx * kChunk + key0 * 128u + swz;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint16_t *src = c < nmain ? P.k + kr_[i] * P.Dm + 64 * c + 8 * piece
                                                            : P.k_rope + kr_[i] * P.Dr + 8 * piece;
                            cp_async16(base + i * 16u * 128u, src);
                        }
                    }
                    if (!ok) break;
                }
                if (!wait_warp(bars.ki_empty(kr.idx), kr.phase ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t base = sbase + P.ki_off + kr.idx * 2u * kChunk + key0 * 128u + swz;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        cp_async16(base + h * kChunk + i * 16u * 128u,
                                   P.ki + kr_[i] * kDi + 64 * h + 8 * piece);
                kr.next(P.ki_slots);
                cp_async_arrive(bars.tile_full(tr.idx));
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) *abort_flag = 1;
    if (err) atomicOr(P.status, err);
}

// ---- MMA issuer --------------------------------------------------------------------------------
__device__ void mma_role(const KlTcParams &P, uint8_t *smem, const Bars &bars,
                         volatile int *abort_flag, uint32_t tmem) {
    const uint32_t sbase = smem_u32(smem);
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const uint32_t cbm = (uint32_t)P.Ng * 128u, cbi = (uint32_t)P.Nh * 128u;
    const int nmain = P.Dm / 64;
    Ring mr, kr, tr;
    uint32_t qph = 0, sph = 0, dsph = 0, dkph = 0, nrow_dq = 0;
    bool ok = true;
    // S~ of the tile whose indexer keys sit in pair slot ki
    auto indexer_scores = [&](uint32_t ki_addr) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint64_t a = sw128_desc(ki_addr + h * kChunk);
            const uint64_t b = sw128_desc(sbase + P.qi_off + h * cbi);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + kColSi, a + 2 * kk, b + 2 * kk, P.idesc_si, (h | kk) != 0);
        }
    };
    for (int it = 0; ok; ++it) {
        const int sl = it & 1;
        if (!wait_(bars.rs_full(sl), (it >> 1) & 1, abort_flag)) { ok = false; break; }
        const int row = slots[sl].row, tiles = slots[sl].tiles;
        mbar_arrive(bars.rs_empty(sl));
        if (row < 0) break;
        if (tiles == 0) continue;
        if (!wait_(bars.q_full(), qph, abort_flag)) { ok = false; break; }
        qph ^= 1u;
        tc_fence_after();
        // pass 1: S_main and S~ per tile
        for (int j = 0; j < tiles && ok; ++j, tr.next(kTileRing)) {
            if (!wait_(bars.s_empty(), sph ^ 1u, abort_flag)) { ok = false; break; }
            if (!wait_(bars.tile_full(tr.idx), tr.phase, abort_flag)) { ok = false; break; }
            fence_async_smem();                  // the gathered rows, for the async proxy
            tc_fence_after();
            for (int c = 0; c < P.nmc; ++c, mr.next(P.main_slots)) {
                const uint64_t a = sw128_desc(sbase + P.main_off + mr.idx * kChunk);
                const uint64_t b = sw128_desc(sbase + P.qm_off + c * cbm);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + kColSm, a + 2 * kk, b + 2 * kk, P.idesc_sm, (c | kk) != 0);
                umma_commit(bars.main_empty(mr.idx));
            }
            indexer_scores(sbase + P.ki_off + kr.idx * 2u * kChunk);
            umma_commit(bars.ki_empty(kr.idx));
            kr.next(P.ki_slots);
            umma_commit(bars.s_full());
            sph ^= 1u;
        }
        if (!ok) break;
        (void)nmain;
        // pass 2: S~ again, then d_qi += dS^T-products and dK per tile
        for (int j = 0; j < tiles && ok; ++j, tr.next(kTileRing)) {
            if (!wait_(bars.s_empty(), sph ^ 1u, abort_flag)) { ok = false; break; }
            if (!wait_(bars.tile_full(tr.idx), tr.phase, abort_flag)) { ok = false; break; }
            fence_async_smem();                  // the gathered rows, for the async proxy
            tc_fence_after();
            const uint32_t ki_addr = sbase + P.ki_off + kr.idx * 2u * kChunk;
            indexer_scores(ki_addr);
            umma_commit(bars.s_full());
            sph ^= 1u;
            // dS of this tile written; the previous tile's dK read out; d_qi of the previous row
            // read out (first tile of the row)
            if (!wait_(bars.ds_full(), dsph, abort_flag)) { ok = false; break; }
            dsph ^= 1u;
            if (!wait_(bars.dk_empty(), dkph ^ 1u, abort_flag)) { ok = false; break; }
            if (j == 0 && nrow_dq > 0 && !wait_(bars.dq_empty(), (nrow_dq - 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {           // dS hi, then lo
                const uint32_t ds = sbase + P.ds_off + part * kChunk;
                // d_qi[h, d] += sum_s dS[s, h] ki[s, d]: A = dS read MN-major (heads on M),
                // B = the key pair read MN-major (dims on N, two 64-dim blocks 8 KB apart)
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint64_t a = sw128_desc_mn(ds + kk * 2048u, 0);
                    const uint64_t b = sw128_desc_mn(ki_addr + kk * 2048u, kChunk);
                    umma_f16(tmem + kColDq, a, b, P.idesc_dq, (j > 0 || part > 0 || kk > 0) ? 1u : 0u);
                }
                // dK[s, d] = sum_h dS[s, h] qi[h, d]: A = dS K-major (keys on M), B = the qi tile
                // read MN-major (dims on N, two blocks one qi chunk apart; heads on K)
                for (int kk = 0; kk < P.Nh / 16; ++kk) {
                    const uint64_t a = sw128_desc(ds) + 2 * kk;
                    const uint64_t b = sw128_desc_mn(sbase + P.qi_off + kk * 2048u, cbi);
                    umma_f16(tmem + kColDk, a, b, P.idesc_dk, (part > 0 || kk > 0) ? 1u : 0u);
                }
            }
            umma_commit(bars.ki_empty(kr.idx));
            kr.next(P.ki_slots);
            umma_commit(bars.ds_empty());
            umma_commit(bars.dk_full());
            dkph ^= 1u;
        }
        if (!ok) break;
        umma_commit(bars.dq_full());
        umma_commit(bars.q_empty());
        ++nrow_dq;
    }
    if (!ok) *abort_flag = 1;
}

// ---- epilogue --------------------------------------------------------------------------------
// Sum (or max) of one value per epilogue thread, the same result in every thread, in a fixed
// order: warp shuffles, then the four warps' partials in warp order. `use` counts the calls
// (alternating buffers and barrier phases).
__device__ __forceinline__ bool epi_reduce(float &v, bool is_max, uint32_t &use, uint8_t *smem,
                                           const Bars &bars, volatile int *abort_flag) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, x) : v + x;
    }
    float *xb = reinterpret_cast<float *>(smem + kXchOff) + (use & 1) * kEpiWarps;
    if (lane == 0) xb[warp] = v;
    mbar_arrive(bars.xch(use & 1));
    const bool ok = wait_warp(bars.xch(use & 1), (use >> 1) & 1u, abort_flag);
    static_assert(kEpiWarps == 8, "eight partials");
    v = is_max ? fmaxf(fmaxf(fmaxf(xb[0], xb[1]), fmaxf(xb[2], xb[3])),
                       fmaxf(fmaxf(xb[4], xb[5]), fmaxf(xb[6], xb[7])))
               : ((xb[0] + xb[1]) + (xb[2] + xb[3])) + ((xb[4] + xb[5]) + (xb[6] + xb[7]));
    ++use;
    return ok;
}

__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

template <int NG>
__device__ void epilogue_role(const KlTcParams &P, uint8_t *smem, const Bars &bars,
                              volatile int *abort_flag, uint32_t tmem) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tid = threadIdx.x;                          // 0..kEpiThreads-1
    const int q = warp & 3;                               // TMEM lane quarter
    const int hf = warp >> 2;                             // half: heads (and dK dims) of the key
    const bool kl = lane < 16;                            // lanes holding a key (or head) row
    const int key = 16 * q + (lane & 15);                 // key of the tile / head of d_qi
    // the 16-lane TMEM loads spread a quarter's 16 keys over the whole warp: lane pair
    // (t, t ^ 2) shares key key2, each lane the heads of parity par
    const int key2 = 16 * q + (lane >> 2) + 8 * (lane & 1);
    const int par = (lane >> 1) & 1;
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const RowSlot *slots = reinterpret_cast<const RowSlot *>(smem + kRowSlotOff);
    const int arr_n = (P.topk + kKeys - 1) / kKeys * kKeys;
    float *parr = reinterpret_cast<float *>(smem + P.parr_off);       // [2 halves][arr_n]
    float *iarr = reinterpret_cast<float *>(smem + P.iarr_off);       // [2 halves][arr_n]
    float *rw = reinterpret_cast<float *>(smem + kRowDataOff);        // w[64]
    float *rmax = rw + 64, *rsum = rw + 96;                           // softmax max / sum [32]
    float *dwx = reinterpret_cast<float *>(smem + kDwOff);            // [64 heads][4 quarters]
    const float kInf = __int_as_float(0x7f800000);
    uint32_t sph = 0, dsph = 0, dkph = 0, nrow_dq = 0, use = 0;
    const float scale2 = P.scale * kLog2e;                // scale in log2 units
    const int h0 = 32 * hf;                               // first indexer head of this half
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
        if (tiles == 0) {
            // no selected key: the row contributes nothing
            for (int e = tid; e < P.H * kDi; e += kEpiThreads) P.d_qi[(int64_t)row * P.H * kDi + e] = 0.f;
            for (int h = tid; h < P.H; h += kEpiThreads) P.d_w[(int64_t)row * P.H + h] = 0.f;
            if (tid == 0) P.row_loss[row] = 0.f;
            continue;
        }
        // the row's weights and main-attention statistics (rw is rewritten only after the
        // exchange below, which every epilogue thread reaches after its last use of the previous
        // row's values)
        {
            float dummy = 0.f;
            if (!epi_reduce(dummy, false, use, smem, bars, abort_flag)) { ok = false; break; }
            if (tid < 64) rw[tid] = tid < P.H ? bf16_val(P.w[(int64_t)row * P.H + tid]) : 0.f;
            // staged for the exponent's FMA: max in log2 units and the reciprocal of the sum
            if (tid < 32) {
                rmax[tid] = tid < P.G ? P.smax[(int64_t)row * P.G + tid] * kLog2e : 0.f;
                rsum[tid] = tid < P.G ? 1.f / P.ssum[(int64_t)row * P.G + tid] : 1.f;
            }
            if (!epi_reduce(dummy, false, use, smem, bars, abort_flag)) { ok = false; break; }
        }
        // ---- pass 1: each half's share of p^ and I of every selected key ----------------------
        for (int j = 0; j < tiles; ++j) {
            const int pos2 = kKeys * j + key2;
            const int32_t v2 = pos2 < P.topk ? __ldg(ir + pos2) : -1;
            const bool valid2 = v2 >= 0 && v2 < P.s2;
            if (!wait_warp(bars.s_full(), sph, abort_flag)) { ok = false; break; }
            sph ^= 1u;
            tc_fence_after();
            // this half's main and indexer heads of key key2, the parity-par ones in this lane,
            // loaded with one wait, then released
            uint32_t smr[NG / 16][8], sir[2][8];
#pragma unroll
            for (int c = 0; c < NG / 16; ++c) tmem_ld16x16_nowait(tmem + lane_addr + kColSm + 16 * c, smr[c]);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (h0 + 16 * c < P.Nh) {
                    tmem_ld16x16_nowait(tmem + lane_addr + kColSi + h0 + 16 * c, sir[c]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) sir[c][i] = 0u;
                }
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_empty());
            // I share over this lane's indexer heads h0 + 16 c + par + 2 i
            float ia = 0.f;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    ia = fmaf(rw[h0 + 16 * c + par + 2 * i], fmaxf(__uint_as_float(sir[c][i]), 0.f), ia);
            // p^ share over this lane's main heads of the half: g = par + 2 i of 16 columns
            // (register indices fixed at compile time for each half)
            auto main_share = [&](auto half_c) -> float {
                constexpr int HF = decltype(half_c)::value;
                constexpr int C = NG == 16 ? 0 : HF;              // the 16 columns of this half
                constexpr int I0 = NG == 16 ? 4 * HF : 0;         // registers of this half
                constexpr int NI = NG == 16 ? 4 : 8;
                float acc = 0.f;
#pragma unroll
                for (int i = I0; i < I0 + NI; ++i) {
                    const int g = 16 * C + par + 2 * i;
                    const float sg = __uint_as_float(smr[C][i]);
                    if (g < P.G) acc = fmaf(exp2f(fmaf(sg, scale2, -rmax[g])), rsum[g], acc);
                }
                return acc;
            };
            float ph = hf == 0 ? main_share(std::integral_constant<int, 0>{})
                               : main_share(std::integral_constant<int, 1>{});
            // the key's half-shares: this lane's heads plus the partner lane's
            ph += __shfl_xor_sync(0xffffffffu, ph, 2);
            ia += __shfl_xor_sync(0xffffffffu, ia, 2);
            if (par == 0 && pos2 < tiles * kKeys) {
                parr[hf * arr_n + pos2] = valid2 ? ph : 0.f;
                iarr[hf * arr_n + pos2] = valid2 ? ia : (hf == 0 ? -kInf : 0.f);
            }
        }
        if (!ok) break;
        // ---- row statistics, loss and dI ----------------------------------------------------------
        const int n = tiles * kKeys;
        {
            // the two halves' shares, written by lanes 0-15 of every epilogue warp: the exchange
            // orders those writes before these reads; p^ and I are their sums (half 0 + half 1)
            float d0 = 0.f;
            if (!epi_reduce(d0, false, use, smem, bars, abort_flag)) { ok = false; break; }
        }
        float zp = 0.f, im = -kInf;
        for (int e = tid; e < n; e += kEpiThreads) {
            const float pe = parr[e] + parr[arr_n + e];
            const float ie = iarr[e] + iarr[arr_n + e];
            parr[e] = pe;
            iarr[e] = ie;
            zp += pe;
            im = fmaxf(im, ie);
        }
        if (!epi_reduce(zp, false, use, smem, bars, abort_flag)) { ok = false; break; }
        if (!epi_reduce(im, true, use, smem, bars, abort_flag)) { ok = false; break; }
        float zi = 0.f;
        for (int e = tid; e < n; e += kEpiThreads)
            if (iarr[e] > -kInf) zi += exp2f((iarr[e] - im) * kLog2e);
        if (!epi_reduce(zi, false, use, smem, bars, abort_flag)) { ok = false; break; }
        const float log_zi = __log2f(zi) * kLn2;
        float loss = 0.f;
        for (int e = tid; e < n; e += kEpiThreads) {
            const float p = zp > 0.f ? parr[e] / zp : 0.f;
            const bool sel = iarr[e] > -kInf;
            const float ls = (iarr[e] - im) - log_zi;                 // log softmax(I)
            const float sig = sel ? exp2f((iarr[e] - im) * kLog2e) / zi : 0.f;
            if (p > 0.f) loss += p * (__log2f(p) * kLn2 - ls);
            parr[e] = sig - p;                                        // dI
        }
        if (!epi_reduce(loss, false, use, smem, bars, abort_flag)) { ok = false; break; }
        if (tid == 0) P.row_loss[row] = loss;
        // ---- pass 2: dS, d_w, d_qi and the dK rows, each half its heads and dims ---------------
        // d_w: each (head, quarter) entry of dwx has one owner (the half holding the head), which
        // adds its tiles' sums in tile order; the four quarters are added in order at the row's
        // end. The previous row's final read of dwx came before the exchanges above.
        // the head whose d_w sum over a quarter's keys this lane holds after the reduction below
        const int dw_idx = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + (lane & 1);
        const int dw_head = h0 + 16 * (dw_idx >> 3) + par + 2 * (dw_idx & 7);
        dwx[dw_head * 4 + q] = 0.f;
        float *slice = P.d_part + (int64_t)blockIdx.x * P.key_rows * kDi;
        for (int j = 0; j < tiles; ++j) {
            const int pos = kKeys * j + key;                  // dK rows: lanes 0-15, key `key`
            const int32_t v = kl && pos < P.topk ? __ldg(ir + pos) : -1;
            const bool valid = v >= 0 && v < P.s2;
            const int pos2 = kKeys * j + key2;                // dS and d_w: every lane, key `key2`
            const int32_t v2 = pos2 < P.topk ? __ldg(ir + pos2) : -1;
            const bool valid2 = v2 >= 0 && v2 < P.s2;
            const float dI2 = pos2 < n ? parr[pos2] : 0.f;
            if (!wait_warp(bars.s_full(), sph, abort_flag)) { ok = false; break; }
            sph ^= 1u;
            tc_fence_after();
            // this tile's S~, this half's heads of key key2, the parity-par ones in this lane (the
            // MMA recomputes the columns for the next tile once released)
            uint32_t svr[2][8];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (h0 + 16 * c < P.Nh) {
                    tmem_ld16x16_nowait(tmem + lane_addr + kColSi + h0 + 16 * c, svr[c]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) svr[c][i] = 0u;
                }
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.s_empty());
            // the dS buffers are free once the previous tile's products are done
            if (!wait_warp(bars.ds_empty(), dsph ^ 1u, abort_flag)) { ok = false; break; }
            dsph ^= 1u;
            uint8_t *dsb = smem + P.ds_off;
            // dS and the d_w terms of this lane's 16 heads h0 + 16 c + par + 2 i (index 8 c + i)
            float dsv[16], dwp[16];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int h = h0 + 16 * c + par + 2 * i;
                    const float sv = __uint_as_float(svr[c][i]);
                    dsv[8 * c + i] = valid2 && h < P.H && sv > 0.f ? dI2 * rw[h] : 0.f;
                    dwp[8 * c + i] = valid2 && h < P.H ? dI2 * fmaxf(sv, 0.f) : 0.f;
                }
            }
            {
                // consecutive head pairs: lane par = 0 assembles heads h0 .. h0 + 15 of key2
                // (its even heads, the partner's odd ones), lane par = 1 heads h0 + 16 .. h0 + 31
                uint32_t hi[8], lo[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float send = par ? dsv[i] : dsv[8 + i];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
                    const float ev = par ? recv : dsv[i];
                    const float od = par ? dsv[8 + i] : recv;
                    // hi = bf16(dS) and lo = bf16(dS - hi), two heads per conversion
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(ev, od);
                    const uint32_t hb = *reinterpret_cast<const uint32_t *>(&h2);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(ev - __uint_as_float(hb << 16),
                                                                    od - __uint_as_float(hb & 0xffff0000u));
                    hi[i] = hb;
                    lo[i] = *reinterpret_cast<const uint32_t *>(&l2);
                }
                // key2's row, 16-byte chunks of heads hb2 .. hb2 + 15, swizzled by key2 % 8
                const int hb2 = h0 + 16 * par;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t chunk = (uint32_t)(hb2 / 8 + u);
                    const uint32_t off = (uint32_t)(key2 >> 3) * 1024u + (uint32_t)(key2 & 7) * 128u +
                                         ((chunk ^ (uint32_t)(key2 & 7)) << 4);
                    *reinterpret_cast<uint4 *>(dsb + off) =
                        make_uint4(hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3]);
                    *reinterpret_cast<uint4 *>(dsb + kChunk + off) =
                        make_uint4(lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3]);
                }
            }
            fence_async_smem();
            mbar_arrive(bars.ds_full());
            // this key's previous partial dK row (this half's 64 dims) is loaded now, so the load
            // is in flight during the d_w sums and the wait for the product
            const int64_t dkr = key_base + (valid ? v : 0);
            const bool dk_on = kl && valid && idx_ok(dkr, P.key_rows, P.status);
            float4 *drow = reinterpret_cast<float4 *>(slice + dkr * kDi) + 16 * hf;
            float4 old[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) old[i] = dk_on ? drow[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            // d_w: per-head sums over the quarter's 16 keys (lanes differing in bits 0, 2, 3, 4);
            // each step halves the values a lane holds, the lanes with the step's bit set keeping
            // the upper half, so lane l ends with head dw_head
            {
#pragma unroll
                for (int st = 0; st < 4; ++st) {
                    const int m = st == 0 ? 16 : st == 1 ? 8 : st == 2 ? 4 : 1;
                    const int half_n = 8 >> st;
                    const bool up = (lane & m) != 0;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        if (k < half_n) {
                            const float keep = up ? dwp[k + half_n] : dwp[k];
                            const float send = up ? dwp[k] : dwp[k + half_n];
                            dwp[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                        }
                    }
                }
                dwx[dw_head * 4 + q] += dwp[0];
            }
            // this tile's dK rows (this half's dims) into the CTA's slice of the partial buffer
            if (!wait_warp(bars.dk_full(), dkph, abort_flag)) { ok = false; break; }
            dkph ^= 1u;
            tc_fence_after();
            {
                uint32_t dkv[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tmem_ld16_nowait(tmem + lane_addr + kColDk + 64 * hf + 16 * c, dkv[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float4 o = old[4 * c + i];
                        o.x += __uint_as_float(dkv[c][4 * i]);
                        o.y += __uint_as_float(dkv[c][4 * i + 1]);
                        o.z += __uint_as_float(dkv[c][4 * i + 2]);
                        o.w += __uint_as_float(dkv[c][4 * i + 3]);
                        old[4 * c + i] = o;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.dk_empty());
            if (dk_on) {
#pragma unroll
                for (int i = 0; i < 16; ++i) drow[i] = old[i];
            }
        }
        if (!ok) break;
        // ---- the row's d_qi (this half's dims) and d_w --------------------------------------------
        if (!wait_warp(bars.dq_full(), nrow_dq & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        {
            uint32_t dqv[4][16];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld16_nowait(tmem + lane_addr + kColDq + 64 * hf + 16 * c, dqv[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.dq_empty());
            if (kl && key < P.H && idx_ok(row, P.rows, P.status)) {
                float4 *dq = reinterpret_cast<float4 *>(P.d_qi + ((int64_t)row * P.H + key) * kDi + 64 * hf);
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dq[4 * c + i] = make_float4(__uint_as_float(dqv[c][4 * i]), __uint_as_float(dqv[c][4 * i + 1]),
                                                    __uint_as_float(dqv[c][4 * i + 2]), __uint_as_float(dqv[c][4 * i + 3]));
            }
        }
        ++nrow_dq;
        {
            float d0 = 0.f;                  // orders every half's dwx entries before the sums
            if (!epi_reduce(d0, false, use, smem, bars, abort_flag)) { ok = false; break; }
        }
        if (tid < P.H)
            P.d_w[(int64_t)row * P.H + tid] =
                (dwx[tid * 4] + dwx[tid * 4 + 1]) + (dwx[tid * 4 + 2] + dwx[tid * 4 + 3]);
        // the d_part rows written above are read by later rows of this CTA through the same
        // threads or others: order them before the next row's updates
        __threadfence_block();
    }
    if (!ok) *abort_flag = 1;
}

template <int NG>
__global__ void __launch_bounds__(kThreads, 1)
kl_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmr,
             const __grid_constant__ CUtensorMap tmi, const KlTcParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) atomicOr(P.status, LI_DEVERR_INTERNAL);
        return;
    }
    Bars bars{sbase + kTailOff};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kFlagOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kFlagOff + 4);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.rs_full(i), 1);
            mbar_init(bars.rs_empty(i), 1 + kEpiWarps + kGatherWarps);
            mbar_init(bars.xch(i), kEpiThreads);
        }
        mbar_init(bars.q_full(), 1);
        mbar_init(bars.q_empty(), 1);
        mbar_init(bars.s_full(), 1);
        mbar_init(bars.s_empty(), kEpiWarps);
        mbar_init(bars.ds_full(), kEpiThreads);
        mbar_init(bars.ds_empty(), 1);
        mbar_init(bars.dk_full(), 1);
        mbar_init(bars.dk_empty(), kEpiWarps);
        mbar_init(bars.dq_full(), 1);
        mbar_init(bars.dq_empty(), kEpiWarps);
        for (int i = 0; i < kTileRing; ++i) mbar_init(bars.tile_full(i), kGatherThreads);
        for (int i = 0; i < kMaxKiSlots; ++i) mbar_init(bars.ki_empty(i), 1);
        for (int i = 0; i < kMaxMainSlots; ++i) mbar_init(bars.main_empty(i), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // heads past G (main query) and H (indexer query) are never loaded: zero them once
    {
        const int pad_m = (P.Ng - P.G) * 8, pad_i = (P.Nh - P.H) * 8;   // 16-byte words per chunk
        for (int i = threadIdx.x; i < P.nmc * pad_m; i += kThreads) {
            const int c = i / pad_m, r = i % pad_m;
            *reinterpret_cast<uint4 *>(smem + P.qm_off + c * P.Ng * 128 + (P.G + r / 8) * 128 + (r % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        for (int i = threadIdx.x; i < 2 * pad_i; i += kThreads) {
            const int c = i / pad_i, r = i % pad_i;
            *reinterpret_cast<uint4 *>(smem + P.qi_off + c * P.Nh * 128 + (P.H + r / 8) * 128 + (r % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();
    }
    if (warp == kSchedWarp && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmq)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmi)) : "memory");
        if (P.Dr > 0)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmr)) : "memory");
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kEpiWarps) {
        epilogue_role<NG>(P, smem, bars, abort_flag, tmem);
    } else if (warp == kMmaWarp) {
        if (lane == 0) mma_role(P, smem, bars, abort_flag, tmem);
        __syncwarp();
    } else if (warp == kSchedWarp) {
        scheduler_role(P, &tmq, &tmr, &tmi, smem, bars, abort_flag);
    } else {
        gather_role(P, smem, bars, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(P.status, LI_DEVERR_TIMEOUT);
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// d_ki[key][d] = sum over the C slices of d_part in slice order.
__global__ void __launch_bounds__(256) kl_dki_sum_kernel(const float *d_part, int chunks,
                                                         int64_t n, float *d_ki) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x) {
        float a = 0.f;
        for (int c = 0; c < chunks; ++c) a += d_part[(int64_t)c * n + e];
        d_ki[e] = a;
    }
}

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

bool kl_tc_plan(const li_kl_args &a, KlTcPlan *L) {
    const bool shapes = a.Dm % 64 == 0 && a.Dm >= 64 && a.Dm <= 512 && (a.Dr == 0 || a.Dr == 64) &&
                        a.G >= 1 && a.G <= 32 && a.H >= 1 && a.H <= 64 && a.topk <= 2048;
    if (!shapes) return false;
    L->Ng = (a.G + 15) / 16 * 16;
    L->Nh = (a.H + 15) / 16 * 16;
    L->nmc = a.Dm / 64 + (a.Dr > 0 ? 1 : 0);
    uint32_t off = 0;
    L->qm_off = off;
    off += (uint32_t)L->nmc * L->Ng * 128u;
    off = (off + 1023u) / 1024u * 1024u;
    L->qi_off = off;
    off += 2u * L->Nh * 128u;
    off = (off + 1023u) / 1024u * 1024u;
    L->ds_off = off;
    off += 2u * kChunk;
    const uint32_t arr = (uint32_t)((a.topk + kKeys - 1) / kKeys * kKeys) * 4u;
    L->parr_off = off;                                   // two halves' shares, then p^ / dI
    off += 2 * arr;
    L->iarr_off = off;
    off += 2 * arr;
    off = (off + 1023u) / 1024u * 1024u;
    L->ki_off = off;
    L->ki_slots = 2;
    off += (uint32_t)L->ki_slots * 2u * kChunk;
    L->main_off = off;
    if (off >= kTailOff) return false;
    int slots = (int)((kTailOff - off) / kChunk);
    if (slots > kMaxMainSlots) slots = kMaxMainSlots;
    // the gather runs at most (slots / nmc + ki slots) tiles ahead of the MMA: below the ring
    if (slots < L->nmc) return false;
    L->main_slots = slots;
    return true;
}

size_t kl_tc_partial_floats(const li_kl_args &a, int chunks) {
    return (size_t)chunks * (size_t)a.batch * (size_t)a.s2 * kDi;
}

int kl_tc_chunks(const li_kl_args &a) {
    const int64_t rows = (int64_t)a.batch * a.s1;
    int c = device_sm_count();
    if (rows < c) c = (int)(rows > 0 ? rows : 1);
    return c;
}

cudaError_t launch_kl_tc(const li_kl_args &a, const KlTcPlan &L, float *row_loss, uint32_t *status,
                         float *d_part, int chunks, float *d_qi, float *d_ki, float *d_w,
                         cudaStream_t st) {
    const int64_t rows = (int64_t)a.batch * a.s1;
    const int64_t key_rows = (int64_t)a.batch * a.s2;
    const size_t part = kl_tc_partial_floats(a, chunks);
    cudaError_t e = cudaMemsetAsync(d_part, 0, part * sizeof(float), st);
    if (e != cudaSuccess) return e;
    if (rows > 0) {
        KlTcParams P{};
        P.k = static_cast<const uint16_t *>(a.k);
        P.k_rope = static_cast<const uint16_t *>(a.k_rope);
        P.ki = static_cast<const uint16_t *>(a.ki);
        P.w = static_cast<const uint16_t *>(a.w);
        P.indices = a.sparse_indices;
        P.smax = a.softmax_max;
        P.ssum = a.softmax_sum;
        P.row_loss = row_loss;
        P.d_qi = d_qi;
        P.d_w = d_w;
        P.d_part = d_part;
        P.status = status;
        P.scale = a.scale;
        P.rows = (int32_t)rows;
        P.s1 = a.s1; P.s2 = a.s2; P.G = a.G; P.Ng = L.Ng; P.Dm = a.Dm; P.Dr = a.Dr;
        P.H = a.H; P.Nh = L.Nh; P.topk = a.topk; P.nmc = L.nmc; P.chunks = chunks;
        P.key_rows = key_rows;
        P.qm_off = L.qm_off; P.qi_off = L.qi_off; P.ds_off = L.ds_off; P.parr_off = L.parr_off;
        P.iarr_off = L.iarr_off; P.main_off = L.main_off; P.ki_off = L.ki_off;
        P.main_slots = L.main_slots; P.ki_slots = L.ki_slots;
        // D fp32, A and B bf16; scores: K-major A and B, M = 64; d_qi: MN-major A and B, M = 64,
        // N = 128; dK: K-major A, MN-major B, M = 64, N = 128
        const uint32_t base = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 4) << 24);
        P.idesc_sm = base | ((uint32_t)(L.Ng >> 3) << 17);
        P.idesc_si = base | ((uint32_t)(L.Nh >> 3) << 17);
        P.idesc_dq = base | (1u << 15) | (1u << 16) | ((uint32_t)(128 >> 3) << 17);
        P.idesc_dk = base | (1u << 16) | ((uint32_t)(128 >> 3) << 17);
        CUtensorMap mq, mr, mi;
        if (!make_map_bf16(&mq, a.q, (uint64_t)rows * a.G, (uint64_t)a.Dm, (uint32_t)a.G))
            return cudaErrorInvalidValue;
        if (a.Dr > 0) {
            if (!make_map_bf16(&mr, a.q_rope, (uint64_t)rows * a.G, (uint64_t)a.Dr, (uint32_t)a.G))
                return cudaErrorInvalidValue;
        } else {
            mr = mq;
        }
        if (!make_map_bf16(&mi, a.qi, (uint64_t)rows * a.H, (uint64_t)kDi, (uint32_t)a.H))
            return cudaErrorInvalidValue;
        auto kern = L.Ng <= 16 ? kl_tc_kernel<16> : kl_tc_kernel<32>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        kern<<<chunks, kThreads, kSmemBytes, st>>>(mq, mr, mi, P);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int64_t n = key_rows * kDi;
    if (n > 0) {
        int grid = (int)((n + 255) / 256);
        if (grid > 4 * device_sm_count()) grid = 4 * device_sm_count();
        kl_dki_sum_kernel<<<grid, 256, 0, st>>>(d_part, chunks, n, d_ki);
    }
    return cudaGetLastError();
}

}  // namespace li
