// Reference-style score kernel on CUDA cores: the first correct path and a debug cross-check for
// the tensor-core kernel. Not a performance path.
//
// For every work item (batch b, rows [q0, q0+nq), keys [j0, j1)) and every row t it writes
//     I[t, j] = sum_h w[t,h] * max(q[t,h,:] . k[j,:], 0)          (fp32, heads in order)
// for the keys of the row's window inside the item's range, into the fp32 score rows of the
// workspace (custom_pypto.npu_lightning_indexer_pto, function description formula;
// lightning_indexer, "Function" steps 1-3). Keys are fetched per layout: BSND / TND rows, or the
// paged cache through the block table (custom_pypto.npu_lightning_indexer_pto, block_table).
#include <cuda_fp8.h>

#include "li_internal.cuh"

namespace li {
namespace {

constexpr int kThreads = 256;

struct Params {
    Problem p;
    SchedView view;
    WsHeader *ws;
    float *scores;
    int64_t ld;
    uint32_t signature;
    Quant qd;
};

__device__ inline float fp8_to_f32(uint8_t c) {
    __nv_fp8_e4m3 x;
    x.__x = c;
    return (float)x;
}

__global__ void __launch_bounds__(kThreads) score_simple_kernel(Params sp) {
    const Problem &p = sp.p;
    const SchedView &view = sp.view;
    int n_items = view.n_items;
    if (view.meta) {
        const MetaHeader *hdr = reinterpret_cast<const MetaHeader *>(view.meta);
        if (hdr->magic != kMetaMagic || hdr->signature != sp.signature) {
            if (threadIdx.x == 0 && blockIdx.x == 0) set_status(&sp.ws->status, kDevErrMetadata);
            return;
        }
        n_items = hdr->n_items;
    }
    const int H = p.n_heads;
    const bool fp16 = p.dtype_qk == LI_DTYPE_FP16;
    const bool fp8 = p.dtype_qk == LI_DTYPE_FP8_E4M3;
    if (blockIdx.x == 0) check_batch_keys(p, view, &sp.ws->status, threadIdx.x, kThreads);

    __shared__ float qs[kMaxHeads][kHeadDim];
    __shared__ float ws_[kMaxHeads];
    uint32_t err = 0;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const WorkItem it = view.item(p, item);
        if (it.j1 <= it.j0) continue;
        const BatchInfo bi = view.batch(p, it.b);
        for (int r = 0; r < it.nq; ++r) {
            const int32_t i = it.q0 + r;
            const int64_t row = (int64_t)bi.q_row0 + i;
            const int32_t hi =
                min(window_hi(p.mask_mode, i, bi.L1u, bi.L2, p.cmp_ratio, bi.pad[2]), it.j1);
            __syncthreads();   // previous row's readers are done with qs / ws_
            for (int e = threadIdx.x; e < H * kHeadDim; e += kThreads) {
                const int h = e / kHeadDim, d = e % kHeadDim;
                const int64_t qi = (row * H + h) * kHeadDim + d;
                if (fp8) {
                    // [reading] the code times its row-and-head scale
                    const float sc = sp.qd.q_descale[row * H + h];
                    if (!good_scale(sc)) err |= LI_DEVERR_DESCALE;
                    qs[h][d] = fp8_to_f32(reinterpret_cast<const uint8_t *>(p.q)[qi]) * sc;
                } else {
                    qs[h][d] = half16_to_f32(p.q[qi], fp16);
                }
            }
            for (int h = threadIdx.x; h < H; h += kThreads)
                ws_[h] = weight_f32(p, row * H + h);
            __syncthreads();
            for (int32_t j = it.j0 + threadIdx.x; j < hi; j += kThreads) {
                const uint16_t *kp = key_ptr(p, bi, it.b, j);
                float I = 0.0f;
                if (kp == nullptr) {
                    err |= LI_DEVERR_TABLE;
                } else if (fp8) {
                    const int64_t kr = key_row(p, bi, it.b, j);
                    const uint8_t *k8 = reinterpret_cast<const uint8_t *>(p.k) + kr * kHeadDim;
                    const float ks = sp.qd.k_descale[kr];
                    if (!good_scale(ks)) err |= LI_DEVERR_DESCALE;
                    float kv[kHeadDim];
#pragma unroll
                    for (int d = 0; d < kHeadDim; ++d) kv[d] = fp8_to_f32(k8[d]) * ks;
                    for (int h = 0; h < H; ++h) {
                        float s = 0.0f;
#pragma unroll
                        for (int d = 0; d < kHeadDim; ++d) s = fmaf(qs[h][d], kv[d], s);
                        I = fmaf(ws_[h], fmaxf(s, 0.0f), I);
                    }
                } else {
                    uint32_t kr[kHeadDim / 2];
                    const uint4 *k4 = reinterpret_cast<const uint4 *>(kp);
#pragma unroll
                    for (int c = 0; c < kHeadDim / 8; ++c) {
                        const uint4 v = __ldg(k4 + c);
                        kr[4 * c + 0] = v.x; kr[4 * c + 1] = v.y;
                        kr[4 * c + 2] = v.z; kr[4 * c + 3] = v.w;
                    }
                    for (int h = 0; h < H; ++h) {
                        float s = 0.0f;
#pragma unroll
                        for (int d2 = 0; d2 < kHeadDim / 2; ++d2) {
                            s = fmaf(qs[h][2 * d2], half16_to_f32(kr[d2] & 0xffffu, fp16), s);
                            s = fmaf(qs[h][2 * d2 + 1], half16_to_f32(kr[d2] >> 16, fp16), s);
                        }
                        I = fmaf(ws_[h], fmaxf(s, 0.0f), I);
                    }
                }
                if (in_bounds(row < sp.p.rows && j < sp.ld, &sp.ws->status))
                    sp.scores[row * sp.ld + j] = I;
            }
        }
    }
    if (err) set_status(&sp.ws->status, err);
}

}  // namespace

cudaError_t launch_score_simple(const Problem &p, const Quant &qd, const Schedule &s,
                                const void *meta, WsHeader *ws, float *scores, int64_t ld,
                                cudaStream_t st) {
    Params sp{p, make_view(p, s, meta), ws, scores, ld, problem_signature(p, s.tq, s.kc), qd};
    int grid = s.max_items < 148 * 8 ? s.max_items : 148 * 8;
    if (grid < 1) grid = 1;
    score_simple_kernel<<<grid, kThreads, 0, st>>>(sp);
    return cudaGetLastError();
}

}  // namespace li
