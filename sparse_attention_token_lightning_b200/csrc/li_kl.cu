// The indexer's backward with the KL loss (torch_npu.npu_sparse_lightning_indexer_grad_kl_loss,
// formulas 1-4), first version on CUDA cores in fp32.
//
// One CTA per query row r (batch b = r / S1):
//   0. stage the row's main-attention query (bf16), indexer query (fp32) and weights in shared
//      memory and compact its selected keys (valid positions of sparse_indices) into key rows;
//   1. per selected key s (threads over keys): the main attention's head sum
//      p^[s] = sum_g exp(scale (q_g . k_s + qr_g . kr_s) - max_g) / sum_g and the indexer score
//      I[s] = sum_h w_h ReLU(qi_h . ki_s);
//   2. block reductions: p = p^ / sum p^, softmax(I), the row's loss sum_s p log(p / softmax(I))
//      (0 log 0 = 0), and dI = softmax(I) - p;
//   3. in chunks of kChunk keys: S_h(s) again, dS[h][s] = dI w_h [S > 0], d_w[h] += dI ReLU(S),
//      d_qi[h][:] += sum_s dS[h][s] ki_s (outputs owned by threads, no atomics) and
//      d_ki[s][:] += sum_h dS[h][s] qi_h (atomic adds into the fp32 output, shared by rows).
// A second kernel adds the per-row losses in a fixed order.
//
// Algorithmic work per selected (row, key): 2 G (Dm + Dr) + 2 H Di flops for phase 1, 2 H Di for
// S again, 4 H Di for the two gradient products.
#include <cuda_bf16.h>

#include "li_internal.cuh"
#include "li_kl.cuh"

namespace li {
namespace {

constexpr int kT = 256;
constexpr int kChunk = 32;
constexpr int kDi = 128;

struct KlParams {
    const __nv_bfloat16 *q, *k, *q_rope, *k_rope, *qi, *ki, *w;
    const int32_t *sparse_indices;
    const float *smax, *ssum;
    float scale;
    int32_t s1, s2, G, Dm, Dr, H, topk;
    float *row_loss;
    uint32_t *status;
    float *d_qi, *d_ki, *d_w;
};

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// Block-wide sum (every thread gets the total).
__device__ float block_sum(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.0f;
    for (int i = 0; i < kT / 32; ++i) t += red[i];
    return t;
}

__device__ float block_max(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = red[0];
    for (int i = 1; i < kT / 32; ++i) t = fmaxf(t, red[i]);
    return t;
}

__global__ void __launch_bounds__(kT) kl_row_kernel(const KlParams P) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ float red[kT / 32];
    __shared__ int32_t s_cnt[kT / 32 + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r = blockIdx.x;
    const int64_t b = r / P.s1;
    const int G = P.G, H = P.H, Dm = P.Dm, Dr = P.Dr, Dq = Dm + Dr, K = P.topk;

    // shared memory: qm [G][Dq] bf16 | qi [H][kDi] f32 | dq [H][kDi] f32 | kc [kChunk][kDi] f32 |
    // dS [H][kChunk] f32 | w [H] | dw [H] | kr [K] int32 | ph [K] f32 | I [K] f32
    __nv_bfloat16 *qm = reinterpret_cast<__nv_bfloat16 *>(dsm);
    float *qi = reinterpret_cast<float *>(dsm + ((size_t)G * Dq * 2 + 15) / 16 * 16);
    float *dq = qi + H * kDi;
    float *kc = dq + H * kDi;
    float *dS = kc + kChunk * kDi;
    float *ws = dS + H * kChunk;
    float *dw = ws + H;
    int32_t *kr = reinterpret_cast<int32_t *>(dw + H);
    float *ph = reinterpret_cast<float *>(kr + K);
    float *Is = ph + K;

    // ---- 0. stage the row ------------------------------------------------------------------
    for (int e = tid; e < G * Dm; e += kT)
        qm[(e / Dm) * Dq + e % Dm] = P.q[(r * G) * Dm + e];
    for (int e = tid; e < G * Dr; e += kT)
        qm[(e / Dr) * Dq + Dm + e % Dr] = P.q_rope[(r * G) * Dr + e];
    for (int e = tid; e < H * kDi; e += kT) {
        qi[e] = bf(P.qi[r * H * kDi + e]);
        dq[e] = 0.0f;
    }
    for (int h = tid; h < H; h += kT) {
        ws[h] = bf(P.w[r * H + h]);
        dw[h] = 0.0f;
    }
    // compact the valid selections: thread t owns entries [t*per, (t+1)*per)
    const int per = (K + kT - 1) / kT;
    uint32_t err = 0;
    int mine = 0;
    for (int i = 0; i < per; ++i) {
        const int e = tid * per + i;
        if (e < K) {
            const int32_t j = P.sparse_indices[r * K + e];
            if (j >= P.s2) err |= LI_DEVERR_LENGTHS;
            if (j >= 0 && j < P.s2) ++mine;
        }
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) s_cnt[warp] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int i = 0; i < kT / 32; ++i) {
            const int c = s_cnt[i];
            s_cnt[i] = run;
            run += c;
        }
        s_cnt[kT / 32] = run;
    }
    __syncthreads();
    int pos = s_cnt[warp] + incl - mine;
    for (int i = 0; i < per; ++i) {
        const int e = tid * per + i;
        if (e < K) {
            const int32_t j = P.sparse_indices[r * K + e];
            if (j >= 0 && j < P.s2) kr[pos++] = (int32_t)(b * P.s2 + j);
        }
    }
    const int n = s_cnt[kT / 32];
    __syncthreads();

    // ---- 1. per selected key: main-attention head sum and indexer score ----------------------
    for (int s = tid; s < n; s += kT) {
        const int64_t row = kr[s];
        const __nv_bfloat16 *kk = P.k + row * Dm;
        const __nv_bfloat16 *kro = Dr ? P.k_rope + row * Dr : nullptr;
        float p_hat = 0.0f;
        for (int g = 0; g < G; ++g) {
            const __nv_bfloat16 *qg = qm + g * Dq;
            float x = 0.0f;
            for (int d = 0; d < Dm; ++d) x = fmaf(bf(qg[d]), bf(kk[d]), x);
            for (int d = 0; d < Dr; ++d) x = fmaf(bf(qg[Dm + d]), bf(kro[d]), x);
            p_hat += __expf(P.scale * x - P.smax[r * G + g]) / P.ssum[r * G + g];
        }
        const __nv_bfloat16 *kiv = P.ki + row * kDi;
        float I = 0.0f;
        for (int h = 0; h < H; ++h) {
            const float *qh = qi + h * kDi;
            float x = 0.0f;
            for (int d = 0; d < kDi; ++d) x = fmaf(qh[d], bf(kiv[d]), x);
            I = fmaf(ws[h], fmaxf(x, 0.0f), I);
        }
        ph[s] = p_hat;
        Is[s] = I;
    }
    __syncthreads();

    // ---- 2. row reductions, loss, dI ---------------------------------------------------------
    float part = 0.0f, imax = -__int_as_float(0x7f800000);
    for (int s = tid; s < n; s += kT) {
        part += ph[s];
        imax = fmaxf(imax, Is[s]);
    }
    const float psum = block_sum(part, red);
    const float mx = block_max(imax, red);
    part = 0.0f;
    for (int s = tid; s < n; s += kT) part += __expf(Is[s] - mx);
    const float esum = block_sum(part, red);
    const float lse = logf(esum);
    part = 0.0f;
    for (int s = tid; s < n; s += kT) {
        const float p = ph[s] / psum;
        const float lsig = Is[s] - mx - lse;              // log softmax(I)[s]
        if (p > 0.0f) part += p * (logf(p) - lsig);
        ph[s] = __expf(lsig) - p;                         // dI
    }
    const float loss = block_sum(part, red);
    if (tid == 0) P.row_loss[r] = n > 0 ? loss : 0.0f;
    __syncthreads();

    // ---- 3. gradients, kChunk keys at a time -------------------------------------------------
    for (int c0 = 0; c0 < n; c0 += kChunk) {
        const int nc = min(kChunk, n - c0);
        for (int e = tid; e < kChunk * kDi; e += kT) {
            const int s = e / kDi;
            kc[e] = s < nc ? bf(P.ki[(int64_t)kr[c0 + s] * kDi + e % kDi]) : 0.0f;
        }
        __syncthreads();
        for (int e = tid; e < H * kChunk; e += kT) {
            const int h = e / kChunk, s = e % kChunk;
            float v = 0.0f;
            if (s < nc) {
                float x = 0.0f;
                for (int d = 0; d < kDi; ++d) x = fmaf(qi[h * kDi + d], kc[s * kDi + d], x);
                const float dI = ph[c0 + s];
                if (x > 0.0f) {
                    v = dI * ws[h];
                    atomicAdd(&dw[h], dI * x);
                }
            }
            dS[e] = v;
        }
        __syncthreads();
        for (int e = tid; e < H * kDi; e += kT) {
            const int h = e / kDi, d = e % kDi;
            float acc = 0.0f;
            for (int s = 0; s < nc; ++s) acc = fmaf(dS[h * kChunk + s], kc[s * kDi + d], acc);
            dq[e] += acc;
        }
        for (int e = tid; e < nc * kDi; e += kT) {
            const int s = e / kDi, d = e % kDi;
            float acc = 0.0f;
            for (int h = 0; h < H; ++h) acc = fmaf(dS[h * kChunk + s], qi[h * kDi + d], acc);
            if (acc != 0.0f && idx_ok(kr[c0 + s], (int64_t)(gridDim.x / P.s1) * P.s2, P.status))
                atomicAdd(&P.d_ki[(int64_t)kr[c0 + s] * kDi + d], acc);
        }
        __syncthreads();
    }

    // ---- 4. the row's outputs ------------------------------------------------------------------
    for (int e = tid; e < H * kDi; e += kT) P.d_qi[r * H * kDi + e] = dq[e];
    for (int h = tid; h < H; h += kT) P.d_w[r * H + h] = dw[h];
    if (err) atomicOr(P.status, err);
}

// Sum of the per-row losses in a fixed order: thread t adds rows t, t + 1024, ... and the
// partial sums are combined by a fixed tree.
__global__ void __launch_bounds__(1024) kl_loss_kernel(const float *row_loss, int64_t rows,
                                                       float *loss) {
    __shared__ float part[1024];
    float a = 0.0f;
    for (int64_t i = threadIdx.x; i < rows; i += 1024) a += row_loss[i];
    part[threadIdx.x] = a;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = part[0];
}

}  // namespace

size_t kl_smem_bytes(int G, int Dm, int Dr, int H, int topk) {
    const size_t qm = ((size_t)G * (Dm + Dr) * 2 + 15) / 16 * 16;
    return qm + 4 * ((size_t)2 * H * kDi + (size_t)kChunk * kDi + (size_t)H * kChunk + 2 * H) +
           4 * (size_t)3 * topk;
}

cudaError_t launch_kl_grad(const li_kl_args &a, float *row_loss, uint32_t *status, float *loss,
                           float *d_qi, float *d_ki, float *d_w, cudaStream_t st) {
    const int64_t rows = (int64_t)a.batch * a.s1;
    cudaError_t e = cudaMemsetAsync(d_ki, 0, (size_t)a.batch * a.s2 * kDi * sizeof(float), st);
    if (e != cudaSuccess) return e;
    if (rows > 0) {
        KlParams P{};
        P.q = static_cast<const __nv_bfloat16 *>(a.q);
        P.k = static_cast<const __nv_bfloat16 *>(a.k);
        P.q_rope = static_cast<const __nv_bfloat16 *>(a.q_rope);
        P.k_rope = static_cast<const __nv_bfloat16 *>(a.k_rope);
        P.qi = static_cast<const __nv_bfloat16 *>(a.qi);
        P.ki = static_cast<const __nv_bfloat16 *>(a.ki);
        P.w = static_cast<const __nv_bfloat16 *>(a.w);
        P.sparse_indices = a.sparse_indices;
        P.smax = a.softmax_max;
        P.ssum = a.softmax_sum;
        P.scale = a.scale;
        P.s1 = a.s1; P.s2 = a.s2; P.G = a.G; P.Dm = a.Dm; P.Dr = a.Dr; P.H = a.H; P.topk = a.topk;
        P.row_loss = row_loss;
        P.status = status;
        P.d_qi = d_qi; P.d_ki = d_ki; P.d_w = d_w;
        const size_t smem = kl_smem_bytes(a.G, a.Dm, a.Dr, a.H, a.topk);
        e = cudaFuncSetAttribute(kl_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kl_row_kernel<<<(unsigned)rows, kT, smem, st>>>(P);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_kl_loss(row_loss, rows, loss, st);
}

cudaError_t launch_kl_loss(const float *row_loss, int64_t rows, float *loss, cudaStream_t st) {
    kl_loss_kernel<<<1, 1024, 0, st>>>(row_loss, rows, loss);
    return cudaGetLastError();
}

}  // namespace li
