// Launcher of the indexer backward with the KL loss (li_kl.cu), called by li_kl_grad in
// li_api.cu after the arguments are validated.
#pragma once

#include <cuda_runtime.h>

#include "li.h"

namespace li {

// Dynamic shared memory of the per-row kernel.
size_t kl_smem_bytes(int G, int Dm, int Dr, int H, int topk);

// CUDA-core path: zeroes d_ki, then queues the per-row kernel (row losses into row_loss, device
// errors OR-ed into *status) and the fixed-order loss sum into *loss.
cudaError_t launch_kl_grad(const li_kl_args &a, float *row_loss, uint32_t *status, float *loss,
                           float *d_qi, float *d_ki, float *d_w, cudaStream_t st);

// Fixed-order sum of the per-row losses into *loss.
cudaError_t launch_kl_loss(const float *row_loss, int64_t rows, float *loss, cudaStream_t st);

// Tensor-core path (li_kl_tc.cu): shared-memory plan for one argument set.
struct KlTcPlan {
    int Ng, Nh, nmc;                     // MMA N of the main and indexer scores; main chunks/tile
    uint32_t qm_off, qi_off, ds_off, parr_off, iarr_off, ki_off, main_off;
    int ki_slots, main_slots;
};
// False when the shapes are outside the tensor-core kernel's (Dm a multiple of 64 up to 512,
// Dr 0 or 64, G <= 32, H <= 64) or its shared memory; the CUDA-core path runs then.
bool kl_tc_plan(const li_kl_args &a, KlTcPlan *plan);
// Row-owning CTAs (the grid) and the floats of their partial d_ki buffer [chunks][B*S2][128].
int kl_tc_chunks(const li_kl_args &a);
size_t kl_tc_partial_floats(const li_kl_args &a, int chunks);
// Queues the tensor-core kernel (row losses, d_qi, d_w, partial d_ki slices) and the fixed-order
// sum of the slices into d_ki; the loss sum follows with launch_kl_loss.
cudaError_t launch_kl_tc(const li_kl_args &a, const KlTcPlan &plan, float *row_loss,
                         uint32_t *status, float *d_part, int chunks, float *d_qi, float *d_ki,
                         float *d_w, cudaStream_t st);

}  // namespace li
