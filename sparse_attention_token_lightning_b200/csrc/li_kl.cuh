// Launcher of the indexer backward with the KL loss (li_kl.cu), called by li_kl_grad in
// li_api.cu after the arguments are validated.
#pragma once

#include <cuda_runtime.h>

#include "li.h"

namespace li {

// Dynamic shared memory of the per-row kernel.
size_t kl_smem_bytes(int G, int Dm, int Dr, int H, int topk);

// Zeroes d_ki, then queues the per-row kernel (row losses into row_loss, device errors OR-ed into
// *status) and the fixed-order loss sum into *loss.
cudaError_t launch_kl_grad(const li_kl_args &a, float *row_loss, uint32_t *status, float *loss,
                           float *d_qi, float *d_ki, float *d_w, cudaStream_t st);

}  // namespace li
