// Launcher of the split-merge kernel (li_merge.cu), called by li_merge_topk in li_api.cu after
// the arguments are validated.
#pragma once

#include <cuda_runtime.h>

#include "li.h"

namespace li {

// Queues the merge of a->n_lists lists into a->idx_out / a->val_out on `stream`. Assumes
// validated arguments with 1 <= rows <= 2^31-1. `check`: verify each list's order and padding
// (LI_DEVERR_MERGE_ORDER); lists the library built itself skip it. The global-memory path (lists
// too large for shared memory) always checks.
cudaError_t launch_merge(const li_merge_args &a, cudaStream_t stream, bool check = true);

// Whether the merge of n_lists lists runs from shared memory (the fast path).
bool merge_fits_smem(int n_lists, int topk_in, int topk_out);

}  // namespace li
