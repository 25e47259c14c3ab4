// Tensor-core score kernel (tcgen05 + TMA + TMEM) -- placeholder until the kernel lands.
#include "li_internal.cuh"

namespace li {

cudaError_t launch_score_tc(const Problem &, const Schedule &, const void *, WsHeader *, float *,
                            int64_t, cudaStream_t, bool *launched) {
    *launched = false;
    return cudaSuccess;
}

}  // namespace li
