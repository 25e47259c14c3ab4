// Sparse attention over the selected keys (li_attn.cu): shared-memory plan and launcher.
#pragma once

#include "li_internal.cuh"

namespace li {

// Shared-memory plan of the attention kernel for one argument set.
struct AttnLayout {
    int N;                  // MMA N: heads rounded up to 16
    int npairs;             // 128-dim pairs of the value/key rows (Dm / 128)
    int q_bufs;             // Q tile buffers (2 when a pair slot of prefetch still fits)
    int pair_slots, rope_slots;
    uint32_t q_bytes, q_off, p_off, pair_off, rope_off;
    uint32_t tmem_cols;
};

// False when the argument set does not fit the kernel's shared memory.
bool attn_layout(const li_attn_args &a, AttnLayout *L);

// status / ticket: the workspace header's status word and ticket counter (zeroed by the caller).
cudaError_t launch_sparse_attention(const li_attn_args &a, uint32_t *status, int32_t *ticket,
                                    float *out, float *smax, float *ssum, cudaStream_t st);

}  // namespace li
