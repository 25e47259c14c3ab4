// Row-split selection (li_select.cu): few very long rows are cut into key pieces, each piece
// selected by its own CTA into a partial top-k list; li_api.cu then merges the lists with the
// split merge (li_merge.cu).
#pragma once

#include "li_internal.cuh"
#include "li_merge.cuh"

namespace li {

constexpr int kPieceMinKeys = 32768;   // rows shorter than this are never split
constexpr int kMaxPieces = 16;

// Pieces per row for this problem (1 = no split): enough CTAs to occupy the GPU, pieces of at
// least kPieceMinKeys / 2 keys, and a merge whose lists fit in shared memory.
int select_pieces(const Problem &p);

// Keys per piece (a multiple of 128).
int32_t piece_len(const Problem &p, int pieces);

// One CTA per (row, piece): list c of the partial buffers [pieces][rows][topk] (int32 indices
// with the row's output offset, fp32 values) holds piece c's top-k.
cudaError_t launch_select_pieces(const Problem &p, const Schedule &s, const void *meta,
                                 WsHeader *ws, const float *scores, int64_t ld, int pieces,
                                 int32_t *part_idx, float *part_val, cudaStream_t st);

}  // namespace li
