"""Row sharding of one BSND indexer problem across ranks (no data-path collective).

Query rows are independent given the keys. For the right-down causal mask (mask_mode 3) row i
of a batch with L1 query rows and L2 keys sees keys j <= i + L2 - L1. The rows [a, b) of every
batch therefore form the BSND problem

    q[:, a:b], w[:, a:b], k[:, :L2'],   L2' = b + S2 - S1 (clipped to [0, S2])

whose own alignment j <= i' + L2' - (b - a) with i' = i - a gives the same windows, and whose
output indices (positions in the batch's keys) are the same. With no mask every key is seen:
L2' = S2. Ranks take equal-size chunks in a zig-zag order (chunk r and chunk 2W-1-r), which
pairs short causal rows with long ones so every rank gets the same work.
"""
from __future__ import annotations

from .synthetic import Problem


def zigzag_chunks(rows: int, world: int, rank: int):
    """Row ranges [a, b) of `rank`: two of 2*world near-equal chunks, paired first-with-last."""
    n = 2 * world
    bounds = [rows * i // n for i in range(n + 1)]
    pick = [rank, n - 1 - rank]
    return [(bounds[c], bounds[c + 1]) for c in sorted(set(pick)) if bounds[c + 1] > bounds[c]]


def sub_problem(pb: Problem, a: int, b: int) -> Problem:
    """The rows [a, b) of every batch of a BSND problem as a problem of their own."""
    if pb.layout_q != "BSND" or pb.layout_k != "BSND":
        raise ValueError("row sharding is defined for BSND q and k")
    if pb.seqused_q is not None or pb.seqused_k is not None:
        raise ValueError("row sharding does not take seqused_q / seqused_k")
    S1, S2 = pb.q_len, pb.k_len
    if pb.mask_mode == 3:
        L2 = min(max(b + S2 - S1, 0), S2)
    else:
        L2 = S2
    return pb.replace(
        name=f"{pb.name}[{a}:{b}]",
        q=pb.q[:, a:b].contiguous(), w=pb.w[:, a:b].contiguous(),
        k=pb.k[:, :L2].contiguous(), q_len=b - a, k_len=L2,
        max_seqlen_q=b - a, max_seqlen_k=L2)
