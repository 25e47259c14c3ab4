"""Row sharding of one BSND indexer problem across ranks (no data-path collective).

Query rows are independent given the keys. For the right-down causal mask (mask_mode 3) row i
of a batch with L1 query rows and L2 keys sees keys j <= i + L2 - L1. The rows [a, b) of every
batch therefore form the BSND problem

    q[:, a:b], w[:, a:b], k[:, :L2'],   L2' = b + S2 - S1 (clipped to [0, S2])

whose own alignment j <= i' + L2' - (b - a) with i' = i - a gives the same windows, and whose
output indices (positions in the batch's keys) are the same. With no mask every key is seen:
L2' = S2. Ranks take equal-size chunks in a zig-zag order (chunk r and chunk 2W-1-r), which
pairs short causal rows with long ones so every rank gets the same work.

Key-range sharding (one very long row, e.g. decode over a long context): rank r holds keys
[s_r, e_r) of every sequence and selects among them with output_idx_offset = s_r, so its indices
are global; the per-range lists are all-gathered and merged (li_merge_topk) into the row's
top-k, which equals the selection over the whole window because the ranges are disjoint and
the order is a total order. Under the right-down mask a row must see every key of every range
but the last (e_r <= L2 - L1 + 1), which then runs without a mask; the last range ends at L2
and keeps the mask, its local alignment j' <= i + (L2 - s) - L1 being the global one. Decode
rows (L1 = 1) see every key, so any split works for them.
"""
from __future__ import annotations

import torch

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


# ---- key-range sharding -------------------------------------------------------------------------

def key_ranges(L2: int, parts: int, align: int = 1, last_start_max: int | None = None):
    """Split keys [0, L2) into `parts` consecutive ranges (some may be empty): near-equal
    boundaries rounded down to multiples of `align`, none past `last_start_max`."""
    if parts < 1 or align < 1:
        raise ValueError("parts and align must be >= 1")
    cap = L2 if last_start_max is None else max(0, min(L2, last_start_max))
    cuts = [0]
    for r in range(1, parts):
        c = min(L2 * r // parts, cap) // align * align
        cuts.append(max(c, cuts[-1]))
    cuts.append(L2)
    return list(zip(cuts[:-1], cuts[1:]))


def _lengths(pb: Problem):
    """Per batch: (used query rows L1u, key length L2) as host ints."""
    if pb.layout_q == "TND":
        cu = pb.cu_seqlens_q.tolist()
        L1 = [cu[b + 1] - cu[b] for b in range(pb.batch)]
    else:
        L1 = [pb.q_len] * pb.batch
    if pb.seqused_q is not None:
        L1 = [min(a, int(u)) for a, u in zip(L1, pb.seqused_q.tolist())]
    if pb.layout_k == "PA_BSND":
        L2 = [int(x) for x in pb.seqused_k.tolist()]
    elif pb.layout_k == "BSND":
        L2 = [pb.k_len] * pb.batch
        if pb.seqused_k is not None:
            L2 = [min(a, int(u)) for a, u in zip(L2, pb.seqused_k.tolist())]
    else:
        raise ValueError("key-range sharding takes BSND or PA_BSND keys")
    return L1, L2


def key_shard(pb: Problem, parts: int, part: int, compact: bool = False) -> Problem:
    """The problem of key range `part` of `parts` (see the module notes): same query rows, the
    range's keys, output indices made global through output_idx_offset. With paged keys the
    range's block-table entries are shifted to the front; `compact` also copies the blocks the
    range uses into a cache of their own (what one GPU of a key-sharded deployment holds)."""
    if not 0 <= part < parts:
        raise ValueError("part outside [0, parts)")
    if pb.cmp_ratio > 1:
        raise ValueError("key-range sharding does not take compressed keys")
    L1, L2 = _lengths(pb)
    last = part == parts - 1
    # under the right-down mask every range but the last must lie inside every row's window
    reach = [l2 - l1 + 1 for l1, l2 in zip(L1, L2) if l1 > 0]
    off0 = (pb.output_idx_offset.tolist() if pb.output_idx_offset is not None
            else [0] * pb.batch)
    dev = pb.k.device
    if pb.layout_k == "BSND":
        cap = min(reach) if (pb.mask_mode == 3 and reach) else None
        s, e = key_ranges(pb.k_len, parts, 1, cap)[part]
        n = e - s
        used = [max(0, min(l2 - s, n)) for l2 in L2]
        kw = dict(k=pb.k[:, s:e].contiguous(), k_len=n, max_seqlen_k=n,
                  seqused_k=(None if all(u == n for u in used)
                             else torch.tensor(used, dtype=torch.int32, device=dev)),
                  output_idx_offset=torch.tensor([o + s for o in off0], dtype=torch.int32,
                                                 device=dev))
    else:
        bs = pb.block_size
        rng = []
        for b in range(pb.batch):
            cap = L2[b] - L1[b] + 1 if (pb.mask_mode == 3 and L1[b] > 0) else None
            rng.append(key_ranges(L2[b], parts, bs, cap)[part])
        width = max(1, max(-(-(e - s) // bs) for s, e in rng))
        table = torch.full((pb.batch, width), -1, dtype=torch.int32, device=pb.block_table.device)
        for b, (s, e) in enumerate(rng):
            nb = -(-(e - s) // bs)
            if nb:
                table[b, :nb] = pb.block_table[b, s // bs: s // bs + nb]
        if compact:
            ids = table.flatten()
            used = ids >= 0
            keep, pos = torch.unique(ids[used], return_inverse=True)
            if keep.numel() == 0:
                keep = torch.zeros(1, dtype=torch.int64, device=table.device)
            ids = ids.clone()
            ids[used] = pos.to(torch.int32)
            table = ids.view(table.shape)
            kc = pb.k.index_select(0, keep.to(device=pb.k.device, dtype=torch.int64)).contiguous()
        else:
            kc = pb.k
        kw = dict(k=kc, num_blocks=int(kc.shape[0]), block_table=table,
                  max_seqlen_k=max(1, max(e - s for s, e in rng)),
                  seqused_k=torch.tensor([e - s for s, e in rng], dtype=torch.int32, device=dev),
                  output_idx_offset=torch.tensor([o + s for o, (s, _e) in zip(off0, rng)],
                                                 dtype=torch.int32, device=dev))
    return pb.replace(name=f"{pb.name}[keys {part}/{parts}]",
                      mask_mode=pb.mask_mode if last else 0, **kw)


def key_sharded_indexer(pb_part: Problem, group=None, run=None, merge=None):
    """One rank's step of a key-range-sharded indexer: select in this rank's range
    (key_shard(pb, world, rank)), all-gather every rank's lists, merge. Returns the whole rows'
    (indices, values) on every rank. `run` and `merge` default to the CUDA library's
    li.indexer and li.merge_topk; the CPU tests pass the oracle's."""
    import torch.distributed as dist
    if run is None or merge is None:
        from . import li
        run = run or li.indexer
        merge = merge or li.merge_topk
    idx, val = run(pb_part)
    world = dist.get_world_size(group)
    gi = torch.empty((world,) + tuple(idx.shape), dtype=idx.dtype, device=idx.device)
    gv = torch.empty((world,) + tuple(val.shape), dtype=val.dtype, device=val.device)
    # list form (views of one buffer): NCCL and gloo both take it
    dist.all_gather(list(gi.unbind(0)), idx.contiguous(), group=group)
    dist.all_gather(list(gv.unbind(0)), val.contiguous(), group=group)
    return merge(gi, gv, pb_part.topk)
