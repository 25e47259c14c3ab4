"""Row sharding of one causal problem across ranks.

CPU: two gloo ranks each run the oracle on their zig-zag chunks, gather them on rank 0, and
the assembled result must equal the oracle on the whole problem (rows are independent, so this
checks the chunk algebra and the gather). GPU: the sharded li_indexer runs (one after the
other, on one device) must be bit-identical to the whole-problem run."""
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_token_lightning_b200 import shard, synthetic


def test_zigzag_chunks_partition_the_rows_with_equal_causal_work():
    for rows, world in [(4096, 2), (4096, 8), (1000, 3), (7, 4)]:
        seen = []
        work = []
        for r in range(world):
            ch = shard.zigzag_chunks(rows, world, r)
            seen += [i for a, b in ch for i in range(a, b)]
            work.append(sum((i + 1) for a, b in ch for i in range(a, b)))
        assert sorted(seen) == list(range(rows))
        if rows >= 64 * world:
            assert max(work) / min(work) < 1.02


def _rank_main(rank, world, init_file, result_file):
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank,
                            world_size=world)
    try:
        from oracle import oracle as orc_mod
        orc = orc_mod.default()
        pb = synthetic.bsnd(2, 96, 96, 4, 24, 3, seed=50)
        out = torch.full((2, 96, pb.topk), -7, dtype=torch.int32)
        for a, b in shard.zigzag_chunks(96, world, rank):
            sp = shard.sub_problem(pb, a, b)
            idx, _val, _rc = orc.topk(sp)
            out[:, a:b] = torch.from_numpy(idx).view(2, b - a, pb.topk)
        # each rank fills only its rows; the others stay -7 and are combined by max
        dist.all_reduce(out, op=dist.ReduceOp.MAX)
        if rank == 0:
            torch.save(out, result_file)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_whole_problem(orc):
    world = 2
    with tempfile.TemporaryDirectory() as d:
        init_file = os.path.join(d, "init")
        result_file = os.path.join(d, "out.pt")
        mp.spawn(_rank_main, args=(world, init_file, result_file), nprocs=world, join=True)
        got = torch.load(result_file)
    pb = synthetic.bsnd(2, 96, 96, 4, 24, 3, seed=50)
    idx, _val, _rc = orc.topk(pb)
    assert np.array_equal(got.view(-1, pb.topk).numpy(), idx)


@pytest.mark.parametrize("mask", [3, 0])
def test_sub_problem_rows_equal_whole_problem_rows(orc, mask):
    pb = synthetic.bsnd(1, 80, 120, 8, 16, mask, seed=51)
    whole_i, whole_v, _ = orc.topk(pb)
    for a, b in [(0, 13), (13, 50), (50, 80)]:
        i, v, _ = orc.topk(shard.sub_problem(pb, a, b))
        assert np.array_equal(i, whole_i[a:b])
        assert np.array_equal(v.view(np.uint32), whole_v[a:b].view(np.uint32))


# ---- key-range sharding ---------------------------------------------------------------------------

def test_key_ranges_partition_the_keys():
    for L2, parts, align, cap in [(1000, 3, 1, None), (1000, 8, 64, None), (100, 4, 1, 50),
                                  (5, 8, 1, None), (0, 3, 1, None), (4097, 2, 64, 4000)]:
        rng = shard.key_ranges(L2, parts, align, cap)
        assert len(rng) == parts and rng[0][0] == 0 and rng[-1][1] == L2
        assert all(a <= b for a, b in rng)
        assert all(rng[i][1] == rng[i + 1][0] for i in range(parts - 1))
        assert all(a % align == 0 for a, _ in rng)
        if cap is not None:
            assert rng[-1][0] <= cap


KEY_SHARD_CASES = {
    "paged_decode": lambda: synthetic.paged([3000, 700, 65, 1], 1, 16, 128, block_size=64,
                                            seed=90, spare_blocks=3),
    "paged_decode_bs16": lambda: synthetic.paged([900, 40], 1, 8, 300, block_size=16, seed=91),
    "paged_causal_rows": lambda: synthetic.paged([1000, 500], 3, 8, 100, block_size=64, seed=92),
    "paged_tnd_q_nomask": lambda: synthetic.paged([700, 300], 0, 8, 64, block_size=32, seed=93,
                                                  mask_mode=0, layout_q="TND", lens_q=[4, 2]),
    "bsnd_causal_seqused": lambda: synthetic.bsnd(2, 6, 500, 8, 150, 3, seed=94,
                                                  seqused_k=[500, 321]),
    "bsnd_nomask_offset": lambda: synthetic.bsnd(2, 5, 400, 4, 64, 0, seed=95,
                                                 output_idx_offset=[7, 1000]),
}


@pytest.mark.parametrize("compact", [False, True])
@pytest.mark.parametrize("parts", [1, 2, 3, 5])
@pytest.mark.parametrize("name", list(KEY_SHARD_CASES))
def test_key_shards_merge_to_the_whole_problem(orc, name, parts, compact):
    """Selecting in every key range with global indices and merging the lists gives the whole
    problem's output bit for bit (oracle on both sides, so this checks the range algebra)."""
    pb = KEY_SHARD_CASES[name]()
    whole = orc.topk(pb)
    lists = [orc.topk(shard.key_shard(pb, parts, r, compact)) for r in range(parts)]
    got = orc.merge_topk([x[0] for x in lists], [x[1] for x in lists], pb.topk)
    assert np.array_equal(got[0], whole[0]), name
    assert np.array_equal(got[1].view(np.uint32), whole[1].view(np.uint32)), name


def test_key_ranges_empty_for_every_sequence(orc):
    """More ranges than blocks: some ranges hold no key of any sequence (the compacted cache then
    keeps one placeholder block), select nothing, and the merge is still the whole selection."""
    pb = synthetic.paged([100, 40], 1, 4, 16, block_size=64, seed=97)
    whole = orc.topk(pb)
    parts = [shard.key_shard(pb, 6, r, compact=True) for r in range(6)]
    assert any(int(p.seqused_k.sum()) == 0 for p in parts)
    lists = [orc.topk(p) for p in parts]
    got = orc.merge_topk([x[0] for x in lists], [x[1] for x in lists], pb.topk)
    assert np.array_equal(got[0], whole[0])
    assert np.array_equal(got[1].view(np.uint32), whole[1].view(np.uint32))


def test_key_shard_rejects_what_it_cannot_split():
    with pytest.raises(ValueError):
        shard.key_shard(synthetic.tnd([5], [90], 4, 8, 3, seed=96), 2, 0)
    with pytest.raises(ValueError):
        shard.key_shard(KEY_SHARD_CASES["paged_decode"](), 2, 2)


def _oracle_run(pb):
    from oracle import oracle as orc_mod
    i, v, rc = orc_mod.default().topk(pb)
    assert rc == 0
    return torch.from_numpy(i), torch.from_numpy(v)


def _oracle_merge(gi, gv, topk):
    from oracle import oracle as orc_mod
    i, v = orc_mod.default().merge_topk(list(gi.numpy()), list(gv.numpy()), topk)
    return torch.from_numpy(i), torch.from_numpy(v)


def _key_rank_main(rank, world, init_file, result_file):
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank,
                            world_size=world)
    try:
        pb = KEY_SHARD_CASES["paged_decode"]()
        part = shard.key_shard(pb, world, rank)
        idx, val = shard.key_sharded_indexer(part, run=_oracle_run, merge=_oracle_merge)
        if rank == 0:
            torch.save((idx, val), result_file)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_merge_key_ranges(orc):
    """Two ranks each hold half of every sequence's keys, select with the oracle, all-gather the
    lists and merge: every rank ends with the whole rows' top-k."""
    world = 2
    with tempfile.TemporaryDirectory() as d:
        init_file = os.path.join(d, "init")
        result_file = os.path.join(d, "out.pt")
        mp.spawn(_key_rank_main, args=(world, init_file, result_file), nprocs=world, join=True)
        idx, val = torch.load(result_file)
    whole = orc.topk(KEY_SHARD_CASES["paged_decode"]())
    assert np.array_equal(idx.numpy(), whole[0])
    assert np.array_equal(val.numpy().view(np.uint32), whole[1].view(np.uint32))


@pytest.mark.gpu
def test_sharded_gpu_runs_are_bit_identical_to_the_whole_run():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_token_lightning_b200 import li
    pb = synthetic.bsnd(1, 1000, 1000, 64, 256, 3, seed=52)
    wi, wv = li.indexer(pb.to("cuda"))
    wi = wi.view(1000, -1).cpu()
    wv = wv.view(1000, -1).cpu()
    for r in range(4):
        for a, b in shard.zigzag_chunks(1000, 4, r):
            si, sv = li.indexer(shard.sub_problem(pb, a, b).to("cuda"))
            assert torch.equal(si.view(b - a, -1).cpu(), wi[a:b])
            assert torch.equal(sv.view(b - a, -1).cpu().view(torch.int32), wv[a:b].view(torch.int32))
