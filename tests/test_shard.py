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
