"""The split merge (li_merge_topk) and the key-range-sharded indexer on one GPU.

Tie-heavy sorted lists are merged on the device and compared with the oracle's merge bit for bit.
The key-range-sharded indexer is emulated on one device (every range selected in turn, then one
merge) and compared with the oracle on the whole, unsplit problem."""
import numpy as np
import pytest
import torch

import parity
from sparse_attention_token_lightning_b200 import li, shard, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    li.lib()


def sorted_lists(n_lists, rows, topk_in, seed, levels=7, ragged=True):
    """Per-row lists in the selection's order with unique indices across lists, scores drawn
    from `levels` values (many ties within and across lists) and random padded tails."""
    g = np.random.default_rng(seed)
    idx = np.full((n_lists, rows, topk_in), -1, dtype=np.int32)
    val = np.full((n_lists, rows, topk_in), -np.inf, dtype=np.float32)
    for r in range(rows):
        pool = g.permutation(n_lists * topk_in * 4)[: n_lists * topk_in].reshape(n_lists, topk_in)
        for l in range(n_lists):
            n = int(g.integers(0, topk_in + 1)) if ragged and g.random() < 0.3 else topk_in
            v = (g.integers(-levels, levels + 1, n) / 4).astype(np.float32)
            j = pool[l, :n].astype(np.int32)
            order = np.lexsort((j, -v))
            idx[l, r, :n], val[l, r, :n] = j[order], v[order]
    return idx, val


@pytest.mark.parametrize("n_lists,rows,topk_in,topk_out", [
    (2, 40, 64, 64), (4, 33, 300, 128), (8, 17, 2048, 2048), (16, 5, 512, 8192), (3, 9, 100, 1),
    (1, 20, 200, 150), (5, 3, 8192, 8192)])
def test_merge_matches_the_oracle_bit_for_bit(orc, n_lists, rows, topk_in, topk_out):
    idx, val = sorted_lists(n_lists, rows, topk_in, seed=n_lists * 1000 + rows)
    want_i, want_v = orc.merge_topk(list(idx), list(val), topk_out)
    gi, gv = li.merge_topk(torch.from_numpy(idx).cuda(), torch.from_numpy(val).cuda(), topk_out)
    torch.cuda.synchronize()
    assert np.array_equal(gi.cpu().numpy(), want_i)
    assert np.array_equal(gv.cpu().numpy().view(np.uint32), want_v.view(np.uint32))
    gi2, gv2 = li.merge_topk(torch.from_numpy(idx).cuda(), torch.from_numpy(val).cuda(), topk_out,
                             return_value=False)
    assert gv2 is None and torch.equal(gi2, gi)


def test_merge_reports_an_unsorted_list():
    idx, val = sorted_lists(2, 4, 50, seed=7, levels=1000, ragged=False)
    idx[1, 2, [3, 4]] = idx[1, 2, [4, 3]]          # two distinct entries swapped
    val[1, 2, [3, 4]] = val[1, 2, [4, 3]]
    with pytest.raises(li.LiError) as e:
        li.merge_topk(torch.from_numpy(idx).cuda(), torch.from_numpy(val).cuda(), 50)
    assert "0x40" in str(e.value)


def test_merge_reports_a_valid_entry_after_padding():
    idx, val = sorted_lists(2, 3, 40, seed=8)
    idx[0, 1, -1], val[0, 1, -1] = 10**6, -100.0
    idx[0, 1, -2], val[0, 1, -2] = -1, -np.inf
    with pytest.raises(li.LiError):
        li.merge_topk(torch.from_numpy(idx).cuda(), torch.from_numpy(val).cuda(), 40)


def run_key_sharded(pb, parts):
    """Every key range selected in turn on one device, then one merge."""
    outs = [li.indexer(shard.key_shard(pb, parts, r).to("cuda")) for r in range(parts)]
    gi = torch.stack([o[0] for o in outs])
    gv = torch.stack([o[1] for o in outs])
    idx, val = li.merge_topk(gi, gv, pb.topk)
    torch.cuda.synchronize()
    return parity.as_rows(idx, pb.topk), parity.as_rows(val, pb.topk)


KEY_SHARDED = {
    "paged_decode_long": lambda: synthetic.paged([30000, 5000, 64, 1], 1, 64, 2048, block_size=64,
                                                 seed=100),
    "paged_causal_rows": lambda: synthetic.paged([4000, 2500], 4, 32, 256, block_size=64,
                                                 seed=101),
    "bsnd_causal_seqused": lambda: synthetic.bsnd(2, 8, 3000, 16, 300, 3, seed=102,
                                                  seqused_k=[3000, 2100]),
    "paged_tnd_q_nomask": lambda: synthetic.paged([3000, 900], 0, 16, 128, block_size=16,
                                                  seed=103, mask_mode=0, layout_q="TND",
                                                  lens_q=[3, 2]),
}


@pytest.mark.parametrize("parts", [2, 8])
@pytest.mark.parametrize("name", list(KEY_SHARDED))
def test_key_sharded_indexer_matches_the_oracle(orc, name, parts):
    pb = KEY_SHARDED[name]()
    gi, gv = run_key_sharded(pb, parts)
    parity.check(orc, pb, gi, gv, label=f"{name} / {parts} ranges")


@pytest.mark.parametrize("parts", [3, 8])
def test_key_sharded_integer_inputs_bit_exact(orc, parts):
    pb = synthetic.paged([6000, 1000, 3], 2, 16, 512, block_size=64, seed=104, integer=True)
    gi, gv = run_key_sharded(pb, parts)
    parity.check(orc, pb, gi, gv, exact=True, label=f"integer / {parts} ranges")


def test_long_row_decode_full_size(orc):
    """The benchmark's one-row decode over 2^20 keys, whole and split into 8 key ranges (the
    8-GPU layout, emulated on one device), against the oracle."""
    pb = synthetic.config("long_row_decode")
    wi, wv = li.indexer(pb.to("cuda"))
    torch.cuda.synchronize()
    parity.check(orc, pb, parity.as_rows(wi, pb.topk), parity.as_rows(wv, pb.topk), label="whole")
    gi, gv = run_key_sharded(pb, 8)
    parity.check(orc, pb, gi, gv, label="8 key ranges")


# ---- rows long enough that li_indexer cuts their selection into key pieces -----------------------

SPLIT_ROWS = {
    "decode_3_rows": lambda: synthetic.paged([200000, 70000, 40000], 1, 64, 2048, block_size=64,
                                             seed=110),
    "causal_4_rows": lambda: synthetic.bsnd(1, 4, 70000, 16, 512, 3, seed=111),
    "topk8192": lambda: synthetic.paged([100000], 1, 8, 8192, block_size=64, seed=112),
    "ragged_pieces": lambda: synthetic.paged([40000, 33000], 1, 8, 300,
                                                          block_size=32, seed=113),
}


@pytest.mark.parametrize("name", list(SPLIT_ROWS))
def test_split_row_selection_matches_the_oracle(orc, name):
    pb = SPLIT_ROWS[name]()
    plan = li.li_plan(li.make_args(pb.to("cuda")))
    assert plan["select_pieces"] > 1, plan
    g = pb.to("cuda")
    ws = li.empty_workspace(li.make_args(g), "cuda")
    idx, val = li.indexer(g, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[8:12].view(torch.int32).item()) == 0      # no piece left the bucket paths
    parity.check(orc, pb, parity.as_rows(idx, pb.topk), parity.as_rows(val, pb.topk), label=name)
    idx2, val2 = li.indexer(g, return_value=False)
    assert val2 is None and torch.equal(idx2, idx)


def test_split_row_selection_integer_inputs_bit_exact(orc):
    pb = synthetic.paged([90000, 40000], 2, 16, 1024, block_size=64, seed=114, integer=True)
    assert li.li_plan(li.make_args(pb.to("cuda")))["select_pieces"] > 1
    gi, gv = li.indexer(pb.to("cuda"))
    torch.cuda.synchronize()
    parity.check(orc, pb, parity.as_rows(gi, pb.topk), parity.as_rows(gv, pb.topk), exact=True,
                 label="integer split rows")


def test_host_pipeline_matches_single_calls():
    """The pipelined host-to-host runner gives every step the same outputs as one li.indexer call
    on that step's problem (different inputs per step, more steps than buffer sets)."""
    probs = [synthetic.bsnd(2, 300, 459, 64, 200, 3, seed=120 + i) for i in range(5)]
    pipe = li.HostPipeline(probs[0], "cuda")
    inputs = [{f: getattr(pb, f).pin_memory() for f in pipe.fields} for pb in probs]
    shape = li.out_shape(probs[0])
    outputs = [(torch.empty(shape, dtype=torch.int32).pin_memory(),
                torch.empty(shape, dtype=torch.float32).pin_memory()) for _ in probs]
    pipe.run(inputs, outputs)
    pipe.synchronize()
    pipe.check()
    for pb, (hi, hv) in zip(probs, outputs):
        ri, rv = li.indexer(pb.to("cuda"))
        assert torch.equal(hi, ri.cpu()) and torch.equal(hv, rv.cpu())
