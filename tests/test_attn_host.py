"""Host side of the sparse attention without a GPU: the paged-key generator keeps every key
row where the block table says it is, the oracle gives the paged and the dense problems the same
answer through that mapping, and the argument builder fills the paged fields of li_attn_args."""
import numpy as np
import torch

from sparse_attention_token_lightning_b200 import li, synthetic


def test_paged_cache_holds_every_key_where_the_table_points():
    ap = synthetic.attn_bsnd(3, 12, 37, 4, 128, 64, 9, seed=21)
    for bs in (1, 5, 16, 40):
        pp = synthetic.attn_paged(ap, bs, seed=bs, spare_blocks=3)
        bt = pp.block_table
        assert pp.s2 == 37 and bt.shape == (3, -(-37 // bs))
        assert pp.k.shape[0] == 3 * bt.shape[1] + 3 and pp.k.shape[1] == bs
        # every physical block is used at most once
        used = bt.reshape(-1)
        assert torch.unique(used).numel() == used.numel()
        for b in range(3):
            for v in range(37):
                blk, off = int(bt[b, v // bs]), v % bs
                assert torch.equal(pp.k[blk, off], ap.k[b, v])
                assert torch.equal(pp.k_rope[blk, off], ap.k_rope[b, v])


def test_oracle_agrees_on_the_dense_form_of_a_paged_problem(orc):
    """The oracle works on logical key rows; rebuilding them from the paged cache through the
    table gives back the dense problem, hence the same attention."""
    ap = synthetic.attn_bsnd(2, 20, 50, 4, 128, 0, 12, seed=22)
    pp = synthetic.attn_paged(ap, 7, seed=3)
    bt = pp.block_table
    rebuilt = torch.stack([torch.stack([pp.k[int(bt[b, v // 7]), v % 7] for v in range(50)])
                           for b in range(2)])
    assert torch.equal(rebuilt, ap.k)
    a = orc.sparse_attention(ap)
    b = orc.sparse_attention(ap.replace(k=rebuilt))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_attention_args_carry_the_paged_fields():
    ap = synthetic.attn_bsnd(2, 8, 30, 16, 256, 64, 6, seed=23)
    a = li.make_attn_args(ap)
    assert a.layout_k == li.LAYOUTS["BSND"] and not a.block_table
    assert (a.s2, a.num_blocks, a.block_size, a.block_table_stride) == (30, 0, 0, 0)
    pp = synthetic.attn_paged(ap, 8, seed=1, spare_blocks=2)
    a = li.make_attn_args(pp)
    assert a.layout_k == li.LAYOUTS["PA_BSND"]
    assert a.block_table == pp.block_table.data_ptr()
    assert (a.s2, a.num_blocks, a.block_size, a.block_table_stride) == (30, 2 * 4 + 2, 8, 4)
    assert (a.batch, a.s1, a.G, a.Dm, a.Dr, a.topk) == (2, 8, 16, 256, 64, 6)
