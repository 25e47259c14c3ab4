"""Property tests (hypothesis) of the host-side partitions: key ranges and zig-zag row chunks
cover their index space exactly once, in order, with the promised alignment and caps."""
from hypothesis import given, settings, strategies as st

from sparse_attention_token_lightning_b200 import shard


@settings(max_examples=300, deadline=None)
@given(L2=st.integers(0, 1 << 20), parts=st.integers(1, 16), align=st.sampled_from([1, 8, 16, 64, 128]),
       cap=st.one_of(st.none(), st.integers(-5, 1 << 20)))
def test_key_ranges_tile_the_keys(L2, parts, align, cap):
    rng = shard.key_ranges(L2, parts, align, cap)
    assert len(rng) == parts
    assert rng[0][0] == 0 and rng[-1][1] == L2
    for (a, b), (c, d) in zip(rng, rng[1:]):
        assert a <= b == c <= d
    for a, _b in rng[1:]:
        assert a % align == 0 or a == L2
        if cap is not None:
            assert a <= max(0, cap) or a == L2


@settings(max_examples=300, deadline=None)
@given(rows=st.integers(1, 5000), world=st.integers(1, 16))
def test_zigzag_chunks_cover_every_row_once(rows, world):
    seen = []
    for r in range(world):
        for a, b in shard.zigzag_chunks(rows, world, r):
            assert 0 <= a < b <= rows
            seen.extend(range(a, b))
    assert sorted(seen) == list(range(rows))


@settings(max_examples=200, deadline=None)
@given(data=st.data(), n_lists=st.integers(1, 6), kin=st.integers(1, 12), kout=st.integers(1, 40))
def test_oracle_merge_is_the_sorted_union(orc, data, n_lists, kin, kout):
    """The oracle's merge equals Python's sort of all valid entries (score descending, index
    ascending) cut to kout and padded, for random lists with many equal scores."""
    import numpy as np
    pool = iter(data.draw(st.permutations(range(n_lists * kin))))
    idx = np.full((n_lists, 1, kin), -1, dtype=np.int32)
    val = np.full((n_lists, 1, kin), -np.inf, dtype=np.float32)
    entries = []
    for l in range(n_lists):
        n = data.draw(st.integers(0, kin))
        ent = sorted(((float(data.draw(st.integers(-3, 3))) / 2, next(pool)) for _ in range(n)),
                     key=lambda t: (-t[0], t[1]))
        for e, (v, j) in enumerate(ent):
            idx[l, 0, e], val[l, 0, e] = j, v
        entries += ent
    want = sorted(entries, key=lambda t: (-t[0], t[1]))[:kout]
    want += [(-np.inf, -1)] * (kout - len(want))
    gi, gv = orc.merge_topk(list(idx), list(val), kout)
    assert gi[0].tolist() == [j for _, j in want]
    assert gv[0].tolist() == [v for v, _ in want]
