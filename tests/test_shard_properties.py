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
