"""li_indexer_noalloc: the indexer for callers that may not allocate device memory (plugin
enqueue steps without an allocator, runtimes that forbid allocation after start-up, real-time
loops). It runs the same deterministic kernels as li_indexer with a caller-provided workspace, so
its outputs must equal li_indexer's bit for bit.

The calls go through the C ABI. Two different problems run back to back, then the first one
again, so each call starts from scratch contents left by a different problem; outputs are
poisoned before each call so stale results cannot pass. A call on invalid device data must hand
its error bits to the caller's status word, and the next clean call must clear them. This file
is collected last.
"""
import numpy as np
import pytest
import torch

import parity
from sparse_attention_token_lightning_b200 import li, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    li.lib()


def _noalloc(g, expect_bits=0):
    args = li.make_args(g)
    idx = torch.full(li.out_shape(g), -7, dtype=torch.int32, device="cuda")
    val = torch.full(li.out_shape(g), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    li.li_indexer_noalloc(args, idx, val, status)
    st, bits = li.li_check_status(status)
    if expect_bits:
        assert st == 6 and bits & expect_bits, (st, bits, li.li_last_error_string())
    else:
        assert st == li.LI_OK and bits == 0, (st, bits, li.li_last_error_string())
    return parity.as_rows(idx, g.topk), parity.as_rows(val, g.topk)


def test_noalloc_matches_li_indexer_on_consecutive_calls(orc):
    problems = [synthetic.bsnd(1, 700, 900, 64, 256, 3, seed=41, name="a"),
                synthetic.tnd([300, 5, 120], [300, 800, 640], 16, 64, 3, seed=42, name="b")]
    refs = []
    for pb in problems:
        g = pb.to("cuda")
        i, v = li.indexer(g)
        refs.append((parity.as_rows(i, pb.topk), parity.as_rows(v, pb.topk)))
    for k in (0, 1, 0):
        pb = problems[k]
        gi, gv = _noalloc(pb.to("cuda"))
        assert np.array_equal(gi, refs[k][0]), f"noalloc {pb.name}: indices differ"
        assert np.array_equal(gv.view(np.uint32), refs[k][1].view(np.uint32)), \
            f"noalloc {pb.name}: values differ"
    # and both match the oracle
    for k, pb in enumerate(problems):
        parity.check(orc, pb, refs[k][0], refs[k][1], rows=parity.sample_rows(pb, 64, seed=3),
                     label=f"li_indexer {pb.name}")


def test_noalloc_reports_device_data_errors():
    """A block-table entry outside the cache sets LI_DEVERR_TABLE in the shared scratch's status
    word; the call copies it to the caller's status word, and the next clean call (which clears
    the scratch header) reports nothing."""
    pb = synthetic.paged([300, 130], 1, 16, 32, block_size=16, seed=44)
    pb.block_table[1, 3] = pb.num_blocks + 5
    _noalloc(pb.to("cuda"), expect_bits=li.DEVERR_TABLE)
    _noalloc(synthetic.paged([300, 130], 1, 16, 32, block_size=16, seed=44).to("cuda"))


def test_noalloc_rejects_problems_above_the_scratch_size():
    pb = synthetic.bsnd(1, 4096, 4096, 64, 2048, 3, seed=43).to("cuda")  # ~64 MB of scores
    args = li.make_args(pb)
    idx = torch.empty(li.out_shape(pb), dtype=torch.int32, device="cuda")
    val = torch.empty(li.out_shape(pb), dtype=torch.float32, device="cuda")
    with pytest.raises(li.LiError) as ei:
        li.li_indexer_noalloc(args, idx, val, None)
    assert ei.value.status == 3
    assert "static scratch" in str(ei.value)
