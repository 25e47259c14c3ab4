"""The parity checker itself, on the CPU: the oracle's own output passes it, and outputs with the
mistakes a selection or merge kernel could plausibly make fail it in tolerance mode (where the
index sets alone would not catch them):

* two indices swapped while the values stay in place (a mis-paired stage slot);
* an index replaced by its neighbouring key (an off-by-one in the key position);
* two entries swapped, indices and values together (out of selection order);
* two bit-equal values whose indices come in the wrong order (tie order);
* a value replaced by the score of another selected key.
"""
import numpy as np
import pytest

import parity
from sparse_attention_token_lightning_b200 import synthetic


def _oracle_rows(orc, pb):
    idx, val, rc = orc.bind(pb).topk()
    assert rc == 0
    return idx.copy(), val.copy()


@pytest.fixture(scope="module")
def case(orc):
    pb = synthetic.bsnd(1, 48, 300, 8, 40, 3, seed=71)
    return pb, _oracle_rows(orc, pb)


def _far_pair(val_row, m, tol):
    """Two valid positions whose values differ by far more than the tolerance."""
    assert val_row[0] - val_row[m - 1] > 10 * tol
    return 0, m - 1


def test_oracle_output_passes(orc, case):
    pb, (gi, gv) = case
    assert parity.check(orc, pb, gi, gv, label="oracle") == pb.rows
    parity.check_pair(orc, pb, gi, gv, gi.copy(), gv.copy(), label="oracle pair")


def _row_with_window(pb, gi, at_least):
    for r in range(gi.shape[0] - 1, -1, -1):
        if (gi[r] >= 0).sum() >= at_least:
            return r
    raise AssertionError("no row long enough")


@pytest.mark.parametrize("mistake", ["swap_indices", "neighbour_key", "swap_entries",
                                     "value_of_other_key"])
def test_planted_mistakes_fail(orc, case, mistake):
    pb, (gi0, gv0) = case
    gi, gv = gi0.copy(), gv0.copy()
    r = _row_with_window(pb, gi, 30)
    m = int((gi[r] >= 0).sum())
    a, b = _far_pair(gv[r], m, 1e-2)
    if mistake == "swap_indices":
        gi[r, a], gi[r, b] = gi[r, b], gi[r, a]
    elif mistake == "neighbour_key":
        # the key next to the top one, outside the selected set if possible
        chosen = set(gi[r, :m].tolist())
        alt = next(j for j in (gi[r, a] + 1, gi[r, a] - 1) if j not in chosen and j >= 0)
        gi[r, a] = alt
    elif mistake == "swap_entries":
        gi[r, [a, b]] = gi[r, [b, a]]
        gv[r, [a, b]] = gv[r, [b, a]]
    else:
        gv[r, b] = gv[r, a]
        gv[r, :m] = np.sort(gv[r, :m])[::-1]          # keep the values sorted
    with pytest.raises(AssertionError):
        parity.check(orc, pb, gi, gv, label=mistake)
    with pytest.raises(AssertionError):
        parity.check_pair(orc, pb, gi0, gv0, gi, gv, label=mistake)


def test_tie_order_is_checked(orc):
    """All-negative weights with integer inputs: many keys score exactly +0, so the order of
    bit-equal values (lower index first) decides; reversing two tied entries must fail."""
    pb = synthetic.bsnd(1, 16, 200, 4, 64, 0, seed=72, integer=True)
    pb = pb.replace(w=-pb.w.abs())
    gi, gv = _oracle_rows(orc, pb)
    parity.check(orc, pb, gi, gv, label="ties")
    r = 0
    m = int((gi[r] >= 0).sum())
    zeros = np.nonzero(gv[r, :m] == 0.0)[0]
    assert zeros.size >= 2
    a, b = zeros[0], zeros[1]
    gi[r, [a, b]] = gi[r, [b, a]]
    with pytest.raises(AssertionError):
        parity.check(orc, pb, gi, gv, label="ties reversed")
