"""The indexer backward with the KL loss (li_kl_grad) against the oracle: loss, d_query_index,
d_key_index and d_weights on causal BSND problems with and without rope parts.

Tolerance: the device works in fp32 (exp and log of fp32 arguments, sums over up to topk keys
and over the rows that share a key, added atomically), the oracle in fp64 from the same inputs.
The loss must agree to 1e-4 relative; each gradient element to 2e-3 of the largest magnitude of
that gradient (plus 1e-6), which covers fp32 accumulation over a few thousand terms."""
import numpy as np
import pytest
import torch

from sparse_attention_token_lightning_b200 import li, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    li.lib()


CASES = {
    "small_rope": lambda: synthetic.kl_bsnd(2, 40, 4, 64, 16, 8, 16, seed=140),
    "h64_no_rope": lambda: synthetic.kl_bsnd(1, 100, 16, 128, 0, 64, 64, seed=141),
    "mla_like": lambda: synthetic.kl_bsnd(1, 300, 8, 512, 64, 32, 256, seed=142),
    "topk_512": lambda: synthetic.kl_bsnd(1, 700, 4, 64, 0, 16, 512, seed=143),
}


def check(orc, kp, got):
    want = orc.kl_grad(kp)
    loss = float(got[0].item())
    assert abs(loss - want[0]) <= 1e-4 * abs(want[0]) + 1e-5, (loss, want[0])
    for name, g, o in zip(("d_qi", "d_ki", "d_w"), got[1:], want[1:]):
        g = g.double().cpu().numpy()
        bound = 2e-3 * np.abs(o).max() + 1e-6
        err = np.abs(g - o).max()
        assert err <= bound, f"{name}: max error {err:.3g} above {bound:.3g}"


@pytest.mark.parametrize("name", list(CASES))
def test_kl_grad_matches_the_oracle(orc, name):
    kp = CASES[name]()
    got = li.kl_grad(kp.to("cuda"))
    torch.cuda.synchronize()
    check(orc, kp, got)


def test_rows_without_selection_contribute_nothing(orc):
    kp = synthetic.kl_bsnd(1, 50, 4, 64, 0, 8, 16, seed=144)
    si = kp.sparse_indices.clone()
    si[0, 10:20] = -1
    kp = kp.replace(sparse_indices=si)
    got = li.kl_grad(kp.to("cuda"))
    check(orc, kp, got)
    assert torch.count_nonzero(got[1][0, 10:20]) == 0 and torch.count_nonzero(got[3][0, 10:20]) == 0


def test_out_of_range_selection_reported():
    kp = synthetic.kl_bsnd(1, 30, 2, 64, 0, 4, 8, seed=145)
    si = kp.sparse_indices.clone()
    si[0, 5, 0, 0] = 30
    with pytest.raises(li.LiError) as e:
        li.kl_grad(kp.replace(sparse_indices=si).to("cuda"))
    assert "0x2" in str(e.value)
