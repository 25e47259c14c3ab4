"""The indexer backward with the KL loss (li_kl_grad) against the oracle: loss, d_query_index,
d_key_index and d_weights on causal BSND problems with and without rope parts.

Shapes with Dm a multiple of 64 (up to 512), Dr 0 or 64, G <= 32 and H <= 64 run on the
tensor-core kernel (scores and both gradient products on tcgen05, dS carried as a bf16 hi + lo
pair, d_key_index summed per key in a fixed order: bit-reproducible); other shapes on the
CUDA-core kernel (d_key_index by atomic adds).

Tolerance: the device works in fp32 (exp and log of fp32 arguments, sums over up to topk keys
and over the rows that share a key), the oracle in fp64 from the same inputs; the hi + lo pair
keeps 16 significant bits of dS. The loss must agree to 1e-4 relative; each gradient element to
2e-3 of the largest magnitude of that gradient (plus 1e-6), which covers fp32 accumulation over a
few thousand terms."""
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
    # the benchmark's head counts and dims on a short causal problem; two batches
    "g16_h64_two_batches": lambda: synthetic.kl_bsnd(2, 160, 16, 512, 64, 64, 100, seed=146),
    # 20 main heads (N = 32), 40 indexer heads (N = 48), topk not a multiple of 64
    "g20_h40": lambda: synthetic.kl_bsnd(1, 200, 20, 256, 64, 40, 90, seed=147),
}
TC_CASES = ("h64_no_rope", "mla_like", "topk_512", "g16_h64_two_batches", "g20_h40")


def _workspace_bytes(kp):
    import ctypes
    a = li.make_kl_args(kp)
    n = ctypes.c_size_t(0)
    li._check(li.lib().li_kl_grad_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


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


@pytest.mark.parametrize("name", TC_CASES)
def test_tensor_core_path_is_taken(name):
    """Eligible shapes carry the per-CTA partial d_key_index buffer in their workspace (the
    tensor-core path); the CUDA-core path needs only the status word and the row losses."""
    kp = CASES[name]().to("cuda")
    rows = kp.w.shape[0] * kp.w.shape[1]
    assert _workspace_bytes(kp) > 256 + (rows * 4 + 255) // 256 * 256


def test_d_key_index_is_bit_reproducible():
    kp = synthetic.kl_bsnd(1, 256, 16, 512, 64, 64, 128, seed=148).to("cuda")
    a = li.kl_grad(kp)
    b = li.kl_grad(kp)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))


@pytest.mark.parametrize("name", ["mla_like", "g20_h40"])
def test_tensor_core_and_cuda_core_paths_agree(orc, name, monkeypatch):
    kp = CASES[name]()
    a = li.kl_grad(kp.to("cuda"))
    monkeypatch.setenv("LI_KL_KERNEL", "simple")
    b = li.kl_grad(kp.to("cuda"))
    check(orc, kp, b)
    want = orc.kl_grad(kp)
    for name_, x, y, o in zip(("d_qi", "d_ki", "d_w"), a[1:], b[1:], want[1:]):
        bound = 2e-3 * np.abs(o).max() + 1e-6
        assert (x - y).abs().max().item() <= bound, name_
