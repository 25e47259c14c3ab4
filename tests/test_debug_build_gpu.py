"""The bounds-checked build of the library (libli_debug.so, compiled with LI_DEBUG) on the
parity workloads.

In that build every computed shared- or global-memory index the kernels form is checked against
its buffer before the access; a failing check sets LI_DEVERR_BOUNDS in the status word and the
access is skipped (no trap). It is the stand-in for a memory checker: every call below must
finish with a clean status (the binding raises on any status bit), and its outputs must equal
the release library's bit for bit, since the checks change no arithmetic. The cases cover each
kernel and path: the tensor-core and CUDA-core score kernels, the register, long-row, exact and
split-row selections, the merge, fp8 inputs, compressed keys, the sparse attention and both
backward kernels.
"""
import numpy as np
import pytest
import torch

from sparse_attention_token_lightning_b200 import build, li, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return li.lib(), li.load(build.build_debug())


def _same(a, b):
    if a is None or b is None:
        return a is None and b is None
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)


def _both(libs, monkeypatch, fn):
    """fn() on the release library, then on the bounds-checked one."""
    rel, dbg = libs
    monkeypatch.setattr(li, "_lib", rel)
    a = fn()
    torch.cuda.synchronize()
    monkeypatch.setattr(li, "_lib", dbg)
    b = fn()                      # raises LiError if any status bit (LI_DEVERR_BOUNDS) is set
    torch.cuda.synchronize()
    monkeypatch.setattr(li, "_lib", rel)
    return a, b


INDEXER = {
    "tiny": lambda: synthetic.config("tiny"),
    "bsnd_causal_ragged": lambda: synthetic.bsnd(2, 300, 459, 64, 200, 3, seed=3),
    "tie_heavy_exact_path": lambda: synthetic.bsnd(1, 40, 333, 1, 64, 0, seed=4),
    "tnd_varlen": lambda: synthetic.tnd([1, 130, 77, 0, 256], [300, 130, 500, 9, 256], 64, 100,
                                        3, seed=7),
    "paged_bs64": lambda: synthetic.paged([700, 129, 1, 64], 3, 64, 128, block_size=64, seed=9),
    "paged_bs48_cuda_cores": lambda: synthetic.paged([333, 200], 2, 16, 40, block_size=48,
                                                     seed=11),
    "paged_bs1": lambda: synthetic.paged([37, 3], 1, 4, 8, block_size=1, seed=12),
    "topk8192_long_rows": lambda: synthetic.bsnd(1, 8, 9000, 2, 8192, 0, seed=14),
    "paged_decode_split_rows": lambda: synthetic.paged([5000, 3000, 100], 1, 64, 256,
                                                       block_size=64, seed=54),
    "fp8_bsnd": lambda: synthetic.quantized(synthetic.bsnd(2, 300, 459, 64, 200, 3, seed=3)),
    "compressed_tnd": lambda: synthetic.compressed(
        synthetic.tnd([200, 40, 1], [60, 70, 5], 64, 32, 3, seed=61), 4, [3, 1, 0]),
    "causal_prefill_full": lambda: synthetic.config("causal_prefill"),
}


@pytest.mark.parametrize("name", list(INDEXER))
def test_indexer_clean_and_identical(libs, monkeypatch, name):
    g = INDEXER[name]().to("cuda")
    (ia, va), (ib, vb) = _both(libs, monkeypatch, lambda: li.indexer(g))
    assert _same(ia, ib) and _same(va, vb)


def test_merge_clean_and_identical(libs, monkeypatch):
    rng = np.random.default_rng(5)
    n, rows, topk = 6, 9, 700
    idx = np.full((n, rows, topk), -1, dtype=np.int32)
    val = np.full((n, rows, topk), -np.inf, dtype=np.float32)
    for r in range(rows):
        pool = rng.permutation(n * topk * 2)[: n * topk].reshape(n, topk)
        for l in range(n):
            k = int(rng.integers(0, topk + 1))
            v = rng.standard_normal(k).astype(np.float32)
            j = pool[l, :k].astype(np.int32)
            o = np.lexsort((j, -v))
            idx[l, r, :k], val[l, r, :k] = j[o], v[o]
    ti, tv = torch.from_numpy(idx).cuda(), torch.from_numpy(val).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    (ia, va), (ib, vb) = _both(libs, monkeypatch,
                               lambda: li.merge_topk(ti, tv, 1024, device_status=status))
    assert _same(ia, ib) and _same(va, vb)
    assert int(status.item()) == 0


ATTN = {
    "g16_dm512_rope": lambda: synthetic.attn_bsnd(1, 300, 300, 16, 512, 64, 200, seed=1),
    "g20_dm384_nomask": lambda: synthetic.attn_bsnd(1, 64, 500, 20, 384, 64, 500, seed=4,
                                                    causal=False),
    "g16_paged_bs48": lambda: synthetic.attn_paged(
        synthetic.attn_bsnd(2, 100, 300, 16, 512, 64, 150, seed=6), 48, seed=1, spare_blocks=2),
}


@pytest.mark.parametrize("name", list(ATTN))
def test_sparse_attention_clean_and_identical(libs, monkeypatch, name):
    g = ATTN[name]().to("cuda")
    a, b = _both(libs, monkeypatch, lambda: li.sparse_attention(g))
    assert all(_same(x, y) for x, y in zip(a, b))


@pytest.mark.parametrize("kernel", ["tensor_cores", "cuda_cores"])
def test_kl_grad_clean_and_identical(libs, monkeypatch, kernel):
    if kernel == "cuda_cores":
        monkeypatch.setenv("LI_KL_KERNEL", "simple")
    g = synthetic.kl_bsnd(1, 300, 8, 512, 64, 32, 256, seed=142).to("cuda")
    a, b = _both(libs, monkeypatch, lambda: li.kl_grad(g))
    # bit-identical on the tensor-core path; the CUDA-core path adds d_key_index and d_weights
    # with atomics (any order)
    for i, (x, y) in enumerate(zip(a, b)):
        if kernel == "cuda_cores" and i in (2, 3):
            assert torch.allclose(x, y, rtol=1e-5, atol=1e-6)
        else:
            assert _same(x, y)
