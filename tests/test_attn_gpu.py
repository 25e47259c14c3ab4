"""GPU parity of the sparse attention over the selected keys (li_sparse_attention) against the
oracle (orc_sparse_attention), through the C ABI.

Tolerances, derived from the kernel's arithmetic, per (row, head), with D = Dm + Dr, u = 2^-24,
V = max |k[s, d]| over the row's selected keys and A = max over those keys of sum_d |q_d k_d|
(the dot product with its terms' magnitudes):
  * every score x = scale (q . k) is an fp32 sum of exact bf16 products: |dx| <= ex = scale D u A;
  * softmax_max: |dm| <= ex;
  * softmax_sum = sum of fp32 exponentials (each within 2 ulp, the sum within n ulp) of x - m:
    |dl| <= l (2 ex + (n + 8) 2^-23);
  * out: the weights enter the value product rounded to bf16 (relative 2^-9) while the
    normaliser sums the unrounded weights, so out moves by at most 2^-9 V; the score errors
    add 2 ex V: |do| <= (2^-8 + 2 ex) V.
Bit-exact is not expected (the tensor cores' summation order is not the oracle's). Small cases
with few selected keys make each key's weight large, so a dropped, repeated or misplaced key
shows far above these bounds; the statistics catch the same on long lists.
"""
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


def _bounds(ap, rows):
    """(ex [n, G], V [n], counts [n]) of the given rows, from the inputs in float64."""
    B, S1, G, Dm = ap.q.shape
    q = ap.q.reshape(B * S1, G, Dm).double()
    k = ap.k.reshape(-1, Dm).double()
    qr = None if ap.q_rope is None else ap.q_rope.reshape(B * S1, G, -1).double()
    kr = None if ap.k_rope is None else ap.k_rope.reshape(-1, ap.k_rope.shape[-1]).double()
    D = Dm + (0 if qr is None else qr.shape[-1])
    sel = ap.sparse_indices.reshape(B * S1, -1)
    S2 = ap.k.shape[1]
    ex, V, cnt = [], [], []
    for r in rows:
        s = sel[r]
        s = s[(s >= 0) & (s < S2)].long() + int(ap.key_base[r])
        cnt.append(int(s.numel()))
        if s.numel() == 0:
            ex.append(np.zeros(G))
            V.append(0.0)
            continue
        A = q[r].abs() @ k[s].abs().T                     # [G, n]
        if qr is not None:
            A = A + qr[r].abs() @ kr[s].abs().T
        ex.append((ap.scale * D * 2.0 ** -24 * A.max(dim=1).values).numpy())
        V.append(float(k[s].abs().max()))
    return np.array(ex), np.array(V), np.array(cnt)


def check_attention(orc, ap_cpu, out, smax, ssum, rows=None, label=""):
    """Compare device outputs (full tensors) with the oracle on `rows` (all when None)."""
    B, S1, G, Dm = ap_cpu.q.shape
    rows = np.arange(B * S1) if rows is None else np.asarray(rows)
    o_out, o_max, o_sum = orc.sparse_attention(ap_cpu.rows(rows))
    g_out = out.reshape(B * S1, G, Dm).cpu().double().numpy()[rows]
    g_max = smax.reshape(B * S1, G).cpu().double().numpy()[rows]
    g_sum = ssum.reshape(B * S1, G).cpu().double().numpy()[rows]
    ex, V, cnt = _bounds(ap_cpu, rows)
    for n, r in enumerate(rows):
        where = f"{label} row {int(r)}"
        if cnt[n] == 0:
            assert np.all(g_out[n] == 0.0), f"{where}: output of a row without keys"
            assert np.all(np.isneginf(g_max[n])) and np.all(g_sum[n] == 0.0), where
            continue
        dm = np.abs(g_max[n] - o_max[n])
        assert np.all(dm <= ex[n] + 1e-6), f"{where}: softmax_max off by {dm.max():.3g}"
        tl = o_sum[n] * (2 * ex[n] + (cnt[n] + 8) * 2.0 ** -23) + 1e-6
        dl = np.abs(g_sum[n] - o_sum[n])
        assert np.all(dl <= tl), f"{where}: softmax_sum off by {(dl / o_sum[n]).max():.3g} (rel)"
        to = (2.0 ** -8 + 2 * ex[n][:, None]) * V[n] + 1e-6
        do = np.abs(g_out[n] - o_out[n])
        bad = np.argwhere(do > to)
        assert bad.size == 0, (f"{where}: out off by {do.max():.3g} at head/dim "
                               f"{bad[0].tolist()} (tol {to.max():.3g})")


def run(ap):
    g = ap.to("cuda")
    out, smax, ssum = li.sparse_attention(g)
    torch.cuda.synchronize()
    return out, smax, ssum


def _interleaved(seed=6):
    """Selections with padding in the middle, repeated keys, rows that select nothing and a
    topk that is not a multiple of the 128-key tile."""
    ap = synthetic.attn_bsnd(2, 40, 300, 16, 256, 64, 170, seed=seed)
    sel = ap.sparse_indices.clone()
    g = torch.Generator().manual_seed(seed)
    holes = torch.rand(sel.shape, generator=g) < 0.3
    sel[holes] = -1
    sel[0, 5, 0, :] = -1                      # no key at all
    sel[1, 7, 0, :] = -1
    sel[1, 7, 0, 150] = 3                     # one key, at the last tile
    sel[0, 9, 0, 10:20] = sel[0, 9, 0, 0]     # one key ten more times
    return ap.replace(sparse_indices=sel)


SMALL = {
    # G, Dm, Dr; several tiles with a ragged last one, causal windows from 1 key up
    "g16_dm512_rope": lambda: synthetic.attn_bsnd(1, 300, 300, 16, 512, 64, 200, seed=1),
    # heads padded to 16, one 128-dim pair, no rope, two batches
    "g5_dm128": lambda: synthetic.attn_bsnd(2, 130, 140, 5, 128, 0, 64, seed=2),
    # 32 MMA columns, two pairs
    "g32_dm256_rope": lambda: synthetic.attn_bsnd(1, 100, 400, 32, 256, 64, 300, seed=3),
    # 20 heads (N = 32), three pairs, no mask, four tiles
    "g20_dm384_nomask": lambda: synthetic.attn_bsnd(1, 64, 500, 20, 384, 64, 500, seed=4,
                                                    causal=False),
    "topk1": lambda: synthetic.attn_bsnd(1, 50, 50, 8, 128, 64, 1, seed=5),
    "interleaved_padding": _interleaved,
    # large scale: peaked softmax whose running max moves often across tiles (rescaling)
    "peaked": lambda: synthetic.attn_bsnd(1, 80, 1000, 16, 512, 64, 1000, seed=7, scale=0.4,
                                          causal=False),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_attention_parity(orc, name):
    ap = SMALL[name]()
    out, smax, ssum = run(ap)
    check_attention(orc, ap, out, smax, ssum, label=name)


def test_statistics_match_the_backward_generators(orc):
    """synthetic.kl_bsnd computes the main attention's statistics over the selected keys in
    torch float64, independently of the oracle: the kernel's softmax_max / softmax_sum must
    match them, and its output must match the oracle."""
    kp = synthetic.kl_bsnd(1, 256, 16, 512, 64, 64, 200, seed=8)
    out, smax, ssum = run(kp)
    ref_max = kp.softmax_max.reshape(-1, 16).double().numpy()
    ref_sum = kp.softmax_sum.reshape(-1, 16).double().numpy()
    g_max = smax.reshape(-1, 16).cpu().double().numpy()
    g_sum = ssum.reshape(-1, 16).cpu().double().numpy()
    assert np.abs(g_max - ref_max).max() <= 1e-3
    assert (np.abs(g_sum - ref_sum) / ref_sum).max() <= 1e-3
    ap = synthetic.AttnProblem(name="kl", q=kp.q, k=kp.k, q_rope=kp.q_rope, k_rope=kp.k_rope,
                               sparse_indices=kp.sparse_indices, key_base=kp.key_base,
                               scale=kp.scale)
    check_attention(orc, ap, out, smax, ssum, rows=np.arange(0, 256, 7), label="kl problem")


def test_full_size_sampled(orc):
    ap = synthetic.attn_config("sparse_attention")
    rows = sorted({0, 1, 127, 128, 2046, 2047, 2048, 4095} |
                  set(np.random.default_rng(3).choice(4096, 12, replace=False).tolist()))
    out, smax, ssum = run(ap)
    check_attention(orc, ap, out, smax, ssum, rows=rows, label="sparse_attention")


def test_deterministic_reruns():
    ap = synthetic.attn_bsnd(1, 256, 256, 16, 512, 64, 128, seed=9).to("cuda")
    a = li.sparse_attention(ap)
    b = li.sparse_attention(ap)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))


PAGED = {
    # (dense problem, block size, spare blocks)
    "g16_dm512_rope_bs64": (lambda: SMALL["g16_dm512_rope"](), 64, 3),
    "g5_dm128_bs1": (lambda: SMALL["g5_dm128"](), 1, 7),
    "g20_dm384_nomask_bs48": (lambda: SMALL["g20_dm384_nomask"](), 48, 0),
    "interleaved_padding_bs16": (lambda: _interleaved(11), 16, 2),
}


@pytest.mark.parametrize("name", list(PAGED))
def test_paged_keys_match_dense_keys(orc, name):
    """Keys in a paged cache (PA_BSND, blocks in a seeded random order) give the same outputs as
    the dense keys, bit for bit (the same rows are gathered in the same order), and the oracle's
    values on the dense problem."""
    make, bs, spare = PAGED[name]
    ap = make()
    pp = synthetic.attn_paged(ap, bs, seed=5, spare_blocks=spare)
    a = run(ap)
    b = run(pp)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))
    check_attention(orc, ap, *b, label=name)


def test_paged_bad_block_table_entry_reported(orc):
    ap = synthetic.attn_bsnd(1, 30, 70, 4, 128, 0, 20, seed=12)
    pp = synthetic.attn_paged(ap, 16, seed=2)
    bt = pp.block_table.clone()
    bt[0, 1] = bt.max() + 5                          # positions 16..31 point past the cache
    pp = pp.replace(block_table=bt)
    g = pp.to("cuda")
    a = li.make_attn_args(g)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 30, 4, 128), dtype=torch.float32, device="cuda")
    sm = torch.empty((1, 1, 30, 4), dtype=torch.float32, device="cuda")
    ss = torch.empty((1, 1, 30, 4), dtype=torch.float32, device="cuda")
    li.li_sparse_attention(a, ws, out, sm, ss)
    st, bits = li.li_check_status(ws)
    assert st == 6 and bits & li.DEVERR_TABLE
    # the affected keys select nothing: the rows equal the oracle on the selection without them
    sel = ap.sparse_indices.clone()
    sel[(sel >= 16) & (sel < 32)] = -1
    check_attention(orc, ap.replace(sparse_indices=sel), out, sm, ss, label="bad table")


def test_out_of_range_index_reported():
    ap = synthetic.attn_bsnd(1, 20, 30, 4, 128, 0, 16, seed=10)
    ap.sparse_indices[0, 3, 0, 2] = 30                 # == S2: selects nothing, reported
    g = ap.to("cuda")
    a = li.make_attn_args(g)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 20, 4, 128), dtype=torch.float32, device="cuda")
    sm = torch.empty((1, 1, 20, 4), dtype=torch.float32, device="cuda")
    ss = torch.empty((1, 1, 20, 4), dtype=torch.float32, device="cuda")
    li.li_sparse_attention(a, ws, out, sm, ss)
    st, bits = li.li_check_status(ws)
    assert st == 6 and bits & li.DEVERR_LENGTHS
