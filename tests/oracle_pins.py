"""Pins for the CPU oracle: checks against facts fixed by the pages and by mathematics, not by
the oracle itself.

Each ``pin_*`` takes an ``Oracle`` and raises AssertionError when it disagrees. They are run on
the real oracle by test_oracle_pins.py and on every planted-mistake build by
test_oracle_mutants.py, which requires each planted mistake to fail at least one of them.
"""
import numpy as np
import torch

import golden_cases
from sparse_attention_token_lightning_b200 import synthetic

INT32_MAX = 2**31 - 1


def _bits(v):
    return np.asarray(v, dtype=np.float32).view(np.uint32)


def _assert_same(a, b, what=""):
    ia, va = a[0], a[1]
    ib, vb = b[0], b[1]
    assert np.array_equal(ia, ib), f"{what}: indices differ"
    assert np.array_equal(_bits(va), _bits(vb)), f"{what}: values differ"


def pin_golden(orc):
    """Hand-worked fixtures under tests/golden (each cites the passages it follows)."""
    for pb, ei, ev in golden_cases.all_cases():
        i, v, rc = orc.topk(pb, check=False)
        assert rc == 0, pb.name
        assert np.array_equal(i, ei), f"{pb.name}: indices {i.tolist()} != {ei.tolist()}"
        assert np.array_equal(_bits(v), _bits(ev)), f"{pb.name}: values {v.tolist()} != {ev.tolist()}"


def _torch_desc(scores64, topk):
    """Reference top-k of a float64 score row by a library sort: values rounded to fp32 once,
    stable descending sort (equal values keep ascending index order)."""
    s32 = torch.as_tensor(scores64).to(torch.float32)
    s32 = torch.where(s32 == 0, torch.zeros_like(s32), s32)
    vals, idx = torch.sort(s32, descending=True, stable=True)
    m = min(topk, s32.numel())
    out_i = np.full(topk, -1, dtype=np.int32)
    out_v = np.full(topk, -np.inf, dtype=np.float32)
    out_i[:m] = idx[:m].numpy()
    out_v[:m] = vals[:m].numpy()
    return out_i, out_v


def pin_single_head_reduces_to_relu_matmul(orc):
    """N1 = 1 and w = 1: the score is ReLU(q . k), a float64 matmul plus ReLU (library calls),
    and the selection is a stable descending sort. topk covers zero scores, so the tie order of
    the ReLU zeros is pinned too. No mask."""
    pb = synthetic.bsnd(1, 6, 200, 1, 150, mask_mode=0, seed=11, name="n1")
    pb.w = torch.ones_like(pb.w)
    idx, val, _ = orc.topk(pb)
    q64 = pb.q.to(torch.float64).reshape(6, 128)
    k64 = pb.k.to(torch.float64).reshape(200, 128)
    ref = torch.relu(q64 @ k64.T)
    for r in range(6):
        ei, ev = _torch_desc(ref[r], 150)
        assert np.array_equal(idx[r], ei), f"row {r}: indices"
        assert np.array_equal(_bits(val[r]), _bits(ev)), f"row {r}: values"


def pin_one_hot_weights_pick_a_head(orc):
    """w[t] = e_h selects head h alone: I[t,j] = ReLU(q[t,h] . k_j) (float64 matmul + ReLU)."""
    pb = synthetic.bsnd(1, 8, 96, 4, 96, mask_mode=0, seed=12, name="onehot")
    heads = [t % 4 for t in range(8)]
    w = torch.zeros(1, 8, 4)
    for t, h in enumerate(heads):
        w[0, t, h] = 1.0
    pb.w = w.to(torch.bfloat16)
    idx, val, _ = orc.topk(pb)
    q64 = pb.q.to(torch.float64).reshape(8, 4, 128)
    k64 = pb.k.to(torch.float64).reshape(96, 128)
    for t, h in enumerate(heads):
        ei, ev = _torch_desc(torch.relu(q64[t, h] @ k64.T), 96)
        assert np.array_equal(idx[t], ei), f"row {t}: indices"
        assert np.array_equal(_bits(val[t]), _bits(ev)), f"row {t}: values"


def pin_linear_in_weights(orc):
    """I is linear in w: I(w1 + w2) = I(w1) + I(w2). Integer-valued inputs keep every sum exact,
    so the identity holds bit for bit in fp64."""
    base = synthetic.bsnd(1, 5, 40, 4, 8, mask_mode=0, seed=13, integer=True, name="lin")
    g = torch.Generator().manual_seed(5)
    w1 = torch.randint(-2, 3, base.w.shape, generator=g).to(torch.bfloat16)
    w2 = torch.randint(-2, 3, base.w.shape, generator=g).to(torch.bfloat16)
    for r in range(5):
        s1 = orc.scores(base.replace(w=w1), r)
        s2 = orc.scores(base.replace(w=w2), r)
        s12 = orc.scores(base.replace(w=(w1.float() + w2.float()).to(torch.bfloat16)), r)
        assert np.array_equal(s1 + s2, s12), f"row {r}: not linear in w"
        s_neg = orc.scores(base.replace(w=(-w1.float()).to(torch.bfloat16)), r)
        assert np.array_equal(s_neg, -s1), f"row {r}: not odd in w"


def pin_head_permutation_invariance(orc):
    """Permuting the heads of q and w together leaves every output unchanged (the head sum is a
    sum, and integer-valued inputs make it exact)."""
    pb = synthetic.bsnd(2, 16, 24, 6, 10, mask_mode=3, seed=14, integer=True, name="perm")
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    pp = pb.replace(q=pb.q[:, :, perm].contiguous(), w=pb.w[:, :, perm].contiguous())
    _assert_same(orc.topk(pb), orc.topk(pp), "head permutation")


def pin_key_permutation_equivariance(orc):
    """Without a mask, permuting the keys permutes the scores: the score multiset of every row
    is unchanged and score(j) follows its key."""
    pb = synthetic.bsnd(1, 4, 50, 4, 50, mask_mode=0, seed=15, name="kperm")
    perm = torch.randperm(50, generator=torch.Generator().manual_seed(3))
    pp = pb.replace(k=pb.k[:, perm].contiguous())
    for r in range(4):
        a = orc.scores(pb, r)
        b = orc.scores(pp, r)
        assert np.array_equal(b, a[perm.numpy()]), f"row {r}"


def _logical_varlen(seed=16):
    """Three batches with L1 != L2 and one empty query batch, as TND/TND."""
    lens_q, lens_k = [5, 1, 0, 7], [9, 4, 3, 12]
    return synthetic.tnd(lens_q, lens_k, 3, 6, mask_mode=3, seed=seed, name="lv"), lens_q, lens_k


def pin_layouts_agree(orc):
    """The same logical data laid out as TND keys, as a paged cache with a shuffled block table,
    and as one dense BSND batch per sequence gives the same outputs bit for bit."""
    pt, lens_q, lens_k = _logical_varlen()
    out_t = orc.topk(pt)
    cu_q = np.cumsum([0] + lens_q)
    cu_k = np.cumsum([0] + lens_k)
    # paged: block size 4, blocks in a shuffled order, two spare blocks
    bs = 4
    nb = [(L + bs - 1) // bs for L in lens_k]
    NB = sum(nb) + 2
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(9)).tolist()
    cache = torch.zeros(NB, bs, 1, 128, dtype=torch.bfloat16)
    table = torch.full((len(lens_k), max(nb)), -1, dtype=torch.int32)
    pos = 0
    for b, L in enumerate(lens_k):
        for blk in range(nb[b]):
            phys = perm[pos]
            pos += 1
            table[b, blk] = phys
            for s in range(bs):
                j = blk * bs + s
                if j < L:
                    cache[phys, s, 0] = pt.k[cu_k[b] + j, 0]
    pp = pt.replace(layout_k="PA_BSND", k=cache, block_table=table,
                    seqused_k=torch.tensor(lens_k, dtype=torch.int32), cu_seqlens_k=None,
                    num_blocks=NB, block_size=bs, k_len=0)
    _assert_same(out_t, orc.topk(pp), "TND vs PA_BSND")
    # dense, one batch at a time
    for b in range(len(lens_q)):
        if lens_q[b] == 0:
            continue
        qb = pt.q[cu_q[b]:cu_q[b + 1]].unsqueeze(0).contiguous()
        wb = pt.w[cu_q[b]:cu_q[b + 1]].unsqueeze(0).contiguous()
        kb = pt.k[cu_k[b]:cu_k[b + 1]].unsqueeze(0).contiguous()
        pd = synthetic.Problem(name="dense", q=qb, k=kb, w=wb, topk=pt.topk, batch=1,
                               q_len=lens_q[b], k_len=lens_k[b], n_heads=pt.n_heads,
                               layout_q="BSND", layout_k="BSND", mask_mode=3)
        i_d, v_d, _ = orc.topk(pd)
        assert np.array_equal(out_t[0][cu_q[b]:cu_q[b + 1]], i_d), f"batch {b}: TND vs BSND idx"
        assert np.array_equal(_bits(out_t[1][cu_q[b]:cu_q[b + 1]]), _bits(v_d)), f"batch {b}"


def pin_single_query_row_sees_all_keys(orc):
    """Right-down causal with one query row (decode) keeps every key: equals the unmasked result.
    With S1 = S2 the last row also sees every key and the first row sees only key 0."""
    pb = synthetic.bsnd(2, 1, 37, 4, 40, mask_mode=3, seed=17, name="dec")
    _assert_same(orc.topk(pb), orc.topk(pb.replace(mask_mode=0)), "decode mask 3 vs 0")
    sq = synthetic.bsnd(1, 20, 20, 4, 25, mask_mode=3, seed=18, name="sq")
    i3, v3, _ = orc.topk(sq)
    i0, v0, _ = orc.topk(sq.replace(mask_mode=0))
    assert np.array_equal(i3[-1], i0[-1]) and np.array_equal(_bits(v3[-1]), _bits(v0[-1]))
    assert i3[0, 0] == 0 and (i3[0, 1:] == -1).all()


def pin_zero_query_ties_by_index(orc):
    """q = 0 makes every score exactly 0: each row returns keys 0, 1, ... in order, values +0."""
    pb = synthetic.bsnd(1, 8, 30, 4, 12, mask_mode=3, seed=19, name="zero")
    pb.q = torch.zeros_like(pb.q)
    idx, val, _ = orc.topk(pb)
    off = 30 - 8
    for t in range(8):
        m = min(12, t + off + 1)
        assert np.array_equal(idx[t, :m], np.arange(m)), f"row {t}"
        assert (_bits(val[t, :m]) == 0).all(), f"row {t}: zero scores must be +0"
        assert (idx[t, m:] == -1).all()


def pin_negative_weights_zero_is_positive(orc):
    """All weights negative: every score is <= 0, keys whose head scores are all <= 0 score zero,
    and that zero is +0; zeros rank first, by index."""
    pb = synthetic.bsnd(1, 6, 64, 2, 64, mask_mode=0, seed=20, integer=True, name="negw")
    pb.w = -pb.w.abs()
    idx, val, _ = orc.topk(pb)
    for t in range(6):
        v = val[t]
        assert (v <= 0).all()
        zeros = v == 0
        assert (_bits(v[zeros]) == 0).all(), f"row {t}: -0 in the output"
        nz = int(zeros.sum())
        assert nz > 0
        assert np.array_equal(idx[t, :nz], np.sort(idx[t, :nz]))


def pin_offset_overflow_is_an_error(orc):
    """An output_idx_offset that pushes an index past INT32_MAX is reported (the pages forbid it)."""
    pb = synthetic.bsnd(1, 2, 3, 1, 3, mask_mode=0, seed=21, name="ovf",
                        output_idx_offset=[INT32_MAX - 1])
    _i, _v, rc = orc.topk(pb, check=False)
    assert rc == 2
    ok = pb.replace(output_idx_offset=torch.tensor([INT32_MAX - 2], dtype=torch.int32))
    i2, _v2, rc2 = orc.topk(ok, check=False)
    assert rc2 == 0 and i2.max() == INT32_MAX


def check_row_invariants(orc, pb, idx, val, rows=None):
    """Invariants of any correct output: m = min(topk, |window|) valid entries then padding;
    indices unique and inside the window; values non-increasing and equal to the fp32 score at
    their index; every selected key beats every unselected one (score, then lower index)."""
    rows = range(pb.rows) if rows is None else rows
    for n, r in enumerate(rows):
        s = orc.scores(pb, r)
        hi = s.size
        m = min(pb.topk, hi)
        ii, vv = idx[n], val[n]
        assert (ii[m:] == -1).all() and np.isneginf(vv[m:]).all(), f"row {r}: padding"
        off = 0
        if pb.output_idx_offset is not None:
            _hi, b, _i = orc.row_info(pb, r)
            off = int(pb.output_idx_offset[b])
        sel = ii[:m].astype(np.int64) - off
        assert (sel >= 0).all() and (sel < hi).all(), f"row {r}: index outside window"
        assert np.unique(sel).size == m, f"row {r}: duplicate index"
        s32 = s.astype(np.float32)
        s32[s32 == 0] = 0.0
        assert np.array_equal(_bits(vv[:m]), _bits(s32[sel])), f"row {r}: value != score"
        assert (np.diff(vv[:m]) <= 0).all(), f"row {r}: not sorted"
        if m < hi:
            mask = np.ones(hi, dtype=bool)
            mask[sel] = False
            un = np.nonzero(mask)[0]
            kth_v, kth_i = vv[m - 1], sel[m - 1]
            worse = (s32[un] < kth_v) | ((s32[un] == kth_v) & (un > kth_i))
            assert worse.all(), f"row {r}: an unselected key beats the k-th"


def pin_invariants_on_random_problems(orc):
    """The invariants on small random problems of every layout and both masks."""
    cases = [
        synthetic.bsnd(2, 33, 70, 4, 16, mask_mode=3, seed=22, name="b3"),
        synthetic.bsnd(1, 20, 20, 3, 7, mask_mode=0, seed=23, name="b0"),
        synthetic.tnd([3, 9, 1], [12, 9, 30], 5, 8, mask_mode=3, seed=24, name="t3"),
        synthetic.paged([17, 5, 40], 2, 4, 12, block_size=8, mask_mode=3, seed=25, name="p3",
                        spare_blocks=3),
        synthetic.bsnd(1, 12, 40, 4, 9, mask_mode=3, seed=26, integer=True, name="int"),
    ]
    for pb in cases:
        idx, val, _ = orc.topk(pb)
        check_row_invariants(orc, pb, idx, val)


def pin_compressed_window_counts_whole_blocks(orc):
    """Compressed keys under the right-down mask: a row keeps exactly the keys whose r original
    tokens all lie in the uncompressed window of the same row over the L2*r + res original
    tokens, so its window is floor(uncompressed window / r). The uncompressed window comes from
    the (separately pinned) uncompressed path on a problem with L2*r + res keys."""
    cases = [(5, 7, 4, [2]), (9, 3, 2, [1]), (6, 11, 3, [0]), (12, 5, 5, [4]), (1, 6, 4, [3])]
    for L1, L2c, r, res in cases:
        comp = synthetic.compressed(synthetic.bsnd(1, L1, L2c, 2, 4, 3, seed=70), r, res)
        full = synthetic.bsnd(1, L1, L2c * r + res[0], 2, 4, 3, seed=70)
        bc, bf = orc.bind(comp), orc.bind(full)
        for i in range(L1):
            hc, _, _ = bc.row_info(i)
            hf, _, _ = bf.row_info(i)
            assert hc == hf // r, (L1, L2c, r, res, i, hc, hf)
    # ratio 1 without residuals is the uncompressed problem, outputs included
    pb = synthetic.bsnd(2, 30, 40, 4, 16, 3, seed=71)
    a = orc.topk(pb)
    b = orc.topk(synthetic.compressed(pb, 1, [0, 0]))
    _assert_same(a[0], b[0], "indices")
    _assert_same(_bits(a[1]), _bits(b[1]), "values")
    # the unmasked window ignores the compression
    pb0 = synthetic.bsnd(1, 8, 10, 2, 4, 0, seed=72)
    for i in range(8):
        assert orc.bind(synthetic.compressed(pb0, 4, [3])).row_info(i)[0] == 10


def pin_fp16_decoding(orc):
    """fp16 queries decode as IEEE binary16 (numpy's float16 is the reference): with one head of
    dimension 1, w = 1 and a single key k = 1, each row's only score is ReLU(q). The patterns
    cover subnormals, normals of every exponent and negative values."""
    pos = np.arange(0, 0x7C00, 5, dtype=np.uint16)              # +0 .. largest finite
    bits = np.concatenate([pos, pos[::7] | np.uint16(0x8000)])   # and some negative ones
    n = len(bits)
    q = torch.from_numpy(bits.view(np.int16).copy()).view(torch.float16).reshape(1, n, 1, 1)
    pb = synthetic.Problem(name="fp16_decode", q=q, k=torch.ones(1, 1, 1, 1, dtype=torch.float16),
                           w=torch.ones(1, n, 1, dtype=torch.bfloat16), topk=1, batch=1, q_len=n,
                           k_len=1, n_heads=1, head_dim=1, mask_mode=0, max_seqlen_q=n,
                           max_seqlen_k=1)
    idx, val, _ = orc.topk(pb)
    want = np.maximum(bits.view(np.float16).astype(np.float32), np.float32(0))
    assert np.array_equal(idx[:, 0], np.zeros(n, dtype=np.int32))
    _assert_same(_bits(val[:, 0]), _bits(want), "fp16 decode")


def pin_dtype_encodings_agree(orc):
    """Integer-valued q, k (in -2..2) and w (in +-1/2, +-1, +-2) are exact in bf16, fp16 and
    fp32, so every encoding of the same values gives the same outputs, bit for bit."""
    base = synthetic.bsnd(2, 40, 70, 8, 24, 3, seed=73, integer=True)
    ref = orc.topk(base)
    for qk, w in [("fp16", "fp32"), ("fp16", "fp16"), ("bf16", "fp32"), ("fp16", "bf16")]:
        got = orc.topk(synthetic.with_dtypes(base, qk, w))
        _assert_same(ref[0], got[0], f"indices {qk}/{w}")
        _assert_same(_bits(ref[1]), _bits(got[1]), f"values {qk}/{w}")


def pin_pages_example_shape(orc):
    """The pages' worked example shape (B=2, S1=64, N1=16, topk=32) with 32 keys and mask 3:
    rows i < 32 see no key (i + S2 - S1 < 0) and row i >= 32 sees i - 31 keys."""
    pb = synthetic.config("pages_example")
    idx, val, _ = orc.topk(pb)
    assert idx.shape == (128, 32)
    for r in range(128):
        i = r % 64
        valid = int((idx[r] >= 0).sum())
        assert valid == max(0, min(32, i - 31)), f"row {r}: {valid} valid entries"


def pin_fp8_decoding(orc):
    """fp8 e4m3 codes decode as the OCP E4M3 format (torch's float8_e4m3fn is the reference): one
    head of dimension 1, w = 1, one key of value 1 and unit scales, so each row's only score is
    ReLU(q). Every code but the two NaNs is covered."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    n = len(codes)
    q = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).reshape(1, n, 1, 1)
    one = torch.ones(1, 1, 1, 1).to(torch.float8_e4m3fn)
    pb = synthetic.Problem(name="fp8_decode", q=q, k=one, w=torch.ones(1, n, 1, dtype=torch.bfloat16),
                           topk=1, batch=1, q_len=n, k_len=1, n_heads=1, head_dim=1, mask_mode=0,
                           max_seqlen_q=n, max_seqlen_k=1, q_descale=torch.ones(1, n, 1),
                           k_descale=torch.ones(1, 1))
    idx, val, _ = orc.topk(pb)
    want = np.maximum(q.reshape(-1).float().numpy(), np.float32(0))
    assert np.array_equal(idx[:, 0], np.zeros(n, dtype=np.int32))
    _assert_same(_bits(val[:, 0]), _bits(want), "fp8 decode")


def pin_fp8_unit_scales_match_bf16(orc):
    """Integer-valued q and k are exact in e4m3; with every scale 1 the fp8 problem is the bf16
    problem, bit for bit (dense, varlen and paged keys)."""
    for base in (synthetic.bsnd(2, 40, 70, 8, 24, 3, seed=74, integer=True),
                 synthetic.tnd([5, 30], [40, 64], 4, 16, 3, seed=75, integer=True),
                 synthetic.paged([90, 20], 2, 8, 32, block_size=16, seed=76, integer=True)):
        _assert_same(orc.topk(base)[:2], orc.topk(synthetic.quantized(base, unit_scales=True))[:2],
                     base.name)


def pin_fp8_scales_act_as_dequantization(orc):
    """Small integer codes times power-of-two scales are exact in fp16, so an fp8 problem with
    per-(row, head) q scales and per-key k scales must equal, bit for bit, the fp16 problem that
    holds the products: the scales multiply the codes, q's by row and head, k's by key row."""
    g = torch.Generator().manual_seed(77)
    for base in (synthetic.bsnd(2, 30, 50, 4, 20, 3, seed=78, integer=True),
                 synthetic.paged([70, 33], 2, 4, 16, block_size=16, seed=79, integer=True)):
        qs = 2.0 ** torch.randint(-2, 3, base.w.shape, generator=g).float()
        ks = 2.0 ** torch.randint(-2, 3, base.k.shape[:-2] if base.k.dim() == 4 else
                                  base.k.shape[:-1], generator=g).float()
        fp8 = base.replace(q=base.q.float().to(torch.float8_e4m3fn),
                           k=base.k.float().to(torch.float8_e4m3fn), q_descale=qs, k_descale=ks)
        fp16 = base.replace(q=(base.q.float() * qs.unsqueeze(-1)).half(),
                            k=(base.k.float() * ks.reshape(base.k.shape[:-1]).unsqueeze(-1)).half())
        _assert_same(orc.topk(fp16)[:2], orc.topk(fp8)[:2], base.name)


class _KLArrays:
    """A backward-with-KL-loss problem held as float64 numpy arrays (shapes as KLProblem)."""

    def __init__(self, rng, B=1, S=5, G=2, Dm=6, Dr=3, H=3, Di=4, topk=3):
        r = lambda *sh: rng.standard_normal(sh)
        self.q, self.k = r(B, S, G, Dm), r(B, S, 1, Dm)
        self.q_rope, self.k_rope = r(B, S, G, Dr), r(B, S, 1, Dr)
        self.qi, self.ki, self.w = r(B, S, H, Di), r(B, S, 1, Di), r(B, S, H)
        idx = np.full((B, S, 1, topk), -1, dtype=np.int32)
        for b in range(B):
            for i in range(S):
                m = min(topk, i + 1)
                idx[b, i, 0, :m] = rng.permutation(i + 1)[:m]
        self.sparse_indices = idx
        self.key_base = np.repeat(np.arange(B, dtype=np.int64) * S, S)
        self.softmax_max = rng.uniform(0.5, 2.0, (B, 1, S, G))
        self.softmax_sum = rng.uniform(1.0, 3.0, (B, 1, S, G))
        self.scale = 0.3


def pin_kl_gradients_match_finite_differences(orc):
    """The backward's gradients are the derivatives of its loss: central differences of the
    loss in every element of query_index, key_index and weights (a key selected by several rows
    included) match d_query_index, d_key_index and d_weights."""
    rng = np.random.default_rng(90)
    for kw in (dict(), dict(B=2, S=4, G=1, Dr=0, H=2, topk=4)):
        kp = _KLArrays(rng, **kw)
        if kw.get("Dr") == 0:
            kp.q_rope = kp.k_rope = None
        _loss, dqi, dki, dw = orc.kl_grad(kp)
        eps = 1e-6
        for name, grad in (("qi", dqi), ("ki", dki), ("w", dw)):
            arr = getattr(kp, name)
            for pos in np.ndindex(arr.shape):
                keep = arr[pos]
                arr[pos] = keep + eps
                lp = orc.kl_grad(kp)[0]
                arr[pos] = keep - eps
                lm = orc.kl_grad(kp)[0]
                arr[pos] = keep
                fd = (lp - lm) / (2 * eps)
                assert abs(fd - grad[pos]) <= 1e-6 + 1e-5 * abs(fd), (name, pos, fd, grad[pos])


def pin_kl_target_is_the_attention_softmax(orc):
    """With one main-attention head, its true softmax statistics and zero weights (so the
    indexer's distribution is uniform over the n selected keys), each row's loss is the KL
    divergence of the attention softmax over the selected keys from uniform: log n - H(p), p
    computed by scipy's softmax and H by scipy's entropy."""
    from scipy.special import softmax
    from scipy.stats import entropy
    kp = synthetic.kl_bsnd(1, 9, 1, 16, 4, 2, 5, seed=91, Di=8)
    kp = kp.replace(w=torch.zeros_like(kp.w))
    want = 0.0
    for i in range(9):
        sel = kp.sparse_indices[0, i, 0]
        sel = sel[sel >= 0].long()
        x = (kp.q[0, i].double() @ kp.k[0, sel, 0].double().T +
             kp.q_rope[0, i].double() @ kp.k_rope[0, sel, 0].double().T)[0].numpy() * kp.scale
        p = softmax(x)
        want += np.log(len(p)) - entropy(p)
    loss, dqi, dki, dw = orc.kl_grad(kp)
    # the forward statistics were rounded to fp32: the head's P sums to 1 within ~1e-7
    assert abs(loss - want) <= 1e-6 * max(1.0, abs(want)), (loss, want)


def pin_kl_target_normalised_over_selected_keys(orc):
    """p is renormalised over each row's selected keys, so scaling every head's softmax_sum of a
    row by one factor changes nothing, while scaling one head's alone reweights the heads."""
    rng = np.random.default_rng(92)
    kp = _KLArrays(rng)
    base = orc.kl_grad(kp)
    kp.softmax_sum[0, 0, 2, :] *= 3.0
    same = orc.kl_grad(kp)
    assert abs(same[0] - base[0]) <= 1e-9 * abs(base[0])
    for a, b in zip(base[1:], same[1:]):
        assert np.allclose(a, b, rtol=1e-9, atol=1e-12)
    kp.softmax_sum[0, 0, 2, 0] *= 5.0
    assert abs(orc.kl_grad(kp)[0] - base[0]) > 1e-6


def pin_kl_loss_is_nonnegative(orc):
    """A sum of KL divergences is never negative (bf16 problems of several sizes)."""
    for seed, (S, G, H, topk) in enumerate([(12, 4, 8, 6), (30, 2, 4, 16), (7, 8, 1, 3)]):
        loss = orc.kl_grad(synthetic.kl_bsnd(1, S, G, 32, 8, H, topk, seed=93 + seed, Di=16))[0]
        assert loss >= 0.0, loss


def pin_attention_matches_scipy_softmax(orc):
    """Attention over the selected keys: for every row and head, scipy's softmax of the scaled
    dot products (with the rope parts) weights the selected key rows (values = keys), its max
    and sum of exponentials are the forward statistics, and one selected key returns that key."""
    from scipy.special import logsumexp, softmax
    kp = synthetic.kl_bsnd(2, 12, 3, 16, 8, 2, 5, seed=95, Di=8)
    out, smax, ssum = orc.sparse_attention(kp)
    q, k = kp.q.double().numpy(), kp.k.double().numpy()
    qr, kr = kp.q_rope.double().numpy(), kp.k_rope.double().numpy()
    for b in range(2):
        for i in range(12):
            sel = kp.sparse_indices[b, i, 0].numpy()
            sel = sel[sel >= 0]
            x = (q[b, i] @ k[b, sel, 0].T + qr[b, i] @ kr[b, sel, 0].T) * kp.scale
            r = b * 12 + i
            assert np.allclose(out[r], softmax(x, axis=1) @ k[b, sel, 0], rtol=1e-12, atol=1e-12)
            assert np.allclose(smax[r], x.max(axis=1), rtol=1e-14, atol=0)
            assert np.allclose(np.log(ssum[r]) + smax[r], logsumexp(x, axis=1), rtol=1e-12)
            if len(sel) == 1:
                assert np.allclose(out[r], np.repeat(k[b, sel, 0], 3, axis=0))


def pin_attention_statistics_feed_the_backward(orc):
    """The backward's generator takes the main attention's statistics over the selected keys (in
    torch, fp64, rounded to fp32); the oracle's attention gives the same statistics."""
    kp = synthetic.kl_bsnd(1, 20, 4, 32, 8, 2, 6, seed=96, Di=8)
    _out, smax, ssum = orc.sparse_attention(kp)
    assert np.allclose(smax, kp.softmax_max.reshape(20, 4).double().numpy(), rtol=1e-6, atol=1e-6)
    assert np.allclose(ssum, kp.softmax_sum.reshape(20, 4).double().numpy(), rtol=1e-6)


def pin_selected_key_order_does_not_matter(orc):
    """Sums over the selected keys cannot depend on the order of sparse_indices: shuffling every
    row's entries (padding included) leaves the attention, its statistics, the loss and all
    gradients unchanged up to fp64 rounding."""
    kp = synthetic.kl_bsnd(2, 10, 3, 16, 8, 4, 6, seed=98, Di=8)
    g = torch.Generator().manual_seed(99)
    si = kp.sparse_indices.clone()
    for b in range(2):
        for i in range(10):
            si[b, i, 0] = si[b, i, 0][torch.randperm(6, generator=g)]
    sh = kp.replace(sparse_indices=si)
    for a, b in zip(orc.sparse_attention(kp), orc.sparse_attention(sh)):
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    la, lb = orc.kl_grad(kp), orc.kl_grad(sh)
    assert abs(la[0] - lb[0]) <= 1e-12 * abs(la[0])
    for a, b in zip(la[1:], lb[1:]):
        assert np.allclose(a, b, rtol=1e-10, atol=1e-12)


def _key_range(pb, s, e, mask_mode):
    """Keys [s, e) of every batch of a dense BSND problem, indices shifted back to global by
    output_idx_offset = s (written out here, independently of the library's shard helpers)."""
    n = e - s
    return pb.replace(name=f"{pb.name}[k{s}:{e}]", k=pb.k[:, s:e].contiguous(), k_len=n,
                      max_seqlen_k=n, mask_mode=mask_mode,
                      output_idx_offset=torch.full((pb.batch,), s, dtype=torch.int32))


def pin_key_range_merge_equals_whole_row(orc):
    """Selection is over the whole window of a row, so splitting the keys into disjoint ranges,
    selecting in each with global indices and merging the lists must give the whole row's
    top-k bit for bit: decode rows (one query row sees every key under mask 3), rows without a
    mask, ranges shorter than topk (padded lists), and causal rows whose window covers every
    range but the last."""
    cases = [
        (synthetic.bsnd(3, 1, 700, 16, 100, 3, seed=80), [0, 128, 333, 700], [0, 0, 3]),
        (synthetic.bsnd(1, 5, 400, 8, 64, 0, seed=81), [0, 30, 250, 400], [0, 0, 0]),
        (synthetic.bsnd(2, 4, 300, 4, 120, 3, seed=82, integer=True), [0, 100, 200, 300],
         [0, 0, 3]),
        (synthetic.bsnd(2, 6, 260, 8, 200, 3, seed=83), [0, 128, 250, 260], [0, 0, 3]),
    ]
    for pb, cuts, masks in cases:
        whole = orc.topk(pb)
        lists = [orc.topk(_key_range(pb, a, b, m)) for a, b, m in zip(cuts, cuts[1:], masks)]
        got = orc.merge_topk([x[0] for x in lists], [x[1] for x in lists], pb.topk)
        _assert_same(whole, got, pb.name)


def pin_merge_brute_force(orc):
    """Tiny lists with many equal scores across lists: the merge equals Python's sort of all
    valid (score, index) pairs by score descending, then index ascending."""
    g = np.random.default_rng(84)
    for n_lists, rows, kin, kout in [(2, 3, 5, 4), (4, 5, 6, 9), (3, 2, 7, 30), (1, 4, 8, 3)]:
        pool = g.permutation(1000)[: n_lists * rows * kin].reshape(n_lists, rows, kin)
        idx = np.full((n_lists, rows, kin), -1, dtype=np.int32)
        val = np.full((n_lists, rows, kin), -np.inf, dtype=np.float32)
        for l in range(n_lists):
            for r in range(rows):
                n = int(g.integers(0, kin + 1))
                ent = sorted(((float(g.integers(-3, 4)) / 2, int(pool[l, r, e])) for e in range(n)),
                             key=lambda t: (-t[0], t[1]))
                for e, (v, j) in enumerate(ent):
                    idx[l, r, e], val[l, r, e] = j, v
        got_i, got_v = orc.merge_topk(list(idx), list(val), kout)
        for r in range(rows):
            ent = sorted(((float(val[l, r, e]), int(idx[l, r, e])) for l in range(n_lists)
                          for e in range(kin) if idx[l, r, e] >= 0), key=lambda t: (-t[0], t[1]))
            ent = ent[:kout] + [(-np.inf, -1)] * max(0, kout - len(ent))
            assert got_i[r].tolist() == [j for _, j in ent], (n_lists, r)
            assert got_v[r].tolist() == [v for v, _ in ent], (n_lists, r)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
