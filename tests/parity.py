"""Comparison of the CUDA path's outputs with the CPU oracle.

Tolerance (the indexer's accuracy target): per entry
    |value_gpu - value_oracle| <= 2e-3 * max_j |I[t, j]| + 1e-4
position-wise on the sorted lists, where max_j runs over the row's window. Every returned entry
is also tied to its own key: the index lies in the row's window and the value is within the same
tolerance of the oracle's exact score I[t, index]; and the list is in selection order (values
non-increasing, indices increasing among bit-equal values). The index sets must be equal except
for keys whose exact oracle score lies within that tolerance of the row's k-th score (near-ties
may legitimately swap). The count of valid entries and the padding are exact. With
integer-valued inputs every score is exact in fp32 and the outputs must match bit for bit.
"""
import numpy as np

TOL_REL = 2e-3
TOL_ABS = 1e-4


def _bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def _check_entries(where, gi, gv, m, off, hi, scores, tol):
    """Entries [0, m) of one output row: each index inside the window [off, off + hi), distinct,
    and (with values) each value within tol of the oracle's exact score of its own index, in
    selection order (value descending, then index ascending among bit-equal values)."""
    j = gi[:m].astype(np.int64) - off
    bad = np.nonzero((j < 0) | (j >= hi))[0]
    assert bad.size == 0, f"{where}: indices {gi[bad[:5]].tolist()} outside the window"
    assert np.unique(j).size == m, f"{where}: duplicate indices"
    if gv is None:
        return
    err = np.abs(gv[:m].astype(np.float64) - scores[j])
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"{where}: value at position {int(bad[0])} is {float(gv[bad[0]]):.6g} "
                           f"but key {int(gi[bad[0]])} scores {float(scores[j[bad[0]]]):.6g} "
                           f"(tol {tol:.3g})")
    v = gv[:m]
    down = v[1:] < v[:-1]
    tie = (v[1:] == v[:-1]) & (gi[1:m] > gi[:m - 1])
    bad = np.nonzero(~(down | tie))[0]
    assert bad.size == 0, (f"{where}: entries {int(bad[0])}, {int(bad[0]) + 1} out of selection "
                           f"order ({v[bad[0]]!r}, {int(gi[bad[0]])}), ({v[bad[0] + 1]!r}, "
                           f"{int(gi[bad[0] + 1])})")


def _row_offset(pb_cpu, b):
    return int(pb_cpu.output_idx_offset[b]) if pb_cpu.output_idx_offset is not None else 0


def as_rows(t, topk):
    return t.detach().cpu().numpy().reshape(-1, topk)


def check(orc, pb_cpu, gpu_idx, gpu_val, rows=None, exact=False, label=""):
    """Compare GPU outputs (all rows, as [rows, topk] numpy arrays) with the oracle on `rows`
    (all rows when None). Returns the number of rows checked."""
    bound = orc.bind(pb_cpu)
    rows = np.arange(pb_cpu.rows) if rows is None else np.asarray(rows, dtype=np.int64)
    o_idx, o_val, rc, maxabs = bound.topk(rows, with_maxabs=True)
    assert rc == 0
    topk = pb_cpu.topk
    for n, r in enumerate(rows):
        gi, gv = gpu_idx[r], gpu_val[r] if gpu_val is not None else None
        oi, ov = o_idx[n], o_val[n]
        where = f"{label} row {int(r)}"
        m = int((oi >= 0).sum())
        mg = int((gi >= 0).sum())
        assert mg == m, f"{where}: {mg} valid entries, oracle {m}"
        assert (gi[m:] == -1).all(), f"{where}: index padding"
        if gv is not None:
            assert np.isneginf(gv[m:]).all(), f"{where}: value padding"
        if exact:
            assert np.array_equal(gi, oi), f"{where}: indices differ (exact inputs)"
            if gv is not None:
                assert np.array_equal(_bits(gv), _bits(ov)), f"{where}: values differ (exact)"
            continue
        if m == 0:
            continue
        tol = TOL_REL * maxabs[n] + TOL_ABS
        hi, b, _pos = bound.row_info(int(r))
        off = _row_offset(pb_cpu, b)
        scores = bound.scores(int(r))
        _check_entries(where, gi, gv, m, off, hi, scores, tol)
        if gv is not None:
            err = np.abs(gv[:m].astype(np.float64) - ov[:m].astype(np.float64))
            bad = np.nonzero(err > tol)[0]
            assert bad.size == 0, (f"{where}: value err {err.max():.3g} > tol {tol:.3g} at "
                                   f"positions {bad[:5].tolist()}")
        diff = set(gi[:m].tolist()) ^ set(oi[:m].tolist())
        if diff:
            kth = float(ov[m - 1])
            for jj in diff:
                j = jj - off
                assert 0 <= j < hi, f"{where}: index {jj} outside the window"
                s = float(scores[j])
                assert abs(s - kth) <= tol, (f"{where}: key {jj} (score {s:.6g}) differs from the "
                                             f"oracle's set, k-th score {kth:.6g}, tol {tol:.3g}")
    return len(rows)


def sample_rows(pb, n, seed=0, must=()):
    """n seeded-random query rows plus the listed ones (deduplicated, sorted)."""
    rng = np.random.default_rng(seed)
    pick = set(int(x) for x in must if 0 <= x < pb.rows)
    if pb.rows > 0:
        pick.update(rng.choice(pb.rows, size=min(n, pb.rows), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def check_pair(orc, pb_cpu, a_idx, a_val, b_idx, b_val, label=""):
    """Two GPU outputs of the same problem agree under the same tolerance rule (values within
    2e-3 * max|I| + 1e-4 position-wise; index sets equal outside the near-tie band), and each of
    them ties every entry to its own key's exact oracle score and keeps the selection order."""
    bound = orc.bind(pb_cpu)
    rows = np.arange(pb_cpu.rows)
    _oi, o_val, rc, maxabs = bound.topk(rows, with_maxabs=True)
    assert rc == 0
    for r in rows:
        where = f"{label} row {int(r)}"
        ai, bi = a_idx[r], b_idx[r]
        m = int((ai >= 0).sum())
        assert int((bi >= 0).sum()) == m, f"{where}: valid counts differ"
        assert (ai[m:] == -1).all() and (bi[m:] == -1).all(), f"{where}: index padding"
        assert np.isneginf(a_val[r][m:]).all() and np.isneginf(b_val[r][m:]).all(), where
        if m == 0:
            continue
        tol = TOL_REL * maxabs[r] + TOL_ABS
        hi, b, _p = bound.row_info(int(r))
        off = _row_offset(pb_cpu, b)
        scores = bound.scores(int(r))
        _check_entries(where + " (first)", ai, a_val[r], m, off, hi, scores, tol)
        _check_entries(where + " (second)", bi, b_val[r], m, off, hi, scores, tol)
        err = np.abs(a_val[r][:m].astype(np.float64) - b_val[r][:m].astype(np.float64))
        assert (err <= tol).all(), f"{where}: values differ by {err.max():.3g} > {tol:.3g}"
        diff = set(ai[:m].tolist()) ^ set(bi[:m].tolist())
        if diff:
            kth = float(o_val[r][m - 1])
            for jj in diff:
                s = float(scores[jj - off])
                assert abs(s - kth) <= tol, f"{where}: key {jj} is not a near-tie"
