"""ctypes wrapper around the C oracle (``li_oracle.c``).

TEST INFRASTRUCTURE: only the tests, the package's smoke check and the benchmark's CPU-baseline
leg use this module. It marshals arguments and nothing else; every step of the computation is
in the C file. It accepts any problem object that carries the attributes listed in
``_FIELDS`` (q, k, w as bf16 CPU tensors or uint16 numpy arrays, int32 side arrays or None,
layouts as strings) and never imports the CUDA package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SOURCE = HERE / "li_oracle.c"
BUILD_DIR = HERE / "_build"

LAYOUTS = {"BSND": 0, "TND": 1, "PA_BSND": 2}
ORC_OK, ORC_EARG, ORC_EDATA, ORC_ENOMEM = 0, 1, 2, 3


def build(mutant: int = 0, out_dir: Path | None = None) -> Path:
    """Compile the oracle with gcc. ``mutant`` > 0 plants the numbered mistake (for tests)."""
    out_dir = Path(out_dir) if out_dir is not None else BUILD_DIR
    out_dir.mkdir(parents=True, exist_ok=True)
    name = "liorc" + (f"_m{mutant}" if mutant else "") + ".so"
    out = out_dir / name
    if out.exists() and out.stat().st_mtime >= SOURCE.stat().st_mtime:
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared", f"-DORC_MUTANT={mutant}",
           "-o", str(out), str(SOURCE), "-lm"]
    subprocess.run(cmd, check=True)
    return out


class _Problem(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("seqused_q", ctypes.c_void_p), ("seqused_k", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("output_idx_offset", ctypes.c_void_p),
        ("block_table_stride", ctypes.c_int64),
        ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("k_len", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("layout_q", ctypes.c_int32), ("layout_k", ctypes.c_int32), ("mask_mode", ctypes.c_int32),
        ("cmp_residual_k", ctypes.c_void_p), ("cmp_ratio", ctypes.c_int32),
        ("dtype_qk", ctypes.c_int32), ("dtype_w", ctypes.c_int32),
        ("q_descale", ctypes.c_void_p), ("k_descale", ctypes.c_void_p),
    ]


DTYPES = {"bf16": 0, "fp16": 1, "fp32": 2, "fp8_e4m3": 3}


def _dtype_name(x) -> str:
    """bf16 / fp16 / fp32 / fp8_e4m3 of a tensor (uint16 arrays are bf16 bit patterns)."""
    if isinstance(x, np.ndarray):
        return "fp32" if x.dtype == np.float32 else "bf16"
    import torch
    return {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32",
            torch.float8_e4m3fn: "fp8_e4m3"}[x.dtype]


def _bits16(x) -> np.ndarray:
    """bf16/fp16 tensor or uint16 array -> contiguous uint16 numpy array of the bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # local: the oracle does not need torch unless handed tensors
    assert x.dtype in (torch.bfloat16, torch.float16), x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()).view(np.uint16)


def _qk_codes(x) -> np.ndarray:
    """q or k as stored: 16-bit patterns (bf16 / fp16) or 8-bit codes (fp8 e4m3)."""
    if not isinstance(x, np.ndarray) and _dtype_name(x) == "fp8_e4m3":
        import torch
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.uint8).numpy())
    return _bits16(x)


def _f32(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _weights(x) -> np.ndarray:
    """w as 16-bit patterns, or fp32 values."""
    if _dtype_name(x) == "fp32":
        if not isinstance(x, np.ndarray):
            x = x.detach().cpu().contiguous().numpy()
        return np.ascontiguousarray(x, dtype=np.float32)
    return _bits16(x)


def _i32(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


class _KL(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_rope", ctypes.c_void_p),
        ("k_rope", ctypes.c_void_p), ("qi", ctypes.c_void_p), ("ki", ctypes.c_void_p),
        ("w", ctypes.c_void_p), ("sparse_indices", ctypes.c_void_p), ("key_base", ctypes.c_void_p),
        ("softmax_max", ctypes.c_void_p), ("softmax_sum", ctypes.c_void_p),
        ("scale", ctypes.c_double), ("rows", ctypes.c_int64), ("key_rows", ctypes.c_int64),
        ("G", ctypes.c_int32), ("Dm", ctypes.c_int32), ("Dr", ctypes.c_int32), ("H", ctypes.c_int32),
        ("Di", ctypes.c_int32), ("topk", ctypes.c_int32),
    ]


def _f64(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


class _Attn(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_rope", ctypes.c_void_p),
        ("k_rope", ctypes.c_void_p), ("sparse_indices", ctypes.c_void_p),
        ("key_base", ctypes.c_void_p), ("scale", ctypes.c_double), ("rows", ctypes.c_int64),
        ("key_rows", ctypes.c_int64), ("G", ctypes.c_int32), ("Dm", ctypes.c_int32),
        ("Dr", ctypes.c_int32), ("topk", ctypes.c_int32),
    ]


class Oracle:
    """One loaded build of the oracle (the normal one, or a planted mutant)."""

    def __init__(self, lib_path: Path | str | None = None):
        self.path = Path(lib_path) if lib_path is not None else build()
        lib = ctypes.CDLL(str(self.path))
        P = ctypes.POINTER(_Problem)
        lib.orc_rows.argtypes = [P]
        lib.orc_rows.restype = ctypes.c_int64
        lib.orc_scores.argtypes = [P, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        lib.orc_scores.restype = ctypes.c_int
        lib.orc_row_info.argtypes = [P, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]
        lib.orc_row_info.restype = ctypes.c_int
        lib.orc_topk.argtypes = [P, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p]
        lib.orc_score_at.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.orc_score_at.restype = ctypes.c_int
        lib.orc_topk.restype = ctypes.c_int
        lib.orc_merge_topk.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p]
        lib.orc_merge_topk.restype = ctypes.c_int
        lib.orc_kl_grad.argtypes = [ctypes.POINTER(_KL)] + [ctypes.c_void_p] * 4
        lib.orc_kl_grad.restype = ctypes.c_int
        lib.orc_sparse_attention.argtypes = [ctypes.POINTER(_Attn)] + [ctypes.c_void_p] * 3
        lib.orc_sparse_attention.restype = ctypes.c_int
        self.lib = lib

    # -- marshalling -----------------------------------------------------------------------
    def _marshal(self, pb):
        keep = {}

        def ptr(name, arr):
            if arr is None:
                return None
            keep[name] = arr
            return arr.ctypes.data

        s = _Problem()
        s.q = ptr("q", _qk_codes(pb.q))
        s.k = ptr("k", _qk_codes(pb.k))
        s.q_descale = ptr("q_descale", _f32(getattr(pb, "q_descale", None)))
        s.k_descale = ptr("k_descale", _f32(getattr(pb, "k_descale", None)))
        s.w = ptr("w", _weights(pb.w))
        s.dtype_qk = DTYPES[_dtype_name(pb.q)]
        s.dtype_w = DTYPES[_dtype_name(pb.w)]
        for f in ("cu_seqlens_q", "cu_seqlens_k", "seqused_q", "seqused_k", "block_table",
                  "output_idx_offset", "cmp_residual_k"):
            setattr(s, f, ptr(f, _i32(getattr(pb, f, None))))
        bt = keep.get("block_table")
        s.block_table_stride = int(bt.shape[-1]) if bt is not None and bt.ndim == 2 else 0
        s.batch = int(pb.batch)
        s.q_len = int(pb.q_len)
        s.k_len = int(getattr(pb, "k_len", 0) or 0)
        s.num_blocks = int(getattr(pb, "num_blocks", 0) or 0)
        s.block_size = int(getattr(pb, "block_size", 0) or 0)
        s.n_heads = int(pb.n_heads)
        s.head_dim = int(pb.head_dim)
        s.topk = int(pb.topk)
        s.layout_q = LAYOUTS[pb.layout_q]
        s.layout_k = LAYOUTS[pb.layout_k]
        s.mask_mode = int(pb.mask_mode)
        s.cmp_ratio = int(getattr(pb, "cmp_ratio", 1) or 1)
        return s, keep

    # -- entry points ----------------------------------------------------------------------
    def bind(self, pb) -> "Bound":
        """Marshal a problem once; the returned object answers repeated queries on it."""
        return Bound(self, pb)

    def rows(self, pb) -> int:
        return self.bind(pb).rows()

    def topk(self, pb, rows=None, check: bool = True, with_maxabs: bool = False):
        """Top-k of the given query rows (all when None). Returns (idx, val, status), plus the
        per-row max |I| over the window when with_maxabs."""
        return self.bind(pb).topk(rows, check, with_maxabs)

    def score_at(self, pb, row: int, j: int) -> float:
        return self.bind(pb).score_at(row, j)

    def scores(self, pb, row: int) -> np.ndarray:
        return self.bind(pb).scores(row)

    def row_info(self, pb, row: int):
        return self.bind(pb).row_info(row)

    def kl_grad(self, kp):
        """Indexer backward with the KL loss (orc_kl_grad) of a problem carrying q, k, q_rope,
        k_rope (main attention), qi, ki, w (indexer), sparse_indices, key_base, softmax_max,
        softmax_sum and scale. Arrays may be tensors of any float type (decoded exactly) or
        numpy arrays. Returns (loss, d_qi, d_ki, d_w) in float64 with the shapes of qi, ki, w."""
        keep = {}

        def ptr(name, arr):
            if arr is None:
                return None
            keep[name] = arr
            return arr.ctypes.data

        a = _KL()
        q, k = _f64(kp.q), _f64(kp.k)
        qi, ki, w = _f64(kp.qi), _f64(kp.ki), _f64(kp.w)
        qr, kr = _f64(getattr(kp, "q_rope", None)), _f64(getattr(kp, "k_rope", None))
        rows, G = w.shape[0] if w.ndim == 2 else w.shape[0] * w.shape[1], q.shape[-2]
        a.q, a.k, a.qi, a.ki, a.w = (ptr(n, v) for n, v in
                                     (("q", q), ("k", k), ("qi", qi), ("ki", ki), ("w", w)))
        a.q_rope, a.k_rope = ptr("qr", qr), ptr("kr", kr)
        si = _i32(kp.sparse_indices)
        kb = np.ascontiguousarray(np.asarray(kp.key_base, dtype=np.int64))
        a.sparse_indices, a.key_base = ptr("si", si), ptr("kb", kb)
        a.softmax_max = ptr("smax", _f64(kp.softmax_max))
        a.softmax_sum = ptr("ssum", _f64(kp.softmax_sum))
        a.scale = float(kp.scale)
        a.rows, a.key_rows = rows, ki.size // ki.shape[-1]
        a.G, a.Dm, a.Dr = G, q.shape[-1], 0 if qr is None else qr.shape[-1]
        a.H, a.Di, a.topk = qi.shape[-2], qi.shape[-1], si.shape[-1]
        loss = ctypes.c_double(0.0)
        d_qi, d_ki, d_w = np.empty_like(qi), np.empty_like(ki), np.empty_like(w)
        rc = self.lib.orc_kl_grad(ctypes.byref(a), ctypes.addressof(loss), d_qi.ctypes.data,
                                  d_ki.ctypes.data, d_w.ctypes.data)
        if rc:
            raise RuntimeError(f"oracle orc_kl_grad returned {rc}")
        return loss.value, d_qi, d_ki, d_w

    def sparse_attention(self, kp):
        """Attention of each row's query heads over its selected keys, values = keys
        (orc_sparse_attention), for a problem carrying q, k, q_rope, k_rope, sparse_indices,
        key_base and scale (e.g. synthetic.KLProblem). Returns (out [rows, G, Dm],
        softmax_max [rows, G], softmax_sum [rows, G]) in float64."""
        q, k = _f64(kp.q), _f64(kp.k)
        qr, kr = _f64(getattr(kp, "q_rope", None)), _f64(getattr(kp, "k_rope", None))
        si = _i32(kp.sparse_indices)
        kb = np.ascontiguousarray(np.asarray(kp.key_base, dtype=np.int64))
        G, Dm = q.shape[-2], q.shape[-1]
        rows = q.size // (G * Dm)
        a = _Attn()
        a.q, a.k = q.ctypes.data, k.ctypes.data
        a.q_rope = None if qr is None else qr.ctypes.data
        a.k_rope = None if kr is None else kr.ctypes.data
        a.sparse_indices, a.key_base = si.ctypes.data, kb.ctypes.data
        a.scale = float(kp.scale)
        a.rows, a.key_rows = rows, k.size // Dm
        a.G, a.Dm, a.Dr, a.topk = G, Dm, 0 if qr is None else qr.shape[-1], si.shape[-1]
        out = np.empty((rows, G, Dm))
        smax, ssum = np.empty((rows, G)), np.empty((rows, G))
        rc = self.lib.orc_sparse_attention(ctypes.byref(a), out.ctypes.data, smax.ctypes.data,
                                           ssum.ctypes.data)
        if rc:
            raise RuntimeError(f"oracle orc_sparse_attention returned {rc}")
        return out, smax, ssum

    def merge_topk(self, idx_lists, val_lists, topk: int):
        """Top-k of the union of per-row lists: idx_lists / val_lists are sequences of
        (rows, topk_in) int32 / float32 arrays (one per key range); returns (idx, val) of shape
        (rows, topk)."""
        idx = np.ascontiguousarray(np.stack([np.asarray(x, dtype=np.int32) for x in idx_lists]))
        val = np.ascontiguousarray(np.stack([np.asarray(x, dtype=np.float32) for x in val_lists]))
        n_lists, rows, topk_in = idx.shape
        out_i = np.empty((rows, topk), dtype=np.int32)
        out_v = np.empty((rows, topk), dtype=np.float32)
        rc = self.lib.orc_merge_topk(rows, n_lists, topk_in, idx.ctypes.data, val.ctypes.data,
                                     topk, out_i.ctypes.data, out_v.ctypes.data)
        if rc:
            raise RuntimeError(f"oracle orc_merge_topk returned {rc}")
        return out_i, out_v


class Bound:
    """A problem marshalled for one oracle build."""

    def __init__(self, orc: Oracle, pb):
        self.lib = orc.lib
        self.s, self._keep = orc._marshal(pb)
        self.topk_k = int(self.s.topk)

    def rows(self) -> int:
        return int(self.lib.orc_rows(ctypes.byref(self.s)))

    def topk(self, rows=None, check: bool = True, with_maxabs: bool = False):
        if rows is None:
            n = self.rows()
            rows_arr = None
        else:
            rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            n = rows_arr.size
        idx = np.empty((n, self.topk_k), dtype=np.int32)
        val = np.empty((n, self.topk_k), dtype=np.float32)
        mx = np.zeros(max(n, 1), dtype=np.float64)
        rc = self.lib.orc_topk(ctypes.byref(self.s),
                               None if rows_arr is None else rows_arr.ctypes.data, n,
                               idx.ctypes.data, val.ctypes.data, mx.ctypes.data)
        if check and rc not in (ORC_OK,):
            raise RuntimeError(f"oracle orc_topk returned {rc}")
        if with_maxabs:
            return idx, val, rc, mx[:n]
        return idx, val, rc

    def score_at(self, row: int, j: int) -> float:
        """Exact (fp64) score of one (row, key) pair inside the row's window."""
        out = ctypes.c_double(0.0)
        rc = self.lib.orc_score_at(ctypes.byref(self.s), int(row), int(j), ctypes.byref(out))
        if rc:
            raise RuntimeError(f"oracle orc_score_at({row}, {j}) returned {rc}")
        return out.value

    def row_info(self, row: int):
        """(window length, batch, position in batch) of a query row."""
        hi = ctypes.c_int64(0)
        b = ctypes.c_int32(0)
        i = ctypes.c_int32(0)
        rc = self.lib.orc_row_info(ctypes.byref(self.s), int(row), ctypes.byref(hi),
                                   ctypes.byref(b), ctypes.byref(i))
        if rc:
            raise RuntimeError(f"oracle orc_row_info returned {rc}")
        return hi.value, b.value, i.value

    def scores(self, row: int) -> np.ndarray:
        """Exact (fp64) scores I[row, j] over the row's key window."""
        hi0, _b, _i = self.row_info(row)
        out = np.empty(max(hi0, 1), dtype=np.float64)
        hi = ctypes.c_int64(0)
        rc = self.lib.orc_scores(ctypes.byref(self.s), int(row), out.ctypes.data,
                                 ctypes.byref(hi))
        if rc:
            raise RuntimeError(f"oracle orc_scores returned {rc}")
        return out[: hi.value]


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The normal (unmutated) oracle build, compiled on first use."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def host_cores() -> int:
    return os.cpu_count() or 1
