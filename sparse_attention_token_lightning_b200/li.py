"""Thin ctypes binding over ``libli.so`` (C ABI in include/li.h).

Argument marshalling only: every step of the indexer runs in the library's CUDA kernels. The
functions keep the C names (``li_metadata``, ``li_indexer``, ``li_merge_topk``, ``li_kl_grad``,
...). ``indexer()``, ``merge_topk()`` and ``kl_grad()`` are conveniences that allocate outputs and
workspaces with torch and call the library on the current stream; ``HostPipeline`` runs the
indexer over host-resident problems with the copies overlapping the kernels. There is no
fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libli.so"
LAYOUTS = {"BSND": 0, "TND": 1, "PA_BSND": 2}
STATUS = {0: "LI_OK", 1: "LI_ERR_INVALID_ARG", 2: "LI_ERR_UNSUPPORTED", 3: "LI_ERR_WORKSPACE",
          4: "LI_ERR_CUDA", 5: "LI_ERR_DEVICE_TIMEOUT", 6: "LI_ERR_DEVICE_DATA"}
LI_OK = 0
DEVERR_TIMEOUT, DEVERR_LENGTHS, DEVERR_TABLE, DEVERR_OFFSET, DEVERR_METADATA = 1, 2, 4, 8, 16
DEVERR_INTERNAL, DEVERR_MERGE_ORDER, DEVERR_DESCALE = 32, 64, 128        # LI_DEVERR_* of li.h


class LiError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class LiArgs(ctypes.Structure):
    """Mirror of ``li_args`` (include/li.h)."""

    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("seqused_q", ctypes.c_void_p), ("seqused_k", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int64),
        ("output_idx_offset", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("k_len", ctypes.c_int32),
        ("max_seqlen_q", ctypes.c_int32), ("max_seqlen_k", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("num_heads_q", ctypes.c_int32), ("num_heads_k", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("layout_q", ctypes.c_int32), ("layout_k", ctypes.c_int32), ("mask_mode", ctypes.c_int32),
        ("dtype_qk", ctypes.c_int32), ("dtype_w", ctypes.c_int32),
        ("return_value", ctypes.c_int32),
        ("cmp_residual_k", ctypes.c_void_p), ("cmp_ratio", ctypes.c_int32),
        ("q_descale", ctypes.c_void_p), ("k_descale", ctypes.c_void_p),
    ]


DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2,
          torch.float8_e4m3fn: 3}                                   # li_dtype


class LiPlanInfo(ctypes.Structure):
    """Mirror of ``li_plan_info`` (include/li.h)."""

    _fields_ = [("tq", ctypes.c_int32), ("kc", ctypes.c_int32), ("max_items", ctypes.c_int32),
                ("dense", ctypes.c_int32), ("kernels", ctypes.c_int32),
                ("score_tc", ctypes.c_int32), ("select_pieces", ctypes.c_int32)]


_lib = None

EXPORTS = ("li_metadata_workspace_size", "li_metadata", "li_indexer_workspace_size",
           "li_indexer", "li_check_status", "li_set_stage_events", "li_last_error_string",
           "li_abi_version", "li_indexer_noalloc", "li_plan", "li_merge_topk",
           "li_kl_grad_workspace_size", "li_kl_grad", "li_sparse_attention_workspace_size",
           "li_sparse_attention")

MERGE_MAX_LISTS = 16          # LI_MERGE_MAX_LISTS


class LiKlArgs(ctypes.Structure):
    """Mirror of li_kl_args (include/li.h)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_rope", ctypes.c_void_p),
        ("k_rope", ctypes.c_void_p), ("qi", ctypes.c_void_p), ("ki", ctypes.c_void_p),
        ("w", ctypes.c_void_p), ("sparse_indices", ctypes.c_void_p),
        ("softmax_max", ctypes.c_void_p), ("softmax_sum", ctypes.c_void_p),
        ("scale", ctypes.c_float), ("batch", ctypes.c_int32), ("s1", ctypes.c_int32),
        ("s2", ctypes.c_int32), ("G", ctypes.c_int32), ("Dm", ctypes.c_int32),
        ("Dr", ctypes.c_int32), ("H", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class LiAttnArgs(ctypes.Structure):
    """Mirror of li_attn_args (include/li.h)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_rope", ctypes.c_void_p),
        ("k_rope", ctypes.c_void_p), ("sparse_indices", ctypes.c_void_p),
        ("scale", ctypes.c_float), ("batch", ctypes.c_int32), ("s1", ctypes.c_int32),
        ("s2", ctypes.c_int32), ("G", ctypes.c_int32), ("Dm", ctypes.c_int32),
        ("Dr", ctypes.c_int32), ("topk", ctypes.c_int32), ("layout_k", ctypes.c_int32),
        ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class LiMergeArgs(ctypes.Structure):
    """Mirror of li_merge_args (include/li.h)."""
    _fields_ = [
        ("idx_in", ctypes.c_void_p * MERGE_MAX_LISTS), ("val_in", ctypes.c_void_p * MERGE_MAX_LISTS),
        ("idx_out", ctypes.c_void_p), ("val_out", ctypes.c_void_p),
        ("device_status", ctypes.c_void_p), ("rows", ctypes.c_int64), ("n_lists", ctypes.c_int32),
        ("topk_in", ctypes.c_int32), ("topk_out", ctypes.c_int32), ("reserved", ctypes.c_int32),
    ]


def lib_path() -> Path:
    return _LIB_PATH


def lib():
    """Load libli.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m sparse_attention_token_lightning_b200.build`")
    _lib = load(_LIB_PATH)
    return _lib


def load(path) -> ctypes.CDLL:
    """A separately loaded build of the library at `path` (same C ABI), with the argument types
    set; used for the test build whose device waits give up after 1 ms."""
    L = ctypes.CDLL(str(path))
    P = ctypes.POINTER(LiArgs)
    sz = ctypes.POINTER(ctypes.c_size_t)
    vp = ctypes.c_void_p
    L.li_metadata_workspace_size.argtypes = [P, sz]
    L.li_metadata.argtypes = [P, vp, ctypes.c_size_t, vp]
    L.li_indexer_workspace_size.argtypes = [P, sz]
    L.li_plan.argtypes = [P, ctypes.POINTER(LiPlanInfo)]
    L.li_plan.restype = ctypes.c_int
    L.li_indexer.argtypes = [P, vp, vp, ctypes.c_size_t, vp, vp, vp]
    L.li_check_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    for f in ("li_metadata_workspace_size", "li_metadata", "li_indexer_workspace_size",
              "li_indexer", "li_check_status"):
        getattr(L, f).restype = ctypes.c_int
    L.li_indexer_noalloc.argtypes = [P, vp, vp, vp, vp]
    L.li_indexer_noalloc.restype = ctypes.c_int
    L.li_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
    L.li_set_stage_events.restype = ctypes.c_int
    L.li_last_error_string.argtypes = []
    L.li_last_error_string.restype = ctypes.c_char_p
    L.li_kl_grad_workspace_size.argtypes = [ctypes.POINTER(LiKlArgs), sz]
    L.li_kl_grad_workspace_size.restype = ctypes.c_int
    L.li_kl_grad.argtypes = [ctypes.POINTER(LiKlArgs), vp, ctypes.c_size_t, vp, vp, vp, vp, vp]
    L.li_kl_grad.restype = ctypes.c_int
    L.li_sparse_attention_workspace_size.argtypes = [ctypes.POINTER(LiAttnArgs), sz]
    L.li_sparse_attention_workspace_size.restype = ctypes.c_int
    L.li_sparse_attention.argtypes = [ctypes.POINTER(LiAttnArgs), vp, ctypes.c_size_t, vp, vp, vp, vp]
    L.li_sparse_attention.restype = ctypes.c_int
    L.li_merge_topk.argtypes = [ctypes.POINTER(LiMergeArgs), vp]
    L.li_merge_topk.restype = ctypes.c_int
    L.li_abi_version.argtypes = []
    L.li_abi_version.restype = ctypes.c_int32
    return L


def li_last_error_string() -> str:
    return lib().li_last_error_string().decode()


def li_abi_version() -> int:
    return int(lib().li_abi_version())


def _check(st: int):
    if st != LI_OK:
        raise LiError(st, li_last_error_string())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def make_args(pb, return_value: int = 1) -> LiArgs:
    """li_args for a problem whose tensors are already on the device (see synthetic.Problem)."""
    a = LiArgs()
    for name in ("q", "k", "w"):
        t = getattr(pb, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    a.q, a.k, a.w = _ptr(pb.q), _ptr(pb.k), _ptr(pb.w)
    a.cu_seqlens_q = _ptr(pb.cu_seqlens_q)
    a.cu_seqlens_k = _ptr(pb.cu_seqlens_k)
    a.seqused_q = _ptr(pb.seqused_q)
    a.seqused_k = _ptr(pb.seqused_k)
    a.block_table = _ptr(pb.block_table)
    a.block_table_stride = int(pb.block_table.shape[-1]) if pb.block_table is not None else 0
    a.output_idx_offset = _ptr(pb.output_idx_offset)
    a.batch = pb.batch
    a.q_len = pb.q_len
    a.k_len = pb.k_len
    a.max_seqlen_q = pb.max_seqlen_q
    a.max_seqlen_k = pb.max_seqlen_k
    a.num_blocks = pb.num_blocks
    a.block_size = pb.block_size
    a.num_heads_q = pb.n_heads
    a.num_heads_k = 1
    a.head_dim = pb.head_dim
    a.topk = pb.topk
    a.layout_q = LAYOUTS[pb.layout_q]
    a.layout_k = LAYOUTS[pb.layout_k]
    a.mask_mode = pb.mask_mode
    a.dtype_qk = DTYPES[pb.q.dtype]
    a.dtype_w = DTYPES[pb.w.dtype]
    a.return_value = int(return_value)
    a.cmp_residual_k = _ptr(getattr(pb, "cmp_residual_k", None))
    a.cmp_ratio = int(getattr(pb, "cmp_ratio", 1) or 1)
    a.q_descale = _ptr(getattr(pb, "q_descale", None))
    a.k_descale = _ptr(getattr(pb, "k_descale", None))
    return a


def li_metadata_workspace_size(args: LiArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().li_metadata_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def li_indexer_workspace_size(args: LiArgs) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().li_indexer_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return int(n.value)


def li_plan(args: LiArgs) -> dict:
    info = LiPlanInfo()
    _check(lib().li_plan(ctypes.byref(args), ctypes.byref(info)))
    return {f: int(getattr(info, f)) for f, _ in LiPlanInfo._fields_}


def li_metadata(args: LiArgs, metadata: torch.Tensor, stream=None):
    _check(lib().li_metadata(ctypes.byref(args), metadata.data_ptr(),
                             metadata.numel() * metadata.element_size(), _stream_handle(stream)))


def li_indexer(args: LiArgs, metadata, workspace: torch.Tensor, sparse_indices: torch.Tensor,
               sparse_values, stream=None):
    _check(lib().li_indexer(ctypes.byref(args), _ptr(metadata), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(),
                            sparse_indices.data_ptr(), _ptr(sparse_values),
                            _stream_handle(stream)))


def li_indexer_noalloc(args: LiArgs, sparse_indices: torch.Tensor, sparse_values,
                       device_status=None, stream=None):
    """li_indexer without a caller workspace (the library's static scratch is used); for
    callers that may not allocate device memory. device_status: a 4-byte device tensor that
    receives the call's status word, or None."""
    _check(lib().li_indexer_noalloc(ctypes.byref(args), sparse_indices.data_ptr(),
                                    _ptr(sparse_values), _ptr(device_status),
                                    _stream_handle(stream)))


def li_check_status(workspace: torch.Tensor, stream=None):
    """Synchronize and read the device status word: returns (status, LI_DEVERR_* bits)."""
    bits = ctypes.c_uint32(0)
    st = lib().li_check_status(workspace.data_ptr(), _stream_handle(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def li_set_stage_events(events):
    """Time li_indexer's kernels: six recorded torch.cuda.Event objects, or None to stop."""
    if not events:
        _check(lib().li_set_stage_events(None, 0))
        return
    assert len(events) == 6
    arr = (ctypes.c_void_p * 6)(*[int(e.cuda_event) for e in events])
    _check(lib().li_set_stage_events(arr, 6))


def li_merge_topk(args: LiMergeArgs, stream=None):
    _check(lib().li_merge_topk(ctypes.byref(args), _stream_handle(stream)))


def merge_topk(idx_lists, val_lists, topk: int, return_value: bool = True, device_status=None,
               stream=None, check: bool = True):
    """Top-k of the union of per-row lists from key-range shards (li_merge_topk).

    idx_lists / val_lists: sequences of device tensors whose last dimension is topk_in and whose
    other dimensions flatten to the same row count (li_indexer outputs, indices already global),
    or one stacked tensor of shape (n_lists, ...). Returns (indices, values) shaped like one
    input list with topk as the last dimension; values is None when return_value is False."""
    if isinstance(idx_lists, torch.Tensor):
        idx_lists, val_lists = list(idx_lists.unbind(0)), list(val_lists.unbind(0))
    n = len(idx_lists)
    if n != len(val_lists) or not 1 <= n <= MERGE_MAX_LISTS:
        raise ValueError(f"{n} index lists and {len(val_lists)} value lists")
    ref = idx_lists[0]
    topk_in = int(ref.shape[-1])
    rows = ref.numel() // max(topk_in, 1)
    for i, v in zip(idx_lists, val_lists):
        if (i.dtype != torch.int32 or v.dtype != torch.float32 or i.shape != ref.shape or
                v.shape != ref.shape or not i.is_contiguous() or not v.is_contiguous()):
            raise ValueError("lists must be contiguous int32 / float32 tensors of one shape")
    out_shape_ = tuple(ref.shape[:-1]) + (int(topk),)
    idx = torch.empty(out_shape_, dtype=torch.int32, device=ref.device)
    val = torch.empty(out_shape_, dtype=torch.float32, device=ref.device) if return_value else None
    own_status = device_status is None and check
    if own_status:
        device_status = torch.zeros(1, dtype=torch.int32, device=ref.device)
    a = LiMergeArgs()
    for l in range(n):
        a.idx_in[l] = idx_lists[l].data_ptr()
        a.val_in[l] = val_lists[l].data_ptr()
    a.idx_out, a.val_out = idx.data_ptr(), _ptr(val)
    a.device_status = _ptr(device_status)
    a.rows, a.n_lists, a.topk_in, a.topk_out = rows, n, topk_in, int(topk)
    li_merge_topk(a, stream)
    if own_status:
        st, bits = li_check_status(device_status, stream)
        if st != LI_OK:
            raise LiError(st, f"{li_last_error_string()} (device bits 0x{bits:x})")
    return idx, val


def make_kl_args(kp) -> LiKlArgs:
    """li_kl_args of a device-resident backward problem (synthetic.KLProblem)."""
    a = LiKlArgs()
    B, S1, G, Dm = kp.q.shape
    a.q, a.k, a.qi, a.ki, a.w = (t.data_ptr() for t in (kp.q, kp.k, kp.qi, kp.ki, kp.w))
    a.q_rope, a.k_rope = _ptr(kp.q_rope), _ptr(kp.k_rope)
    a.sparse_indices = kp.sparse_indices.data_ptr()
    a.softmax_max, a.softmax_sum = kp.softmax_max.data_ptr(), kp.softmax_sum.data_ptr()
    a.scale = float(kp.scale)
    a.batch, a.s1, a.s2 = B, S1, kp.k.shape[1]
    a.G, a.Dm, a.Dr = G, Dm, 0 if kp.q_rope is None else kp.q_rope.shape[-1]
    a.H, a.topk = kp.qi.shape[2], kp.sparse_indices.shape[-1]
    return a


def kl_grad(kp, stream=None, check: bool = True):
    """The indexer backward with the KL loss on a device-resident problem: returns (loss,
    d_query_index, d_key_index, d_weights) as fp32 device tensors (loss of shape (1,))."""
    a = make_kl_args(kp)
    n = ctypes.c_size_t(0)
    _check(lib().li_kl_grad_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    dev = kp.q.device
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    d_qi = torch.empty(kp.qi.shape, dtype=torch.float32, device=dev)
    d_ki = torch.empty(kp.ki.shape, dtype=torch.float32, device=dev)
    d_w = torch.empty(kp.w.shape, dtype=torch.float32, device=dev)
    _check(lib().li_kl_grad(ctypes.byref(a), ws.data_ptr(), n.value, loss.data_ptr(),
                            d_qi.data_ptr(), d_ki.data_ptr(), d_w.data_ptr(), _stream_handle(stream)))
    if check:
        st, bits = li_check_status(ws, stream)
        if st != LI_OK:
            raise LiError(st, f"{li_last_error_string()} (device bits 0x{bits:x})")
    return loss, d_qi, d_ki, d_w


def make_attn_args(ap) -> LiAttnArgs:
    """li_attn_args of a device-resident attention problem (q, k, q_rope, k_rope,
    sparse_indices, scale: synthetic.AttnProblem or synthetic.KLProblem)."""
    a = LiAttnArgs()
    B, S1, G, Dm = ap.q.shape
    a.q, a.k = ap.q.data_ptr(), ap.k.data_ptr()
    a.q_rope, a.k_rope = _ptr(ap.q_rope), _ptr(ap.k_rope)
    a.sparse_indices = ap.sparse_indices.data_ptr()
    a.scale = float(ap.scale)
    a.batch, a.s1, a.s2 = B, S1, ap.k.shape[1]
    a.G, a.Dm, a.Dr = G, Dm, 0 if ap.q_rope is None else ap.q_rope.shape[-1]
    a.topk = ap.sparse_indices.shape[-1]
    bt = getattr(ap, "block_table", None)
    if bt is not None:
        # paged keys: k is the cache (num_blocks, block_size, 1, Dm), S2 the logical length
        a.layout_k = LAYOUTS["PA_BSND"]
        a.block_table = bt.data_ptr()
        a.block_table_stride = bt.shape[1]
        a.num_blocks, a.block_size = ap.k.shape[0], ap.k.shape[1]
        a.s2 = int(ap.s2)
    else:
        a.layout_k = LAYOUTS["BSND"]
    return a


def li_sparse_attention(args: LiAttnArgs, workspace: torch.Tensor, out: torch.Tensor,
                        softmax_max: torch.Tensor, softmax_sum: torch.Tensor, stream=None):
    _check(lib().li_sparse_attention(ctypes.byref(args), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), out.data_ptr(),
                                     softmax_max.data_ptr(), softmax_sum.data_ptr(),
                                     _stream_handle(stream)))


def sparse_attention(ap, stream=None, check: bool = True):
    """Attention of every row over its selected keys (values = keys) on a device-resident
    problem: returns (out (B,S1,G,Dm), softmax_max (B,1,S1,G), softmax_sum (B,1,S1,G)), fp32."""
    a = make_attn_args(ap)
    n = ctypes.c_size_t(0)
    _check(lib().li_sparse_attention_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    dev = ap.q.device
    B, S1, G, Dm = ap.q.shape
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    out = torch.empty((B, S1, G, Dm), dtype=torch.float32, device=dev)
    smax = torch.empty((B, 1, S1, G), dtype=torch.float32, device=dev)
    ssum = torch.empty((B, 1, S1, G), dtype=torch.float32, device=dev)
    li_sparse_attention(a, ws, out, smax, ssum, stream)
    if check:
        st, bits = li_check_status(ws, stream)
        if st != LI_OK:
            raise LiError(st, f"{li_last_error_string()} (device bits 0x{bits:x})")
    return out, smax, ssum


class HostPipeline:
    """li_indexer over a series of host-resident problems of one shape: inputs copied in from
    pinned host memory, outputs read back to pinned host memory, with the copies overlapping the
    kernels. Three streams (copy in, kernels, copy out) and `depth` sets of device buffers let
    step i's host-to-device copy, step i-1's kernels and step i-2's device-to-host copy run at
    the same time; events keep a buffer set from being refilled before its kernels have read it
    or overwritten before its outputs have been copied out.

    template: a problem giving the shapes, types and scalar arguments (its tensors are copied
    once to size the device buffers). run(inputs, outputs): inputs[i] maps the problem's tensor
    fields (q, k, w and the side arrays) to pinned host tensors of the template's shapes;
    outputs[i] is a pair of pinned host tensors (indices, values) of li.out_shape. Returns when
    the work is queued; synchronize() waits for it."""

    def __init__(self, template, device, depth: int = 2):
        from .synthetic import Problem
        self.fields = [f for f in Problem.TENSORS if getattr(template, f) is not None]
        self.sets = []
        for _ in range(depth):
            pb = template.to(device)
            args = make_args(pb)
            self.sets.append(dict(
                pb=pb, args=args, ws=empty_workspace(args, device),
                idx=torch.empty(out_shape(pb), dtype=torch.int32, device=device),
                val=torch.empty(out_shape(pb), dtype=torch.float32, device=device),
                loaded=torch.cuda.Event(), ran=torch.cuda.Event(), saved=torch.cuda.Event()))
        self.s_in = torch.cuda.Stream(device)
        self.s_run = torch.cuda.Stream(device)
        self.s_out = torch.cuda.Stream(device)

    def run(self, inputs, outputs):
        for i, (h, (hi, hv)) in enumerate(zip(inputs, outputs)):
            S = self.sets[i % len(self.sets)]
            self.s_in.wait_event(S["ran"])          # the set's previous kernels are done with it
            with torch.cuda.stream(self.s_in):
                for f in self.fields:
                    getattr(S["pb"], f).copy_(h[f], non_blocking=True)
                S["loaded"].record(self.s_in)
            self.s_run.wait_event(S["loaded"])
            self.s_run.wait_event(S["saved"])       # its previous outputs are back on the host
            li_indexer(S["args"], None, S["ws"], S["idx"], S["val"], self.s_run)
            S["ran"].record(self.s_run)
            self.s_out.wait_event(S["ran"])
            with torch.cuda.stream(self.s_out):
                hi.copy_(S["idx"], non_blocking=True)
                hv.copy_(S["val"], non_blocking=True)
                S["saved"].record(self.s_out)

    def check(self):
        """Device status of every buffer set (raises LiError on a data error)."""
        for S in self.sets:
            st, bits = li_check_status(S["ws"], self.s_run)
            if st != LI_OK:
                raise LiError(st, f"{li_last_error_string()} (device bits 0x{bits:x})")

    def synchronize(self):
        self.s_out.synchronize()


def out_shape(pb):
    return (pb.batch, pb.q_len, 1, pb.topk) if pb.layout_q == "BSND" else (pb.q_len, 1, pb.topk)


def empty_workspace(args: LiArgs, device) -> torch.Tensor:
    n = li_indexer_workspace_size(args)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def indexer(pb, return_value: bool = True, metadata: bool | torch.Tensor = False,
            workspace: torch.Tensor | None = None, stream=None, check: bool = True):
    """Run the indexer on a device-resident problem. Returns (sparse_indices, sparse_values).

    metadata: False = built inline by li_indexer; True = built by a separate li_metadata call;
    a tensor = a schedule the caller built before."""
    args = make_args(pb, int(return_value))
    dev = pb.q.device
    idx = torch.empty(out_shape(pb), dtype=torch.int32, device=dev)
    val = torch.empty(out_shape(pb), dtype=torch.float32, device=dev) if return_value else None
    ws = workspace if workspace is not None else empty_workspace(args, dev)
    meta = None
    if isinstance(metadata, torch.Tensor):
        meta = metadata
    elif metadata:
        meta = torch.empty(li_metadata_workspace_size(args), dtype=torch.uint8, device=dev)
        li_metadata(args, meta, stream)
    li_indexer(args, meta, ws, idx, val, stream)
    if check:
        st, bits = li_check_status(ws, stream)
        if st != LI_OK:
            raise LiError(st, f"{li_last_error_string()} (device bits 0x{bits:x})")
    return idx, val
