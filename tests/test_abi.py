"""The C ABI without a GPU: the library loads, exports every function include/li.h declares, the
ctypes mirror of li_args matches the C layout, and host-side validation rejects bad arguments
before any launch."""
import ctypes
import re
import subprocess
from pathlib import Path

import pytest

from sparse_attention_token_lightning_b200 import li
from sparse_attention_token_lightning_b200 import build as libbuild

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "li.h"


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return li.lib()


def declared_functions():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"^[a-z0-9_ ]+[ *](li_[a-z_]+)\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in li.EXPORTS:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", str(li.lib_path())], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (li_[a-z_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(L, n)


@pytest.mark.parametrize("which", ["debug", "waittest"])
def test_test_builds_export_every_declared_symbol(which):
    """The bounds-checked build and the wait-limit test build keep the same C ABI."""
    path = libbuild.build_debug() if which == "debug" else libbuild.build_wait_test()
    out = subprocess.run(["nm", "-D", "--defined-only", str(path)], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (li_[a-z_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert li.load(path).li_abi_version() == 6


def test_abi_version(L):
    assert li.li_abi_version() == 6


@pytest.mark.parametrize("cls,cname", [(li.LiArgs, "li_args"), (li.LiPlanInfo, "li_plan_info")])
def test_ctypes_struct_matches_c_layout(tmp_path, cls, cname):
    fields = [f for f, _ in cls._fields_]
    prog = tmp_path / "probe.c"
    body = "\n".join(f'  printf("%zu\\n", offsetof({cname}, {f}));' for f in fields)
    prog.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "li.h"\nint main(void){\n'
                    f'  printf("%zu\\n", sizeof({cname}));\n{body}\n  return 0;\n}}\n')
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", str(ROOT / "include"), str(prog), "-o", str(exe)],
                   check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(cls)
    for f, off in zip(fields, vals[1:]):
        assert getattr(cls, f).offset == off, f


def _args(**kw):
    """A valid BSND argument set with fake (never dereferenced) aligned device pointers."""
    a = li.LiArgs()
    a.q, a.k, a.w = 0x10000, 0x20000, 0x30000
    a.batch, a.q_len, a.k_len = 1, 64, 64
    a.max_seqlen_q, a.max_seqlen_k = 64, 64
    a.num_heads_q, a.num_heads_k, a.head_dim, a.topk = 8, 1, 128, 16
    a.layout_q = a.layout_k = 0
    a.mask_mode = 3
    a.return_value = 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _ws_status(a):
    n = ctypes.c_size_t(0)
    return li.lib().li_indexer_workspace_size(ctypes.byref(a), ctypes.byref(n)), n.value


def test_valid_args_size_the_workspace(L):
    st, n = _ws_status(_args())
    assert st == 0
    # header + schedule + fp32 score rows (64 rows x 64 keys)
    assert n >= 256 + 64 * 64 * 4
    st, m = 0, ctypes.c_size_t(0)
    st = L.li_metadata_workspace_size(ctypes.byref(_args()), ctypes.byref(m))
    assert st == 0 and m.value > 0 and m.value % 256 == 0


@pytest.mark.parametrize("kw,status", [
    (dict(num_heads_q=0), 1), (dict(num_heads_q=65), 1), (dict(num_heads_k=2), 1),
    (dict(head_dim=64), 1), (dict(topk=0), 1), (dict(topk=8193), 1), (dict(mask_mode=1), 1),
    (dict(layout_q=2), 1), (dict(layout_k=5), 1), (dict(dtype_qk=2), 1), (dict(dtype_qk=4), 1), (dict(dtype_w=3), 1),
    (dict(dtype_qk=-1), 1), (dict(dtype_w=2, w=0x30002), 1), (dict(w=0x30001), 1), (dict(q=None), 1),
    (dict(q=0x10008), 1), (dict(layout_q=1), 1), (dict(layout_k=1), 1), (dict(layout_k=2), 1),
    (dict(layout_k=2, seqused_k=0x40000, block_table=0x50000, block_table_stride=4,
          num_blocks=4, block_size=0), 1),
    (dict(layout_k=2, seqused_k=0x40000, block_table=0x50000, block_table_stride=4,
          num_blocks=4, block_size=1025), 1),
    (dict(cu_seqlens_q=0x40000), 1), (dict(block_table=0x40000), 1), (dict(batch=-1), 1),
    (dict(max_seqlen_k=65), 1), (dict(return_value=2), 1),
    # compressed keys: residuals exactly with cmp_ratio > 1 under mask_mode 3
    (dict(cmp_ratio=-1), 1), (dict(cmp_ratio=4), 1), (dict(cmp_residual_k=0x60000), 1),
    (dict(cmp_ratio=4, mask_mode=0, cmp_residual_k=0x60000), 1),
    # 32-bit row coordinates: query rows x heads and key rows beyond 2^31-1
    (dict(batch=40000, q_len=1000, max_seqlen_q=1000, num_heads_q=64), 2),
    (dict(batch=3, k_len=1 << 30, max_seqlen_k=64), 2),
    (dict(layout_k=2, k_len=0, seqused_k=0x40000, block_table=0x50000, block_table_stride=4,
          num_blocks=1 << 25, block_size=128), 2),
])
def test_invalid_args_rejected_on_host(L, kw, status):
    st, _ = _ws_status(_args(**kw))
    assert st == status, li.li_last_error_string()
    assert li.li_last_error_string()


def test_fp8_requires_both_scales(L):
    fp8 = dict(dtype_qk=3, q_descale=0x70000, k_descale=0x74000)
    assert _ws_status(_args(**fp8))[0] == 0
    assert _ws_status(_args(dtype_qk=3))[0] == 1                        # no scales
    assert _ws_status(_args(dtype_qk=3, q_descale=0x70000))[0] == 1     # one scale
    assert _ws_status(_args(q_descale=0x70000, k_descale=0x74000))[0] == 1   # scales without fp8
    assert _ws_status(_args(**dict(fp8, k_descale=0x74002)))[0] == 1    # misaligned


@pytest.mark.parametrize("qk,w", [(0, 0), (0, 1), (0, 2), (1, 0), (1, 1), (1, 2)])
def test_every_dtype_pair_accepted(L, qk, w):
    assert _ws_status(_args(dtype_qk=qk, dtype_w=w))[0] == 0
    # a 16-bit w needs 2-byte alignment only
    if w != 2:
        assert _ws_status(_args(dtype_qk=qk, dtype_w=w, w=0x30002))[0] == 0


def _merge_args(**kw):
    a = li.LiMergeArgs()
    n = kw.pop("n_lists", 2)
    for l in range(min(n, li.MERGE_MAX_LISTS)):
        a.idx_in[l] = 0x10000 + 0x1000 * l
        a.val_in[l] = 0x40000 + 0x1000 * l
    a.idx_out, a.val_out, a.device_status = 0x80000, 0x90000, 0xA0000
    a.rows, a.n_lists, a.topk_in, a.topk_out = 0, n, 64, 64
    for k, v in kw.items():
        if k.startswith("idx_in_"):
            a.idx_in[int(k[7:])] = v
        else:
            setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw", [
    dict(n_lists=0), dict(n_lists=17), dict(rows=-1), dict(topk_in=0), dict(topk_out=8193),
    dict(topk_in=8193), dict(reserved=1), dict(idx_out=None), dict(idx_in_1=None),
    dict(idx_in_1=0x11002), dict(val_out=0x90002), dict(device_status=0xA0001)])
def test_invalid_merge_args_rejected_on_host(L, kw):
    assert L.li_merge_topk(ctypes.byref(_merge_args(**kw)), None) == 1
    assert li.li_last_error_string()


def test_merge_rows_limit_and_empty_call(L):
    assert L.li_merge_topk(ctypes.byref(_merge_args(rows=1 << 31)), None) == 2
    # no rows: validated, nothing launched (no device needed)
    assert L.li_merge_topk(ctypes.byref(_merge_args(rows=0, val_out=None, device_status=None,
                                                    n_lists=16)), None) == 0


def test_merge_args_struct_matches_the_header(L):
    # 16 + 16 list pointers, 3 more pointers, int64 rows, four int32
    assert ctypes.sizeof(li.LiMergeArgs) == 35 * 8 + 8 + 16


def _kl_args(**kw):
    a = li.LiKlArgs()
    a.q, a.k, a.qi, a.ki, a.w = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000
    a.sparse_indices, a.softmax_max, a.softmax_sum = 0x60000, 0x70000, 0x80000
    a.scale, a.batch, a.s1, a.s2 = 0.05, 2, 64, 64
    a.G, a.Dm, a.Dr, a.H, a.topk = 16, 512, 0, 64, 32
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw", [
    dict(G=0), dict(G=129), dict(H=65), dict(topk=0), dict(topk=2049), dict(Dm=0), dict(Dm=580),
    dict(Dm=100), dict(Dr=64), dict(Dr=12, q_rope=0x90000, k_rope=0xA0000), dict(G=128, Dm=512),
    dict(q=None), dict(softmax_sum=None), dict(scale=0.0), dict(reserved=1), dict(batch=-1),
    dict(q_rope=0x90000, k_rope=0xA0000), dict(w=0x50002)])
def test_invalid_kl_args_rejected_on_host(L, kw):
    n = ctypes.c_size_t(0)
    assert L.li_kl_grad_workspace_size(ctypes.byref(_kl_args(**kw)), ctypes.byref(n)) == 1
    assert li.li_last_error_string()


def test_kl_workspace_holds_a_loss_per_row(L):
    n = ctypes.c_size_t(0)
    assert L.li_kl_grad_workspace_size(ctypes.byref(_kl_args()), ctypes.byref(n)) == 0
    assert n.value >= 256 + 2 * 64 * 4
    ok = _kl_args(Dr=64, q_rope=0x90000, k_rope=0xA0000)
    assert L.li_kl_grad_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0


def test_compressed_key_args_accepted(L):
    assert _ws_status(_args(cmp_ratio=4, cmp_residual_k=0x60000))[0] == 0
    assert _ws_status(_args(cmp_ratio=4, mask_mode=0))[0] == 0
    # residuals are per batch and read on the device: the schedule kernel always runs
    pl = li.li_plan(_args(cmp_ratio=4, cmp_residual_k=0x60000))
    assert pl["dense"] == 0 and pl["kernels"] == 3


def test_topk_accepts_every_value_up_to_8192(L):
    # the pages' Atlas set is [1, 2048] plus multiples of 1024 up to 8192; every value in
    # [1, 8192] is accepted here
    for k in (1, 2047, 2048, 2049, 3000, 3072, 8191, 8192):
        st, _ = _ws_status(_args(topk=k))
        assert st == 0, k


def test_paged_args_accepted(L):
    st, n = _ws_status(_args(layout_k=2, k_len=0, seqused_k=0x40000, block_table=0x50000,
                             block_table_stride=8, num_blocks=16, block_size=64,
                             max_seqlen_k=512))
    assert st == 0 and n > 0


def test_indexer_rejects_small_workspace(L):
    a = _args()
    st = L.li_indexer(ctypes.byref(a), None, 0x100000, 16, 0x200000, 0x300000, None)
    assert st == 3
    st = L.li_indexer(ctypes.byref(a), None, 0x100010, 1 << 30, 0x200000, 0x300000, None)
    assert st == 3   # misaligned workspace
    st = L.li_indexer(ctypes.byref(a), None, 0x100000, 1 << 30, None, 0x300000, None)
    assert st == 1   # no output


def test_plan_reports_schedule_and_kernel_count(L):
    # dense causal BSND: closed-form work list, score + select kernels only
    pl = li.li_plan(_args(q_len=4096, k_len=4096, max_seqlen_q=4096, max_seqlen_k=4096,
                          num_heads_q=64, topk=2048))
    assert pl == dict(tq=4, kc=0, max_items=1024, dense=1, kernels=2, score_tc=1,
                      select_pieces=1)
    # one query row per batch (decode): tq capped by max_seqlen_q, schedule kernel needed
    pl = li.li_plan(_args(layout_k=2, k_len=0, q_len=1, max_seqlen_q=1, batch=64,
                          num_heads_q=64, seqused_k=0x40000, block_table=0x50000,
                          block_table_stride=512, num_blocks=64 * 512, block_size=64,
                          max_seqlen_k=32768, topk=2048))
    assert pl["tq"] == 1 and pl["dense"] == 2 and pl["kernels"] == 2 and pl["score_tc"] == 1
    assert pl["kc"] > 0 and pl["max_items"] >= 64 * (32768 // pl["kc"])
    # one very long decode row: its selection is cut into key pieces plus one merge kernel,
    # and the workspace grows by the pieces' lists
    long_row = dict(layout_k=2, k_len=0, q_len=1, max_seqlen_q=1, batch=1, num_heads_q=64,
                    seqused_k=0x40000, block_table=0x50000, block_table_stride=16384,
                    num_blocks=16384, block_size=64, topk=2048)
    pl = li.li_plan(_args(max_seqlen_k=1 << 20, **long_row))
    assert pl["select_pieces"] > 1 and pl["kernels"] == 3
    one = li.li_plan(_args(max_seqlen_k=16384, **long_row))
    assert one["select_pieces"] == 1 and one["kernels"] == 2
    st_a, n_split = _ws_status(_args(max_seqlen_k=1 << 20, **long_row))
    st_b, n_whole = _ws_status(_args(max_seqlen_k=(1 << 20) - 128, **long_row))
    assert st_a == st_b == 0
    # every block size runs on the tensor-core score kernel (12: pieces of 4 rows, copied row
    # by row; 1 and 1024 too)
    for bs in (1, 12, 48, 1000, 1024):
        pl = li.li_plan(_args(layout_k=2, k_len=0, seqused_k=0x40000, block_table=0x50000,
                              block_table_stride=64, num_blocks=64, block_size=bs,
                              max_seqlen_k=512))
        assert pl["score_tc"] == 1 and pl["kernels"] == 3 and pl["dense"] == 0, bs
    # no query rows: nothing launches
    assert li.li_plan(_args(batch=0))["kernels"] == 0
    # argument errors come back as status codes
    a = _args(num_heads_q=0)
    assert L.li_plan(ctypes.byref(a), ctypes.byref(li.LiPlanInfo())) == 1
    assert L.li_plan(ctypes.byref(_args()), None) == 1


def _paged(**over):
    """Paged-key fields of li_attn_args (S2 = 64 keys in blocks of 32), with overrides."""
    kw = dict(layout_k=2, block_table=0x60000, block_table_stride=2, num_blocks=8, block_size=32)
    kw.update(over)
    return kw


def _attn_args(**kw):
    a = li.LiAttnArgs()
    a.q, a.k, a.sparse_indices = 0x10000, 0x20000, 0x30000
    a.scale, a.batch, a.s1, a.s2 = 0.04, 2, 64, 64
    a.G, a.Dm, a.Dr, a.topk = 16, 512, 0, 32
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw", [
    dict(G=0), dict(G=33), dict(Dm=64), dict(Dm=576), dict(Dm=200), dict(Dr=32),
    dict(Dr=64), dict(q_rope=0x40000, k_rope=0x50000), dict(topk=0), dict(topk=8193),
    dict(scale=0.0), dict(scale=float("inf")), dict(reserved=1), dict(batch=-1), dict(s2=0),
    dict(q=None), dict(sparse_indices=None), dict(q=0x10008), dict(sparse_indices=0x30002),
    # key layouts: TND is not one; PA_BSND needs a block table, a block size in [1, 1024], at
    # least one block and a table wide enough for S2; BSND takes none of the paged fields
    dict(layout_k=1), _paged(block_table=None), _paged(block_size=0), _paged(block_size=1025),
    _paged(num_blocks=0), _paged(block_table_stride=1), _paged(block_table=0x60002),
    dict(block_table=0x60000), dict(block_size=32)])
def test_invalid_attention_args_rejected_on_host(L, kw):
    n = ctypes.c_size_t(0)
    assert L.li_sparse_attention_workspace_size(ctypes.byref(_attn_args(**kw)), ctypes.byref(n)) == 1
    assert li.li_last_error_string()


@pytest.mark.parametrize("kw", [dict(), dict(Dr=64, q_rope=0x40000, k_rope=0x50000),
                                dict(G=32, Dm=512, Dr=64, q_rope=0x40000, k_rope=0x50000),
                                dict(G=1, Dm=128), dict(batch=0, s2=0), _paged(),
                                _paged(block_size=1, block_table_stride=64),
                                _paged(block_size=1024, block_table_stride=1)])
def test_attention_args_accepted(L, kw):
    n = ctypes.c_size_t(0)
    assert L.li_sparse_attention_workspace_size(ctypes.byref(_attn_args(**kw)), ctypes.byref(n)) == 0
    assert n.value == 256
