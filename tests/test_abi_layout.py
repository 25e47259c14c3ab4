"""The ctypes mirrors in li.py match the C structs of include/li.h field by field: a small C
program built with gcc prints sizeof and offsetof of every field, and each must equal the
mirror's. (Names in the C structs that hold several declarators, e.g. `const void *q, *k`, are
listed one by one here.)"""
import ctypes
import shutil
import subprocess
from pathlib import Path

import pytest

from sparse_attention_token_lightning_b200 import li

ROOT = Path(__file__).resolve().parents[1]
MIRRORS = {"li_args": li.LiArgs, "li_plan_info": li.LiPlanInfo, "li_merge_args": li.LiMergeArgs,
           "li_kl_args": li.LiKlArgs, "li_attn_args": li.LiAttnArgs}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "li.h"', 'int main(void) {']
    for cname, mirror in MIRRORS.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _t in mirror._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    d = tmp_path_factory.mktemp("layout")
    src, exe = d / "layout.c", d / "layout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.run(["gcc", "-std=c11", "-I", str(ROOT / "include"), "-o", str(exe), str(src)],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    table = {}
    for line in out.splitlines():
        cname, fname, val = line.split()
        table[(cname, fname)] = int(val)
    return table


@pytest.mark.parametrize("cname", list(MIRRORS))
def test_mirror_matches_the_header(c_layout, cname):
    mirror = MIRRORS[cname]
    assert ctypes.sizeof(mirror) == c_layout[(cname, "size")], cname
    for fname, _t in mirror._fields_:
        assert getattr(mirror, fname).offset == c_layout[(cname, fname)], (cname, fname)


ORACLE_MIRRORS = {"orc_problem": "_Problem", "orc_kl": "_KL", "orc_attn": "_Attn"}


def test_oracle_mirrors_match_the_oracle_source(tmp_path):
    """The same check for the oracle's ctypes mirrors against the structs of li_oracle.c."""
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    from oracle import oracle as orc_mod
    lines = ['#include <stddef.h>', '#include <stdio.h>',
             f'#include "{ROOT / "oracle" / "li_oracle.c"}"', 'int main(void) {']
    for cname, pname in ORACLE_MIRRORS.items():
        mirror = getattr(orc_mod, pname)
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _t in mirror._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    src, exe = tmp_path / "olayout.c", tmp_path / "olayout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.run(["gcc", "-std=c11", "-o", str(exe), str(src), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    table = {tuple(l.split()[:2]): int(l.split()[2]) for l in out.splitlines()}
    for cname, pname in ORACLE_MIRRORS.items():
        mirror = getattr(orc_mod, pname)
        assert ctypes.sizeof(mirror) == table[(cname, "size")], cname
        for fname, _t in mirror._fields_:
            assert getattr(mirror, fname).offset == table[(cname, fname)], (cname, fname)


def test_python_constants_match_the_header():
    """Status codes, device error bits and type codes named in li.py equal the header's."""
    text = (ROOT / "include" / "li.h").read_text()
    import re
    defs = dict(re.findall(r"#define (LI_DEVERR_\w+)\s+(0x[0-9a-fA-F]+)u", text))
    for name, val in [("TIMEOUT", li.DEVERR_TIMEOUT), ("LENGTHS", li.DEVERR_LENGTHS),
                      ("TABLE", li.DEVERR_TABLE), ("OFFSET", li.DEVERR_OFFSET),
                      ("METADATA", li.DEVERR_METADATA), ("INTERNAL", li.DEVERR_INTERNAL),
                      ("MERGE_ORDER", li.DEVERR_MERGE_ORDER), ("DESCALE", li.DEVERR_DESCALE)]:
        assert int(defs["LI_DEVERR_" + name], 16) == val, name
    enum = dict((k, int(v)) for k, v in re.findall(r"(LI_(?:ERR_\w+|OK)) = (\d+)", text))
    assert {v: k for k, v in enum.items()} == li.STATUS
    dt = dict((k, int(v)) for k, v in re.findall(r"LI_DTYPE_(\w+) = (\d+)", text))
    assert dt == {"BF16": 0, "FP16": 1, "FP32": 2, "FP8_E4M3": 3}
    assert sorted(li.DTYPES.values()) == [0, 1, 2, 3]
