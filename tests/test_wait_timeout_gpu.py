"""The score kernel's bounded waits end in an error status, not a hang.

Every mbarrier wait of the tensor-core score kernel gives up after a time limit (2 s in the
library), records LI_DEVERR_TIMEOUT, makes every warp role leave its loop, frees TMEM and returns,
so li_check_status reports LI_ERR_DEVICE_TIMEOUT and the CUDA context stays usable. The library's
test build (libli_waittest.so: 1 ms limit, and a producer that issues no TMA load and never
arrives on the full barriers, so no bulk copy is ever in flight) makes the MMA warp's first wait
run out on purpose. The test checks the reported status and then that a normal call on the same
device still gives the oracle's answer. Nothing here faults, traps or spins without a limit.
"""
import ctypes
import time

import pytest
import torch

import parity
from sparse_attention_token_lightning_b200 import build, li, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def waittest_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    li.lib()
    return li.load(build.build_wait_test())


@pytest.mark.parametrize("make", [
    lambda: synthetic.bsnd(1, 256, 256, 64, 32, 3, seed=81),
    lambda: synthetic.paged([700, 300], 1, 64, 64, block_size=64, seed=82),
])
def test_wait_runs_out_and_is_reported(orc, waittest_lib, make):
    L = waittest_lib
    pb = make()
    g = pb.to("cuda")
    args = li.make_args(g)
    n = ctypes.c_size_t(0)
    assert L.li_indexer_workspace_size(ctypes.byref(args), ctypes.byref(n)) == li.LI_OK
    # zeroed workspace: the selection that follows the aborted score kernel reads zeros
    ws = torch.zeros(n.value, dtype=torch.uint8, device="cuda")
    idx = torch.empty(li.out_shape(g), dtype=torch.int32, device="cuda")
    val = torch.empty(li.out_shape(g), dtype=torch.float32, device="cuda")
    stream = li._stream_handle(None)
    plan = li.LiPlanInfo()
    assert L.li_plan(ctypes.byref(args), ctypes.byref(plan)) == li.LI_OK
    assert plan.score_tc == 1
    t0 = time.perf_counter()
    assert L.li_indexer(ctypes.byref(args), None, ws.data_ptr(), n.value, idx.data_ptr(),
                        val.data_ptr(), stream) == li.LI_OK
    bits = ctypes.c_uint32(0)
    st = L.li_check_status(ws.data_ptr(), stream, ctypes.byref(bits))
    elapsed = time.perf_counter() - t0
    assert st == 5, (st, L.li_last_error_string())                 # LI_ERR_DEVICE_TIMEOUT
    assert bits.value & li.DEVERR_TIMEOUT
    assert elapsed < 20.0
    # the context is intact: the normal library on the same device matches the oracle
    gi, gv = li.indexer(g)
    torch.cuda.synchronize()
    parity.check(orc, pb, parity.as_rows(gi, pb.topk), parity.as_rows(gv, pb.topk),
                 label="after timeout")
