"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Small problems span several 128-key tiles with ragged tails and are compared on every row; the
full-size workloads (causal prefill, paged decode, varlen, long context) run in the benchmark's
configuration and are compared on seeded samples of rows. Integer-valued inputs make every score
exact in fp32, so there the outputs must match the oracle bit for bit, ties included.
"""
import numpy as np
import pytest
import torch

import parity
from sparse_attention_token_lightning_b200 import li, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    li.lib()


def run(pb, **kw):
    g = pb.to("cuda")
    idx, val = li.indexer(g, **kw)
    torch.cuda.synchronize()
    return (parity.as_rows(idx, pb.topk), None if val is None else parity.as_rows(val, pb.topk))


def run_counting_fallbacks(pb):
    """Like run(), also returning how many rows the selection finished on its exact fallback
    path (read from the workspace header, third int32)."""
    g = pb.to("cuda")
    ws = li.empty_workspace(li.make_args(g), "cuda")
    idx, val = li.indexer(g, workspace=ws)
    torch.cuda.synchronize()
    exact_rows = int(ws[8:12].view(torch.int32).item())
    return parity.as_rows(idx, pb.topk), parity.as_rows(val, pb.topk), exact_rows


# ---- small problems, every row ------------------------------------------------------------------

SMALL = {
    "tiny": lambda: synthetic.config("tiny"),
    "pages_example": lambda: synthetic.config("pages_example"),
    "bsnd_causal_ragged": lambda: synthetic.bsnd(2, 300, 459, 64, 200, 3, seed=3),
    "bsnd_nomask_n1": lambda: synthetic.bsnd(1, 40, 333, 1, 64, 0, seed=4),
    "bsnd_n3_topk_gt_keys": lambda: synthetic.bsnd(1, 50, 130, 3, 256, 3, seed=5),
    "bsnd_n16_q_longer": lambda: synthetic.bsnd(2, 200, 150, 16, 32, 3, seed=6),
    "tnd_varlen": lambda: synthetic.tnd([1, 130, 77, 0, 256], [300, 130, 500, 9, 256], 64, 100,
                                        3, seed=7),
    "tnd_nomask": lambda: synthetic.tnd([17, 5], [40, 290], 8, 50, 0, seed=8),
    "paged_bs64": lambda: synthetic.paged([700, 129, 1, 64], 3, 64, 128, block_size=64,
                                          seed=9, spare_blocks=5),
    "paged_bs16_tnd_q": lambda: synthetic.paged([300, 45], 0, 32, 64, block_size=16, seed=10,
                                                layout_q="TND", lens_q=[4, 2]),
    "paged_bs48": lambda: synthetic.paged([333, 200], 2, 16, 40, block_size=48, seed=11),
    "paged_bs1": lambda: synthetic.paged([37, 3], 1, 4, 8, block_size=1, seed=12),
    "topk1": lambda: synthetic.bsnd(1, 64, 200, 8, 1, 3, seed=13),
    "topk8192": lambda: synthetic.bsnd(1, 8, 9000, 2, 8192, 0, seed=14),
    "topk8192_n16": lambda: synthetic.bsnd(1, 4, 9000, 16, 8192, 0, seed=45),
    "offset_seqused": lambda: synthetic.tnd([10, 30], [60, 90], 4, 40, 3, seed=15,
                                            seqused_q=[7, 30], output_idx_offset=[1000, 5]),
    # head counts that do not divide 256: tq = 5 / 10 rows, N = 240 (generic epilogue path)
    "bsnd_n48": lambda: synthetic.bsnd(2, 130, 260, 48, 100, 3, seed=47),
    "bsnd_n24_nomask": lambda: synthetic.bsnd(1, 50, 300, 24, 64, 0, seed=48),
    # paged blocks of one full key tile, of two tiles, and without a mask
    "paged_bs128": lambda: synthetic.paged([600, 300], 2, 64, 128, block_size=128, seed=49),
    "paged_bs256_nomask": lambda: synthetic.paged([700, 90], 1, 32, 64, block_size=256,
                                                  mask_mode=0, seed=50),
    # small blocks over long windows: more than 32 key pieces per item (staged rows refilled)
    "paged_bs16_long": lambda: synthetic.paged([1500, 700], 2, 16, 100, block_size=16, seed=52),
    "paged_bs8_long": lambda: synthetic.paged([1900], 1, 8, 64, block_size=8, seed=53),
    # compressed keys (cmp_ratio > 1, per-batch residuals) under the right-down mask
    "cmp_pages_example": lambda: synthetic.compressed(
        synthetic.bsnd(2, 64, 130 // 4, 16, 32, 3, seed=59), 4, [130 % 4, 130 % 4]),
    "cmp_bsnd_ragged": lambda: synthetic.compressed(
        synthetic.bsnd(2, 300, 120, 64, 64, 3, seed=60), 3, [2, 0]),
    "cmp_tnd": lambda: synthetic.compressed(
        synthetic.tnd([200, 40, 1], [60, 70, 5], 64, 32, 3, seed=61), 4, [3, 1, 0]),
    "cmp_paged_decode": lambda: synthetic.compressed(
        synthetic.paged([3000, 700], 1, 64, 128, block_size=64, seed=62), 8, [7, 2]),
    "cmp_nomask": lambda: synthetic.compressed(synthetic.bsnd(1, 50, 90, 8, 40, 0, seed=63), 4,
                                               None),
    # few query blocks and long windows: key ranges split across work items
    "paged_decode_split": lambda: synthetic.paged([5000, 3000, 100], 1, 64, 256, block_size=64,
                                                  seed=51),
    # block sizes the TMA pieces do not tile at 8 rows: pieces of the largest power of two
    # dividing the block size (24: 8, 1000: 8) or row copies below 8 (3, 100: 4, 6: 2)
    "paged_bs3": lambda: synthetic.paged([200, 31, 2], 2, 16, 32, block_size=3, seed=64),
    "paged_bs6_tnd_q": lambda: synthetic.paged([150, 40], 0, 8, 24, block_size=6, seed=65,
                                               layout_q="TND", lens_q=[20, 7]),
    "paged_bs24": lambda: synthetic.paged([500, 130], 2, 64, 100, block_size=24, seed=66),
    "paged_bs100_decode": lambda: synthetic.paged([1300, 700, 90], 1, 64, 128, block_size=100,
                                                  seed=67),
    "paged_bs1000": lambda: synthetic.paged([2500, 999], 1, 32, 200, block_size=1000, seed=68),
    "paged_bs1024": lambda: synthetic.paged([3000, 1025, 1], 2, 64, 256, block_size=1024,
                                            seed=69),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(orc, name):
    pb = SMALL[name]()
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, label=name)


@pytest.mark.parametrize("name", [n for n in SMALL if n.startswith("paged")])
def test_every_block_size_takes_the_tensor_core_kernel(name):
    """Paged keys of any block size in [1, 1024] run on the tcgen05 score kernel: TMA pieces of
    the largest power of two dividing the block size when that is 8 or more, row copies
    otherwise (lightning_indexer, "Constraints": block size 1 to 1024)."""
    pb = SMALL[name]()
    assert li.li_plan(li.make_args(pb))["score_tc"] == 1


EXACT = {
    "bsnd_causal": lambda: synthetic.bsnd(2, 333, 333, 64, 100, 3, seed=20, integer=True),
    "bsnd_n4_nomask": lambda: synthetic.bsnd(1, 100, 260, 4, 300, 0, seed=21, integer=True),
    "tnd": lambda: synthetic.tnd([5, 200, 1], [129, 200, 700], 16, 64, 3, seed=22, integer=True),
    "paged": lambda: synthetic.paged([500, 64, 65], 2, 64, 96, block_size=64, seed=23,
                                     integer=True, spare_blocks=2),
    "paged_bs1_rows": lambda: synthetic.paged([300, 64, 5], 2, 16, 96, block_size=1, seed=24,
                                              integer=True, spare_blocks=3),
    "paged_bs48_pieces": lambda: synthetic.paged([500, 47], 1, 64, 128, block_size=48, seed=25,
                                                 integer=True),
}


@pytest.mark.parametrize("name", list(EXACT))
def test_integer_inputs_bit_exact(orc, name):
    pb = EXACT[name]()
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, exact=True, label=name)


# q and k in fp16 (one type for both), w in bf16, fp16 or fp32: the MMA takes fp16 operands and
# the weights are staged as fp32, so the oracle decodes the same bits
DT = synthetic.with_dtypes
DTYPE_CASES = {
    "pages_example_fp16_fp32": lambda: DT(synthetic.config("pages_example"), "fp16", "fp32"),
    "bsnd_causal_ragged_fp16_fp16": lambda: DT(SMALL["bsnd_causal_ragged"](), "fp16", "fp16"),
    "bsnd_n48_fp16_bf16": lambda: DT(SMALL["bsnd_n48"](), "fp16", "bf16"),
    "tnd_varlen_bf16_fp32": lambda: DT(SMALL["tnd_varlen"](), "bf16", "fp32"),
    "paged_bs64_fp16_fp32": lambda: DT(SMALL["paged_bs64"](), "fp16", "fp32"),
    "paged_decode_split_fp16_fp32": lambda: DT(SMALL["paged_decode_split"](), "fp16", "fp32"),
    "paged_bs16_long_bf16_fp16": lambda: DT(SMALL["paged_bs16_long"](), "bf16", "fp16"),
    "cmp_tnd_fp16_fp32": lambda: DT(SMALL["cmp_tnd"](), "fp16", "fp32"),
    "topk8192_n16_fp16_fp32": lambda: DT(SMALL["topk8192_n16"](), "fp16", "fp32"),
}


@pytest.mark.parametrize("name", list(DTYPE_CASES))
def test_dtype_parity(orc, name):
    pb = DTYPE_CASES[name]()
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, label=name)
    assert exact_rows == 0


@pytest.mark.parametrize("qk,w", [("fp16", "fp32"), ("fp16", "fp16"), ("bf16", "fp32")])
@pytest.mark.parametrize("name", ["bsnd_causal", "paged"])
def test_integer_inputs_bit_exact_in_every_dtype(orc, name, qk, w):
    pb = DT(EXACT[name](), qk, w)
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, exact=True, label=f"{name} {qk} {w}")


def test_dtypes_change_only_the_rounding(orc):
    """Integer-valued inputs are exact in every type: all six q/k and w type pairs must give
    the same bits on the device."""
    base = EXACT["tnd"]()
    ref = run(base)
    for qk in ("bf16", "fp16"):
        for w in ("bf16", "fp16", "fp32"):
            got = run(DT(base, qk, w))
            assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]), (qk, w)


# fp8 e4m3 q and k with per-(row, head) and per-key scales (kind::f8f6f4 MMA)
Q8 = synthetic.quantized
FP8_CASES = {
    "pages_example_fp8": lambda: Q8(synthetic.config("pages_example")),
    "bsnd_causal_ragged_fp8": lambda: Q8(SMALL["bsnd_causal_ragged"]()),
    "bsnd_n48_fp8": lambda: Q8(SMALL["bsnd_n48"]()),
    "bsnd_n16_fp8_fp32w": lambda: (lambda pb: pb.replace(w=pb.w.float()))(
        Q8(SMALL["bsnd_n16_q_longer"]())),
    "tnd_varlen_fp8": lambda: Q8(SMALL["tnd_varlen"]()),
    "paged_bs64_fp8": lambda: Q8(SMALL["paged_bs64"]()),
    "paged_bs16_long_fp8": lambda: Q8(SMALL["paged_bs16_long"]()),
    "paged_decode_split_fp8": lambda: Q8(SMALL["paged_decode_split"]()),
    "paged_bs256_nomask_fp8": lambda: Q8(SMALL["paged_bs256_nomask"]()),
    "paged_bs3_fp8": lambda: Q8(SMALL["paged_bs3"]()),
    "paged_bs100_decode_fp8": lambda: Q8(SMALL["paged_bs100_decode"]()),
}


@pytest.mark.parametrize("name", list(FP8_CASES))
def test_fp8_parity(orc, name):
    pb = FP8_CASES[name]()
    assert li.li_plan(li.make_args(pb))["score_tc"] == 1
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, label=name)


@pytest.mark.parametrize("name", list(EXACT))
def test_fp8_unit_scales_bit_exact(orc, name):
    pb = Q8(EXACT[name](), unit_scales=True)
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, exact=True, label=f"{name} fp8")


@pytest.mark.parametrize("name", ["bsnd_causal", "paged"])
def test_fp8_power_of_two_scales_bit_exact(orc, name):
    """Integer codes with power-of-two scales: every product and partial sum is exact in fp32,
    so the device must match the oracle bit for bit, which checks where each scale applies."""
    base = EXACT[name]()
    g = torch.Generator().manual_seed(130)
    qs = 2.0 ** torch.randint(-2, 3, base.w.shape, generator=g).float()
    ks = 2.0 ** torch.randint(-2, 3, base.k.shape[:-2], generator=g).float()
    pb = base.replace(q=base.q.float().to(torch.float8_e4m3fn),
                      k=base.k.float().to(torch.float8_e4m3fn), q_descale=qs, k_descale=ks)
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, exact=True, label=f"{name} fp8 scaled")


def test_fp8_bad_scale_reported():
    pb = Q8(synthetic.bsnd(1, 20, 60, 8, 16, 3, seed=131))
    ks = pb.k_descale.clone()
    ks[0, 5] = 0.0
    with pytest.raises(li.LiError) as e:
        li.indexer(pb.replace(k_descale=ks).to("cuda"))
    assert "0x80" in str(e.value)


def test_indices_only(orc):
    pb = synthetic.bsnd(1, 64, 300, 8, 50, 3, seed=30)
    gi, gv = run(pb, return_value=False)
    assert gv is None
    gi2, gv2 = run(pb)
    assert np.array_equal(gi, gi2)


def test_separate_metadata_matches_inline():
    pb = synthetic.tnd([100, 3, 250], [100, 400, 260], 64, 64, 3, seed=31)
    a = run(pb, metadata=False)
    b = run(pb, metadata=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


@pytest.mark.parametrize("shape", [(2, 300, 459, 64, 200, 3), (1, 200, 150, 16, 32, 3),
                                   (3, 64, 64, 8, 16, 0)])
def test_dense_closed_form_schedule_matches_metadata(shape):
    """Dense BSND problems run without a schedule kernel (closed-form work list); a schedule
    built by li_metadata for the same call must give bit-identical outputs."""
    pb = synthetic.bsnd(*shape, seed=46)
    a = run(pb, metadata=False)
    b = run(pb, metadata=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


@pytest.mark.parametrize("make", [
    lambda: synthetic.paged([5000, 3000, 100], 1, 64, 256, block_size=64, seed=54),
    lambda: synthetic.paged([300, 45, 0], 2, 32, 64, block_size=16, seed=55),
    lambda: synthetic.bsnd(3, 1, 3000, 64, 100, 3, seed=56, seqused_k=[3000, 10, 2500]),
    lambda: synthetic.bsnd(2, 3, 700, 16, 40, 0, seed=57, seqused_k=[700, 0]),
    # more batches than the score kernel's register-held work list takes (256)
    lambda: synthetic.paged([(7 * b) % 400 + 1 for b in range(300)], 1, 8, 32, block_size=16,
                            seed=58),
])
def test_decode_closed_form_schedule_matches_metadata(orc, make):
    """One query block per batch with per-batch key lengths: the work list is a closed form of
    seqused_k (no schedule kernel); an explicit schedule must give bit-identical outputs, and
    both must match the oracle."""
    pb = make()
    assert li.li_plan(li.make_args(pb))["dense"] == 2
    a = run(pb, metadata=False)
    b = run(pb, metadata=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))
    parity.check(orc, pb, a[0], a[1], label="decode closed form")


@pytest.mark.parametrize("make", [
    lambda seed: synthetic.bsnd(1, 300, 300, 64, 64, 3, seed=seed),
    lambda seed: synthetic.paged([900, 300, 4100], 1, 64, 128, block_size=64, seed=seed),
    lambda seed: synthetic.tnd([100, 3, 250], [100, 400, 260], 64, 64, 3, seed=seed),
])
def test_indexer_replays_in_a_cuda_graph(make):
    """li_indexer launches stream-ordered work only, so a captured call replays: new data copied
    into the same buffers gives the outputs of an eager call on that data, bit for bit."""
    pb = make(60).to("cuda")
    args = li.make_args(pb)
    ws = li.empty_workspace(args, "cuda")
    idx = torch.empty(li.out_shape(pb), dtype=torch.int32, device="cuda")
    val = torch.empty(li.out_shape(pb), dtype=torch.float32, device="cuda")
    li.li_indexer(args, None, ws, idx, val)        # first call outside capture
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        li.li_indexer(args, None, ws, idx, val, side)
    fresh = make(61)
    for f in synthetic.Problem.TENSORS:        # data, lengths and block table alike
        if getattr(pb, f) is not None:
            getattr(pb, f).copy_(getattr(fresh, f))
    g.replay()
    torch.cuda.synchronize()
    st, bits = li.li_check_status(ws)
    assert st == li.LI_OK, bits
    ei, ev = li.indexer(fresh.to("cuda"))
    assert torch.equal(idx, ei) and torch.equal(val.view(torch.int32), ev.view(torch.int32))


def test_deterministic_reruns():
    pb = synthetic.bsnd(1, 1024, 1024, 64, 256, 3, seed=32).to("cuda")
    i1, v1 = li.indexer(pb)
    i2, v2 = li.indexer(pb)
    assert torch.equal(i1, i2) and torch.equal(v1.view(torch.int32), v2.view(torch.int32))


def test_batch_without_rows():
    pb = synthetic.bsnd(0, 16, 16, 4, 8, 3, seed=33)
    gi, gv = run(pb)
    assert gi.size == 0


# ---- device-data errors are reported, not faulted ------------------------------------------------

def _status_of(pb):
    g = pb.to("cuda")
    args = li.make_args(g)
    ws = li.empty_workspace(args, "cuda")
    idx = torch.empty(li.out_shape(g), dtype=torch.int32, device="cuda")
    val = torch.empty(li.out_shape(g), dtype=torch.float32, device="cuda")
    li.li_indexer(args, None, ws, idx, val)
    return li.li_check_status(ws)


def test_bad_cu_seqlens_reported():
    pb = synthetic.tnd([10, 10], [20, 20], 4, 8, 3, seed=34)
    pb.cu_seqlens_k = torch.tensor([0, 25, 20], dtype=torch.int32)   # not monotone
    st, bits = _status_of(pb)
    assert st == 6 and bits & li.DEVERR_LENGTHS


def test_bad_block_table_reported():
    pb = synthetic.paged([100, 50], 1, 4, 8, block_size=16, seed=35)
    pb.block_table[0, 2] = pb.num_blocks + 7                            # outside the cache
    st, bits = _status_of(pb)
    assert st == 6 and bits & li.DEVERR_TABLE


def test_offset_overflow_reported():
    pb = synthetic.bsnd(1, 4, 40, 4, 8, 3, seed=36, output_idx_offset=[2**31 - 10])
    st, bits = _status_of(pb)
    assert st == 6 and bits & li.DEVERR_OFFSET


def test_mismatched_metadata_reported():
    pb = synthetic.bsnd(1, 64, 64, 4, 8, 3, seed=37).to("cuda")
    other = synthetic.bsnd(1, 64, 64, 4, 8, 0, seed=37).to("cuda")    # other mask mode
    meta = torch.empty(li.li_metadata_workspace_size(li.make_args(other)), dtype=torch.uint8,
                       device="cuda")
    li.li_metadata(li.make_args(other), meta)
    args = li.make_args(pb)
    ws = li.empty_workspace(args, "cuda")
    idx = torch.empty(li.out_shape(pb), dtype=torch.int32, device="cuda")
    val = torch.empty(li.out_shape(pb), dtype=torch.float32, device="cuda")
    li.li_indexer(args, meta, ws, idx, val)
    st, bits = li.li_check_status(ws)
    assert st == 6 and bits & li.DEVERR_METADATA


def test_compressed_residual_out_of_range_reported():
    pb = synthetic.compressed(synthetic.bsnd(2, 8, 20, 4, 8, 3, seed=64), 4, [1, 4])
    st, bits = _status_of(pb)
    assert st == 6 and bits & li.DEVERR_LENGTHS


def test_seqused_k_above_max_reported():
    pb = synthetic.paged([100, 50], 1, 4, 8, block_size=16, seed=38)
    pb.max_seqlen_k = 60                                               # batch 0 has 100 keys
    st, bits = _status_of(pb)
    assert st == 6 and bits & li.DEVERR_LENGTHS


# ---- full-size workloads, sampled rows -----------------------------------------------------------

FULL = {
    # name: (rows to sample, rows that must be checked)
    "causal_prefill": (24, (0, 1, 127, 128, 2046, 2047, 2048, 2049, 4095)),
    "paged_decode": (8, (0, 63)),
    "varlen": (16, (0, 32767)),
    "long_2048": (6, (0, 2047, 2048, 65535)),
    "long_8192": (4, (8191, 8192, 65535)),
    "cmp_prefill": (16, (0, 3, 4, 2047, 4095)),
    "fp16_prefill": (16, (0, 2047, 4095)),
    "fp8_prefill": (16, (0, 2047, 4095)),
    "fp8_decode": (8, (0, 63)),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled(orc, name):
    pb = synthetic.config(name)
    n, must = FULL[name]
    rows = parity.sample_rows(pb, n, seed=1, must=must)
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, rows=rows, label=name)
    assert exact_rows == 0, f"{exact_rows} rows left the bucket selection paths"


FULL_EXACT = {
    # name: (problem, rows to sample, rows that must be checked). Integer-valued inputs make every
    # score exact in fp32, so these compare bit for bit, tie order included, at the benchmark's
    # shapes: the headline causal prefill (rows around the topk = 2048 boundary and the longest
    # row), topk 8192 over rows of more than 8192 keys, and paged decode rows of up to 32K keys.
    "causal_prefill": (lambda: synthetic.config("causal_prefill", integer=True), 16,
                       (0, 1, 127, 2046, 2047, 2048, 2049, 4094, 4095)),
    "topk8192_long_rows": (lambda: synthetic.bsnd(1, 48, 12000, 16, 8192, 3, seed=73,
                                                  integer=True, name="topk8192_long_rows"),
                           48, ()),
    "paged_decode": (lambda: synthetic.config("paged_decode", integer=True), 8, ()),
}


@pytest.mark.parametrize("name", list(FULL_EXACT))
def test_full_size_integer_inputs_bit_exact(orc, name):
    make, n, must = FULL_EXACT[name]
    pb = make()
    if name == "paged_decode":
        # the longest and the shortest decode rows, plus a seeded sample
        lens = pb.seqused_k.tolist()
        must = (int(np.argmax(lens)), int(np.argmin(lens)))
        assert max(lens) > 32000
    rows = parity.sample_rows(pb, n, seed=2, must=must)
    gi, gv = run(pb)
    parity.check(orc, pb, gi, gv, rows=rows, exact=True, label=f"{name} integer")


@pytest.mark.parametrize("name", ["tiny", "bsnd_causal_ragged", "tnd_varlen", "paged_bs64",
                                  "topk8192_n16", "paged_bs16_tnd_q", "offset_seqused"])
def test_tie_free_rows_use_the_bucket_paths(orc, name):
    """Random-normal scores have (almost) no exact ties, so every row must finish on the bucket
    paths (registers for short rows, digit histogram + candidates for long rows); the exact
    radix path is only for tie-heavy rows. Guards against a fast path silently falling back."""
    pb = SMALL[name]()
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, label=name)
    assert exact_rows == 0


def test_long_rows_with_small_topk(orc):
    """Rows well past the register path (up to 12000 keys) selecting few keys: exercises the
    long-row digit histogram, the candidate gather and the bucket sort on the candidates."""
    pb = synthetic.tnd([3, 1, 2], [12000, 4097, 9000], 64, 100, 3, seed=44)
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, label="long rows")
    assert exact_rows == 0


def test_tie_heavy_rows_fall_back_correctly(orc):
    """One head and no weight: about half the keys score exactly 0, one bucket overflows, and
    the exact radix path must produce the same answer as the oracle."""
    pb = SMALL["bsnd_nomask_n1"]()
    gi, gv, exact_rows = run_counting_fallbacks(pb)
    parity.check(orc, pb, gi, gv, label="ties")
    assert exact_rows > 0


# ---- the two score kernels agree ------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "bsnd_causal_ragged", "paged_bs64", "tnd_varlen",
                                  "pages_example_fp16_fp32", "paged_bs16_long_bf16_fp16",
                                  "bsnd_causal_ragged_fp8", "paged_bs64_fp8"])
def test_cuda_core_score_kernel_matches_tensor_core(orc, name, monkeypatch):
    """LI_SCORE_KERNEL=simple selects the CUDA-core score kernel (a debugging path); both
    kernels must produce outputs that agree under the parity tolerance."""
    pb = (SMALL[name]() if name in SMALL else DTYPE_CASES[name]() if name in DTYPE_CASES
          else FP8_CASES[name]())
    a = run(pb)
    monkeypatch.setenv("LI_SCORE_KERNEL", "simple")
    b = run(pb)
    parity.check_pair(orc, pb, a[0], a[1], b[0], b[1], label=name)
