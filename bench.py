#!/usr/bin/env python
"""Benchmark of the Lightning Indexer forward pass on B200.

One step = one li_indexer call on one batch of synthetic input: schedule build, score kernel
(ReLU, weights, head sum, mask fused), top-k selection and padding, i.e. the whole hot path.
Default workload: causal prefill, B=1, S1=S2=4096, N1=64, D=128, topk=2048, right-down causal
mask, BSND, bf16 inputs (fp32 accumulation); other workloads by --config (paged decode,
varlen, long context, compressed keys, fp16 and fp8 inputs, one long row). The metric is query
tokens per second; the roofline object reports the score kernel's tensor throughput against the
measured bf16 peak (the HBM bandwidth for paged keys).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

Multi-GPU (torchrun): each rank runs its own independent problem (seed = rank); no data-path
collective exists because query rows are independent (weak scaling). The key-sharded workload
(--config long_row_decode) splits one long row's keys across the ranks instead: every rank
selects in its range, the lists are all-gathered (NCCL) and merged by li_merge_topk (strong
scaling). The reported time is the max over ranks of the device time of the K steps.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from sparse_attention_token_lightning_b200 import li, shard, synthetic  # noqa: E402

METRIC = "indexer query-tokens/s; TFLOP/s as % bf16 tensor peak (N1=64,D=128,topk=2048)"
UNIT = "query-tokens/s"
L2_FLUSH_BYTES = 256 << 20

WORKLOAD_TEXT = {
    "causal_prefill": "causal prefill: B=1, S1=S2=4096, N1=64, N2=1, D=128, topk=2048, "
                      "mask_mode=3, BSND, q,k ~N(0,1), w ~N(0,1/64), bf16",
    "tiny": "tiny prefill: B=1, S1=S2=256, N1=4, D=128, topk=32, mask_mode=3, BSND",
    "paged_decode": "paged decode: B=64, S1=1, N1=64, D=128, topk=2048, mask_mode=3, PA_BSND "
                    "block_size=64, seqused_k~U[4096,32768], permuted block_table",
    "varlen": "varlen TND: 8 sequences summing to T1=T2=32768, N1=64, D=128, topk=2048, "
              "mask_mode=3",
    "long_2048": "long-context prefill: B=1, S1=S2=65536, N1=64, D=128, topk=2048, mask_mode=3",
    "long_8192": "long-context prefill: B=1, S1=S2=65536, N1=64, D=128, topk=8192, mask_mode=3",
    "cmp_prefill": "compressed-key causal prefill: B=1, S1=4096 queries, 4096 original tokens "
                   "compressed 4:1 into 1024 keys (cmp_ratio=4, residual 0), N1=64, D=128, "
                   "topk=512, mask_mode=3, BSND",
    "fp16_prefill": "causal prefill in fp16: B=1, S1=S2=4096, N1=64, N2=1, D=128, topk=2048, "
                    "mask_mode=3, BSND, q,k fp16 ~N(0,1), w fp32 ~N(0,1/64)",
    "fp8_prefill": "causal prefill, fp8: B=1, S1=S2=4096, N1=64, D=128, topk=2048, mask_mode=3, "
                   "BSND, q and k e4m3 with per-(row, head) and per-key fp32 scales, w bf16",
    "fp8_decode": "paged decode, fp8: B=64, S1=1, N1=64, D=128, topk=2048, mask_mode=3, PA_BSND "
                  "block_size=64, seqused_k~U[4096,32768], q and k e4m3 with fp32 scales",
    "long_row_decode": "one decode row over a long context: B=1, S1=1, seqused_k=1048576, N1=64, "
                       "D=128, topk=2048, mask_mode=3, PA_BSND block_size=64; on N GPUs each "
                       "holds 1/N of the keys, selects in its range, then all-gather + merge",
}
WORKLOAD_TEXT["kl_backward"] = (
    "indexer backward with the KL loss: B=1, S1=S2=2048 causal, 1024 selected keys per row, main "
    "attention G=16 heads of Dm=512 + Dr=64, indexer H=64 heads of 128, bf16 inputs, fp32 "
    "outputs")
WORKLOAD_TEXT["sparse_attention"] = (
    "sparse attention over the selected keys: B=1, S1=S2=4096 causal, each row min(2048, i+1) "
    "selected keys (random, indexer-shaped), G=16 heads of Dm=512 + Dr=64, values = keys, bf16 "
    "inputs, fp32 outputs and statistics")

# workloads whose keys (not rows) are split across GPUs: strong scaling, all-gather + merge
KEY_SHARDED = ("long_row_decode",)


def valid_pairs(pb) -> int:
    """(query row, key) pairs inside the mask windows, from the integer lengths alone."""
    if pb.layout_q == "TND":
        cu = pb.cu_seqlens_q.tolist()
        L1s = [cu[i + 1] - cu[i] for i in range(pb.batch)]
    else:
        L1s = [pb.q_len] * pb.batch
    if pb.layout_k == "TND":
        cu = pb.cu_seqlens_k.tolist()
        L2s = [cu[i + 1] - cu[i] for i in range(pb.batch)]
    elif pb.layout_k == "PA_BSND":
        L2s = pb.seqused_k.tolist()
    else:
        L2s = [pb.k_len] * pb.batch
    if pb.seqused_k is not None and pb.layout_k != "PA_BSND":
        L2s = [min(a, b) for a, b in zip(L2s, pb.seqused_k.tolist())]
    total = 0
    for b in range(pb.batch):
        L1, L2 = L1s[b], L2s[b]
        used = L1 if pb.seqused_q is None else min(L1, int(pb.seqused_q[b]))
        if pb.mask_mode == 0:
            total += used * max(L2, 0)
            continue
        # row i sees min(L2, max(0, i + L2 - used + 1)) keys; compressed keys (r original tokens
        # each, res past the last whole key): min(L2, max(0, (i + L2*r + res - used + 1) // r))
        r = int(getattr(pb, "cmp_ratio", 1) or 1)
        if r > 1 and pb.cmp_residual_k is not None:
            res = int(pb.cmp_residual_k[b])
            for i in range(used):
                total += min(L2, max(0, (i + L2 * r + res - used + 1) // r))
            continue
        lo = L2 - used + 1
        for i in range(used):
            total += min(L2, max(0, i + lo))
    return total


def key_bytes(pb) -> int:
    """Bytes of keys the path must read once: one key row (256 B in 16-bit types, 128 B in fp8,
    plus its 4-byte scale) per valid key per batch."""
    row = pb.head_dim * pb.k.element_size() + (4 if pb.k_descale is not None else 0)
    if pb.layout_k == "PA_BSND":
        return int(pb.seqused_k.sum()) * row
    return pb.k.numel() // pb.head_dim * row


def score_kernel_bytes(pb, pairs) -> int:
    """Algorithmic DRAM bytes of one score-kernel launch: each valid key once (256 B), q and w
    of every query row, the block table rows in use, and the fp32 score of every valid pair."""
    q = pb.q.numel() * pb.q.element_size()
    w = pb.w.numel() * pb.w.element_size() * (2 if pb.q_descale is not None else 1)
    table = 0
    if pb.layout_k == "PA_BSND":
        table = sum(-(-int(L) // pb.block_size) for L in pb.seqused_k.tolist()) * 4
    return key_bytes(pb) + q + w + table + pairs * 4


# DRAM traffic of one launch of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum
# from one ncu capture of `python bench.py [--config NAME] --steps 3 --warmup 3 --cpu-seconds 0`
# (plus --no-e2e for the indexer workloads)), with the sha256 of the kernel's sources the
# counters were taken on; reported only while the sources still match. Writes that stay in L2
# when the kernel ends are not in the counter.
SCORE_SOURCES = ('sparse_attention_token_lightning_b200/csrc/li_score_tc.cu', 'sparse_attention_token_lightning_b200/csrc/li_internal.cuh', 'sparse_attention_token_lightning_b200/csrc/li_sm100.cuh')
ATTN_SOURCES = ('sparse_attention_token_lightning_b200/csrc/li_attn.cu', 'sparse_attention_token_lightning_b200/csrc/li_attn.cuh', 'sparse_attention_token_lightning_b200/csrc/li_internal.cuh', 'sparse_attention_token_lightning_b200/csrc/li_sm100.cuh')
KL_SOURCES = ('sparse_attention_token_lightning_b200/csrc/li_kl_tc.cu', 'sparse_attention_token_lightning_b200/csrc/li_kl.cuh', 'sparse_attention_token_lightning_b200/csrc/li_internal.cuh', 'sparse_attention_token_lightning_b200/csrc/li_sm100.cuh')
KERNEL_TRAFFIC = {
    "causal_prefill": {"bytes": 68751360 + 9356800, "sources": SCORE_SOURCES,
                       "src_sha256": "0095f6af9f2a659de9051d799cffc612e39053c51bce781b29188ccd99b6dbb1"},
    "sparse_attention": {"bytes": 114988544 + 90959360, "sources": ATTN_SOURCES,
                         "src_sha256": "85c665056494cd6af8891ba21c3073d1d5b42028e4eb8c30becb916f8f960201"},
    "kl_backward": {"bytes": 340291840 + 611383296, "sources": KL_SOURCES,
                    "src_sha256": "b6e122e3ad169be982fbbcac26ef1a02db549224c351af4bc4412770a057ef56"},
}


def kernel_traffic(config: str):
    import hashlib
    rec = KERNEL_TRAFFIC.get(config)
    if rec is None:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        h.update((ROOT / f).read_bytes())
    return rec["bytes"] if h.hexdigest() == rec["src_sha256"] else None


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def host_cpu() -> dict:
    """The host's CPU model and logical core count (the oracle timing runs on one of them)."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu": model, "nproc": os.cpu_count()}


class one_core:
    """Context manager: the process runs on one host core (the lowest it may use) inside the
    block, and on its previous cores again afterwards."""

    def __enter__(self):
        self.saved = None
        if hasattr(os, "sched_getaffinity"):
            self.saved = os.sched_getaffinity(0)
            self.core = min(self.saved)
            os.sched_setaffinity(0, {self.core})
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False


def usable_cores() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def cpu_oracle_rate(pb, seconds: float, seed: int = 0):
    """Time the CPU oracle (as it stands, one thread, pinned to one core) on seeded random rows of
    the workload for about `seconds`; returns (query rows per second, rows timed, seconds)."""
    import numpy as np
    from oracle import oracle as orc

    bound = orc.default().bind(pb)
    rng = np.random.default_rng(seed)
    order = rng.permutation(pb.rows)
    done, t_total, chunk = 0, 0.0, 4
    with one_core():
        while done < pb.rows and t_total < seconds:
            rows = order[done: done + chunk]
            t0 = time.perf_counter()
            bound.topk(rows)
            t_total += time.perf_counter() - t0
            done += len(rows)
            chunk = min(chunk * 2, 256)
    return done / t_total, done, t_total


def cpu_oracle_rate_parallel(pb, rows: int, threads: int, seed: int = 7):
    """The same oracle, unchanged, over `rows` seeded random rows split across `threads` host
    threads (each calls the C oracle on its own share; the C call releases the interpreter lock):
    a row-parallel figure beside the single-core one. Returns (rows per second, rows, seconds)."""
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as orc

    bound = orc.default().bind(pb)
    rng = np.random.default_rng(seed)
    pick = rng.permutation(pb.rows)[: max(rows, threads)]
    shares = np.array_split(pick, threads)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda r: bound.topk(r) if len(r) else None, shares))
    t = time.perf_counter() - t0
    return len(pick) / t, len(pick), t


def cpu_baseline(pb, seconds: float) -> dict:
    """cpu_baseline of the bench line: the oracle on one pinned core for about `seconds`, plus a
    labelled row-parallel figure on all usable host cores (about a third of that time)."""
    rate, n, t = cpu_oracle_rate(pb, seconds)
    threads = usable_cores()
    out = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{n} seeded-random query rows of the same workload, {t:.1f} s, "
                     "single-threaded C oracle (fp64) pinned to one host core; rows/s scales to "
                     "the workload (row cost is unbiased)",
           "host": host_cpu()}
    if threads > 1:
        prate, pn, pt = cpu_oracle_rate_parallel(pb, int(rate * threads * seconds / 3), threads)
        out["row_parallel"] = {"value": prate, "unit": UNIT, "threads": threads,
                               "sample": f"{pn} seeded-random rows split over {threads} host "
                                         f"threads, {pt:.1f} s, the same oracle unchanged"}
    return out


def run_reference_kl(a):
    """The reference arm of the backward workload: the oracle on the 16 longest rows per step."""
    from oracle import oracle as orc
    kp = synthetic.kl_config(a.config)
    rows = kp.w.shape[0] * kp.w.shape[1]
    part = synthetic.kl_rows(kp, rows - 16, rows)
    o = orc.default()
    times = []
    with one_core():
        for _ in range(a.warmup):
            o.kl_grad(part)
        for _ in range(a.steps):
            t0 = time.perf_counter()
            o.kl_grad(part)
            times.append(time.perf_counter() - t0)
    t = statistics.mean(times)
    line = {"metric": "indexer backward query-rows/s", "value": 16 / t, "unit": "query-rows/s",
            "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config},
            "extrapolated_full_workload_ms": rows / (16 / t) * 1e3,
            "cpu_baseline": {"value": 16 / t, "unit": "query-rows/s", "cores": 1,
                             "kind": "oracle", "sample": "the 16 longest rows per step, one pinned host core"},
            "e2e": {"value": 16 / t, "unit": "query-rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_attn(a):
    """The reference arm of the attention workload: the oracle on 8 seeded-random rows per step."""
    import numpy as np
    from oracle import oracle as orc
    ap = synthetic.attn_config(a.config)
    B, S1 = ap.q.shape[:2]
    o = orc.default()
    rng = np.random.default_rng(5)
    R = 8
    times = []
    with one_core():
        for s in range(a.warmup + a.steps):
            part = ap.rows(rng.choice(B * S1, R, replace=False))
            t0 = time.perf_counter()
            o.sparse_attention(part)
            if s >= a.warmup:
                times.append(time.perf_counter() - t0)
    t = statistics.mean(times)
    line = {"metric": "sparse attention query-tokens/s", "value": R / t, "unit": "query-tokens/s",
            "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config,
                       "step": f"the oracle on {R} seeded-random rows"},
            "extrapolated_full_workload_ms": B * S1 / (R / t) * 1e3,
            "cpu_baseline": {"value": R / t, "unit": "query-tokens/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"{R} seeded-random rows per step, one pinned host core",
                             "host": host_cpu()},
            "e2e": {"value": R / t, "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference(a):
    """The CPU oracle as the reference arm: each step times a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if a.config == "kl_backward":
        return run_reference_kl(a)
    if a.config == "sparse_attention":
        return run_reference_attn(a)
    pb = synthetic.config(a.config)
    step_seconds = a.ref_step_seconds
    for s in range(a.warmup):
        cpu_oracle_rate(pb, step_seconds / 4, seed=1000 + s)
    rows, secs = 0, 0.0
    for s in range(a.steps):
        _r, n, t = cpu_oracle_rate(pb, step_seconds, seed=s)
        rows += n
        secs += t
    value = rows / secs
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD_TEXT.get(a.config, a.config), "name": a.config,
                       "rows_per_step": pb.rows,
                       "sampled_rows_per_step": rows / a.steps,
                       "step": "each timed step runs the oracle on a bounded seeded-random sample "
                               "of the workload's rows (ms_per_step is that sample's time)"},
            "extrapolated_full_workload_ms": pb.rows / value * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{rows} seeded-random query rows over {a.steps} steps "
                                       f"(~{step_seconds:.0f} s each), single-threaded C oracle "
                                       "pinned to one host core; per-row cost is unbiased so "
                                       "rows/s scales to the workload",
                             "host": host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_emulated_ranges(a, dev):
    """One GPU runs every key range of a key-sharded workload in turn (li_indexer per range,
    into the slots an all-gather would fill), then li_merge_topk; reports the step and the merge
    kernel's own time and bandwidth."""
    G = a.emulate_ranges
    pb_full = synthetic.config(a.config, seed=0)
    parts = [shard.key_shard(pb_full, G, r, compact=True).to(dev) for r in range(G)]
    argv = [li.make_args(p) for p in parts]
    wss = [li.empty_workspace(x, dev) for x in argv]
    shape = li.out_shape(parts[0])
    gi = torch.empty((G,) + tuple(shape), dtype=torch.int32, device=dev)
    gv = torch.empty((G,) + tuple(shape), dtype=torch.float32, device=dev)
    out_i, out_v = torch.empty(shape, dtype=torch.int32, device=dev), torch.empty(
        shape, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    m = li.LiMergeArgs()
    for l in range(G):
        m.idx_in[l], m.val_in[l] = gi[l].data_ptr(), gv[l].data_ptr()
    m.idx_out, m.val_out, m.device_status = out_i.data_ptr(), out_v.data_ptr(), status.data_ptr()
    m.rows, m.n_lists, m.topk_in, m.topk_out = parts[0].rows, G, pb_full.topk, pb_full.topk
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K = a.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]

    def step(s=None):
        for r in range(G):
            li.li_indexer(argv[r], None, wss[r], gi[r], gv[r], stream)
        if s is not None:
            ev[s][1].record(stream)
        li.li_merge_topk(m, stream)

    for _ in range(a.warmup):
        step()
    for w in wss:
        st, bits = li.li_check_status(w)
        if st != li.LI_OK:
            raise SystemExit(f"device status {st} bits {bits:#x}")
    st, bits = li.li_check_status(status)
    if st != li.LI_OK:
        raise SystemExit(f"merge status {st} bits {bits:#x}")
    torch.cuda.synchronize()
    for s in range(K):
        flush.zero_()
        ev[s][0].record(stream)
        step(s)
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    step_ms = statistics.mean(ev[s][0].elapsed_time(ev[s][2]) for s in range(K))
    merge_ms = statistics.mean(ev[s][1].elapsed_time(ev[s][2]) for s in range(K))
    # merge traffic: every input entry read once (8 B), every output slot written once (8 B)
    mbytes = G * gi[0].numel() * 8 + out_i.numel() * 8
    peaks = load_peaks()
    line = {"metric": METRIC, "value": pb_full.rows / (step_ms / 1e3), "unit": UNIT, "n_gpus": 1,
            "steps": K, "warmup": a.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config,
                       "emulated_key_ranges": G,
                       "l2": "flushed before every step by a 256 MB write outside the step's "
                             "CUDA events"},
            "merge": {"ms": merge_ms, "bytes": mbytes,
                      "achieved_gbs": mbytes / (merge_ms / 1e3) / 1e9,
                      "peak_gbs": peaks["hbm_gbs"], "lists": G},
            "gpu_launches": (sum(li.li_plan(x)["kernels"] for x in argv) + 1) * K}
    print(json.dumps(line), flush=True)
    return 0


def kl_flops(kp) -> float:
    """Algorithmic flops of one backward step: per selected (row, key), the main-attention dot
    products 2 G (Dm + Dr), the indexer score 2 H Di, its recomputation 2 H Di and the two
    gradient products 4 H Di."""
    n = int((kp.sparse_indices >= 0).sum())
    G, Dm = kp.q.shape[-2], kp.q.shape[-1]
    Dr = 0 if kp.q_rope is None else kp.q_rope.shape[-1]
    H, Di = kp.qi.shape[-2], kp.qi.shape[-1]
    return n * (2.0 * G * (Dm + Dr) + 8.0 * H * Di)


def attn_flops(ap) -> float:
    """Algorithmic flops of one attention step: per selected (row, key), the scores 2 G (Dm + Dr)
    and the value product 2 G Dm."""
    n = int(((ap.sparse_indices >= 0) & (ap.sparse_indices < ap.k.shape[1])).sum())
    G, Dm = ap.q.shape[-2], ap.q.shape[-1]
    Dr = 0 if ap.q_rope is None else ap.q_rope.shape[-1]
    return n * (2.0 * G * (Dm + Dr) + 2.0 * G * Dm), n


def run_attn(a, dev, world, rank):
    """Sparse attention over the selected keys (li_sparse_attention): one step = every row."""
    ap_cpu = synthetic.attn_config(a.config, seed=rank)
    ap = ap_cpu.to(dev)
    args = li.make_attn_args(ap)
    B, S1, G, Dm = ap.q.shape
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    out = torch.empty((B, S1, G, Dm), dtype=torch.float32, device=dev)
    smax = torch.empty((B, 1, S1, G), dtype=torch.float32, device=dev)
    ssum = torch.empty((B, 1, S1, G), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        li.li_sparse_attention(args, ws, out, smax, ssum, stream)

    for _ in range(a.warmup):
        step()
    st, bits = li.li_check_status(ws)
    if st != li.LI_OK:
        raise SystemExit(f"device status {st} bits {bits:#x}")
    K = a.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for s in range(K):
        flush.zero_()
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = sum(e0.elapsed_time(e1) for e0, e1 in ev)
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    ms = total_ms / K
    rows = B * S1
    flops, pairs = attn_flops(ap_cpu)
    achieved = flops / (ms / 1e3) / 1e12
    peaks = load_peaks()
    Dr = 0 if ap_cpu.q_rope is None else ap_cpu.q_rope.shape[-1]
    gathered = pairs * (Dm + Dr) * 2
    line = {"metric": "sparse attention query-tokens/s", "value": rows * world / (ms / 1e3),
            "unit": "query-tokens/s", "n_gpus": world, "steps": K, "warmup": a.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config,
                       "selected_pairs": pairs,
                       "l2": "flushed before every step by a 256 MB write outside the step's "
                             "CUDA events",
                       "parallelism": f"{world} independent replicas (one problem per GPU)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": kernel_traffic(a.config),
                         "kernel": "sparse_attn_kernel (gather + tcgen05 scores, softmax, "
                                   "value product)",
                         "peak_source": f"{peaks['source']} bf16 burst"},
            "gather": {"bytes": gathered, "achieved_gbs": gathered / (ms / 1e3) / 1e9,
                       "note": "selected key rows copied into shared memory once per (row, key)"},
            "clocks": clk, "gpu_launches": K}
    if rank == 0 and world == 1 and a.cpu_seconds > 0:
        from oracle import oracle as orc
        import numpy as np
        R = 16
        pick = np.random.default_rng(1).choice(rows, R, replace=False)
        part = ap_cpu.rows(pick)
        with one_core():
            t0 = time.perf_counter()
            orc.default().sparse_attention(part)
            t = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": R / t, "unit": "query-tokens/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"{R} seeded-random rows, {t:.1f} s, single-threaded C "
                                          "oracle (fp64), one pinned core",
                                "host": host_cpu()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_kl(a, dev, world, rank):
    """The indexer backward with the KL loss (li_kl_grad): one step = one call over every row."""
    kp_cpu = synthetic.kl_config(a.config, seed=rank)
    kp = kp_cpu.to(dev)
    args = li.make_kl_args(kp)
    n = li.ctypes.c_size_t(0)
    L = li.lib()
    li._check(L.li_kl_grad_workspace_size(li.ctypes.byref(args), li.ctypes.byref(n)))
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    d_qi = torch.empty(kp.qi.shape, dtype=torch.float32, device=dev)
    d_ki = torch.empty(kp.ki.shape, dtype=torch.float32, device=dev)
    d_w = torch.empty(kp.w.shape, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        li._check(L.li_kl_grad(li.ctypes.byref(args), ws.data_ptr(), n.value, loss.data_ptr(),
                               d_qi.data_ptr(), d_ki.data_ptr(), d_w.data_ptr(),
                               li._stream_handle(stream)))

    for _ in range(a.warmup):
        step()
    st, bits = li.li_check_status(ws)
    if st != li.LI_OK:
        raise SystemExit(f"device status {st} bits {bits:#x}")
    K = a.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for s in range(K):
        flush.zero_()
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = sum(e0.elapsed_time(e1) for e0, e1 in ev)
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    ms = total_ms / K
    rows = kp_cpu.w.shape[0] * kp_cpu.w.shape[1]
    flops = kl_flops(kp_cpu)
    achieved = flops / (ms / 1e3) / 1e12
    peaks = load_peaks()
    line = {"metric": "indexer backward query-rows/s", "value": rows * world / (ms / 1e3),
            "unit": "query-rows/s", "n_gpus": world, "steps": K, "warmup": a.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in, fp32 compute", "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config,
                       "l2": "flushed before every step by a 256 MB write outside the step's "
                             "CUDA events",
                       "parallelism": f"{world} independent replicas (one problem per GPU)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": kernel_traffic(a.config),
                         "kernel": "kl_tc_kernel (tcgen05: main and indexer scores, d_qi and "
                                   "d_ki products; fp32 softmax, loss and dS)",
                         "peak_source": f"{peaks['source']} bf16 burst"},
            "clocks": clk, "gpu_launches": 3 * K}
    if rank == 0 and world == 1 and a.cpu_seconds > 0:
        from oracle import oracle as orc
        R = 64
        part = synthetic.kl_rows(kp_cpu, rows - R, rows)
        with one_core():
            t0 = time.perf_counter()
            orc.default().kl_grad(part)
            t = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": R / t, "unit": "query-rows/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"the last {R} rows (the longest), {t:.1f} s, "
                                          "single-threaded C oracle (fp64), one pinned core",
                                "host": host_cpu()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="causal_prefill", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU-oracle sample budget for cpu_baseline (0 = skip)")
    ap.add_argument("--ref-step-seconds", type=float, default=3.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--emulate-ranges", type=int, default=0,
                    help="split the workload's keys into this many ranges and, on one GPU, select "
                         "in each range in turn, then merge (the N-GPU key-sharded data path "
                         "without the gather)")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.impl == "reference":
        return run_reference(a)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

    def barrier():
        if dist:
            torch.distributed.barrier()

    li.lib()
    keyshard = a.config in KEY_SHARDED
    if a.config in ("kl_backward", "sparse_attention"):
        rc = (run_kl if a.config == "kl_backward" else run_attn)(a, dev, world, rank)
        if dist:
            torch.distributed.destroy_process_group()
        return rc
    if a.emulate_ranges and (world > 1 or a.emulate_ranges > li.MERGE_MAX_LISTS):
        ap.error("--emulate-ranges takes one GPU and at most 16 ranges")
    if a.emulate_ranges:
        return run_emulated_ranges(a, dev)
    if keyshard:
        # one problem; this rank holds its key range (and only the cache blocks it uses)
        pb_full = synthetic.config(a.config, seed=0)
        pb_cpu = shard.key_shard(pb_full, world, rank, compact=True)
        rows_total = pb_full.rows
    else:
        pb_cpu = synthetic.config(a.config, seed=rank)
        rows_total = pb_cpu.rows * world
    pb = pb_cpu.to(dev)
    args = li.make_args(pb)
    plan = li.li_plan(args)
    ws = li.empty_workspace(args, dev)
    idx = torch.empty(li.out_shape(pb), dtype=torch.int32, device=dev)
    val = torch.empty(li.out_shape(pb), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    merged = keyshard and world > 1
    if merged:
        gi = torch.empty((world,) + tuple(idx.shape), dtype=torch.int32, device=dev)
        gv = torch.empty((world,) + tuple(val.shape), dtype=torch.float32, device=dev)
        out_i, out_v = torch.empty_like(idx), torch.empty_like(val)
        margs = li.LiMergeArgs()
        for l in range(world):
            margs.idx_in[l], margs.val_in[l] = gi[l].data_ptr(), gv[l].data_ptr()
        margs.idx_out, margs.val_out = out_i.data_ptr(), out_v.data_ptr()
        margs.device_status = ws.data_ptr()
        margs.rows, margs.n_lists = pb.rows, world
        margs.topk_in = margs.topk_out = pb.topk
    else:
        out_i, out_v = idx, val

    def step():
        li.li_indexer(args, None, ws, idx, val, stream)
        if merged:
            torch.distributed.all_gather(list(gi.unbind(0)), idx)
            torch.distributed.all_gather(list(gv.unbind(0)), val)
            li.li_merge_topk(margs, stream)

    for _ in range(a.warmup):
        step()
    st, bits = li.li_check_status(ws)
    if st != li.LI_OK:
        raise SystemExit(f"device status {st} bits {bits:#x}")

    K = a.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(K)]
    for e in ev:
        for x in e:
            x.record(stream)            # materialise the CUDA events before handing them out
    torch.cuda.synchronize()

    # timed steps: one event pair around each step and nothing else inside it
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for s in range(K):
        flush.zero_()                   # evict the inputs from L2 (outside the step's events)
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]

    # stage breakdown and the score kernel's duration: another K steps with the library's
    # events around each kernel (each event pair adds about 2.5 us of device time to a step)
    for s in range(K):
        flush.zero_()
        li.li_set_stage_events(ev[s][2:8])
        step()
    li.li_set_stage_events(None)
    torch.cuda.synchronize()
    meta_ms = [ev[s][2].elapsed_time(ev[s][3]) for s in range(K)]
    score_ms = [ev[s][4].elapsed_time(ev[s][5]) for s in range(K)]
    sel_ms = [ev[s][6].elapsed_time(ev[s][7]) for s in range(K)]
    total_ms = sum(step_ms)
    if dist:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / K
    value = rows_total / (ms_per_step / 1e3)

    # ---- end to end through the public API with host buffers ---------------------------------
    e2e = None
    if not a.no_e2e:
        host = {f: getattr(pb_cpu, f).pin_memory() for f in synthetic.Problem.TENSORS
                if getattr(pb_cpu, f) is not None}
        h_idx = torch.empty(out_i.shape, dtype=out_i.dtype, pin_memory=True)
        h_val = torch.empty(out_v.shape, dtype=out_v.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = h_idx.numel() * 4 + h_val.numel() * 4

        def e2e_step():
            for f, t in host.items():
                getattr(pb, f).copy_(t, non_blocking=True)
            step()
            h_idx.copy_(out_i, non_blocking=True)
            h_val.copy_(out_v, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        serial_ms = e0.elapsed_time(e1) / K
        e2e_ms, mode = serial_ms, "one stream: copy in, kernels, copy out, step after step"
        if not merged:
            # the public pipelined runner: step i's copy in, step i-1's kernels and step i-2's
            # copy out overlap (three streams, two device buffer sets)
            pipe = li.HostPipeline(pb_cpu, dev)
            outs = [(torch.empty(out_i.shape, dtype=torch.int32, pin_memory=True),
                     torch.empty(out_v.shape, dtype=torch.float32, pin_memory=True))
                    for _ in range(2)]
            pipe.run([host] * 3, [outs[i % 2] for i in range(3)])
            torch.cuda.synchronize()
            pipe.check()
            barrier()
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(pipe.s_in)
            pipe.run([host] * K, [outs[i % 2] for i in range(K)])
            p1.record(pipe.s_out)
            torch.cuda.synchronize()
            pipe.check()
            e2e_ms = p0.elapsed_time(p1) / K
            mode = ("li.HostPipeline: copy in of step i, kernels of step i-1 and copy out of "
                    "step i-2 overlap on three streams")
        if dist:
            t = torch.tensor([e2e_ms, serial_ms], device=dev)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_ms, serial_ms = float(t[0].item()), float(t[1].item())
        barrier()
        e2e = {"value": rows_total / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "mode": mode,
               "serial_ms_per_step": serial_ms}

    peaks = load_peaks()
    dtype = {torch.bfloat16: "bf16", torch.float16: "fp16",
             torch.float8_e4m3fn: "fp8_e4m3"}[pb_cpu.q.dtype]
    pairs = valid_pairs(pb_cpu)
    flops = 2.0 * pairs * pb.n_heads * pb.head_dim
    sc = statistics.mean(score_ms)
    if pb_cpu.layout_k == "PA_BSND":
        # HBM-bound: every valid key (256 B) is read once; plus q, w and the fp32 score rows
        nbytes = score_kernel_bytes(pb_cpu, pairs)
        achieved = nbytes / (sc / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": kernel_traffic(a.config),
                    "algorithmic_bytes": nbytes,
                    "kernel": "score kernel (paged key gather + contraction + epilogue)",
                    "peak_source": f"{peaks['source']} HBM copy"}
    else:
        achieved = flops / (sc / 1e3) / 1e12
        # fp8 contractions run at twice the bf16 rate (nominal dense 4.5 vs 2.25 PFLOP/s)
        peak = peaks["bf16_tflops"] * (2.0 if dtype == "fp8_e4m3" else 1.0)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": kernel_traffic(a.config),
                    "algorithmic_bytes": score_kernel_bytes(pb_cpu, pairs),
                    "kernel": "score kernel (q.k contraction + ReLU/weight/head-sum epilogue)",
                    "peak_source": f"{peaks['source']} bf16 burst"
                                   + (" (fp16 runs at the bf16 rate)" if dtype == "fp16" else "")
                                   + (" x 2, the nominal fp8/bf16 ratio" if dtype == "fp8_e4m3"
                                      else "")}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": a.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if keyshard else "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[a.config], "name": a.config,
                       "rows_per_step": rows_total, "valid_pairs_per_gpu": valid_pairs(pb_cpu),
                       "l2": "flushed before every step by a 256 MB write outside the step's "
                             "CUDA events",
                       "parallelism": (f"{world} key ranges of one problem (all-gather + merge)"
                                       if merged else
                                       f"{world} independent replicas (one problem per GPU)"),
                       "schedule": {k: plan[k] for k in ("tq", "kc", "dense", "score_tc")}},
            "roofline": roofline,
            "stages_ms": {"schedule": statistics.mean(meta_ms), "score": sc,
                          "select": statistics.mean(sel_ms)},
            "tflops_whole_step": flops / (ms_per_step / 1e3) / 1e12,
            "clocks": clk, "gpu_launches": (plan["kernels"] + (1 if merged else 0)) * K}
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and a.cpu_seconds > 0:
        line["cpu_baseline"] = cpu_baseline(pb_cpu, a.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
