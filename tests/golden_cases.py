"""Loads the hand-worked fixtures under tests/golden/ into indexer problems.

Each fixture is a text file: '#' comment lines (the worked derivation and its citations) followed
by a JSON body with the inputs and the expected outputs."""
import json
import math
import os

import numpy as np
import torch

from sparse_attention_token_lightning_b200.synthetic import Problem

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
D = 128


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        body = "".join(line for line in f if not line.lstrip().startswith("#"))
    return json.loads(body)


def _f(x):
    return -math.inf if x == "-inf" else float(x)


def _expected(idx, val):
    return (np.asarray(idx, dtype=np.int32),
            np.asarray([[_f(v) for v in row] for row in val], dtype=np.float32))


def _bf16(a):
    return torch.as_tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _single_key_dim(g, name):
    S1, S2, N1, topk = g["S1"], g["S2"], g["N1"], g["topk"]
    q = torch.zeros(1, S1, N1, D)
    k = torch.zeros(1, S2, 1, D)
    w = torch.zeros(1, S1, N1)
    if g.get("q_onehot"):
        for t in range(S1):
            for h in range(N1):
                q[0, t, h, h] = 1.0
        for j, row in enumerate(g["k01"]):
            k[0, j, 0, : len(row)] = torch.tensor(row, dtype=torch.float32)
    else:
        for t in range(S1):
            for h in range(N1):
                q[0, t, h, 0] = g["q0"][t][h]
        for j, v in enumerate(g["k0"]):
            k[0, j, 0, 0] = v
    w[0] = torch.tensor(g["w"], dtype=torch.float32)
    out = []
    for case, c in g["cases"].items():
        pb = Problem(name=f"{name}:{case}", q=_bf16(q), k=_bf16(k), w=_bf16(w), topk=topk,
                     batch=1, q_len=S1, k_len=S2, n_heads=N1, head_dim=D, layout_q="BSND",
                     layout_k="BSND", mask_mode=c["mask_mode"], max_seqlen_q=S1, max_seqlen_k=S2)
        out.append((pb,) + _expected(c["idx"], c["val"]))
    return out


def _paged(g, name):
    bs = g["block_size"]
    blocks = g["blocks"]
    B = len(g["seqused_k"])
    k = torch.zeros(len(blocks), bs, 1, D)
    for b, blk in enumerate(blocks):
        for s, v in enumerate(blk):
            k[b, s, 0, 0] = v
    q = torch.zeros(B, 1, 1, D)
    q[:, 0, 0, 0] = 1.0
    w = torch.ones(B, 1, 1)
    pb = Problem(name=name, q=_bf16(q), k=_bf16(k), w=_bf16(w), topk=g["topk"], batch=B,
                 q_len=1, k_len=0, n_heads=1, head_dim=D, layout_q="BSND", layout_k="PA_BSND",
                 mask_mode=3, max_seqlen_q=1, max_seqlen_k=max(g["seqused_k"]),
                 seqused_k=torch.tensor(g["seqused_k"], dtype=torch.int32),
                 block_table=torch.tensor(g["block_table"], dtype=torch.int32),
                 output_idx_offset=torch.tensor(g["output_idx_offset"], dtype=torch.int32),
                 num_blocks=len(blocks), block_size=bs)
    return [(pb,) + _expected(g["idx"], g["val"])]


def _varlen(g, name):
    cu_q, cu_k = g["cu_seqlens_q"], g["cu_seqlens_k"]
    T1, T2, B = cu_q[-1], cu_k[-1], len(cu_q) - 1
    q = torch.zeros(T1, 1, D)
    q[:, 0, 0] = 1.0
    k = torch.zeros(T2, 1, D)
    k[:, 0, 0] = torch.tensor(g["k0"], dtype=torch.float32)
    w = torch.ones(T1, 1)
    out = []
    for case, c in g["cases"].items():
        su = c["seqused_q"]
        pb = Problem(name=f"{name}:{case}", q=_bf16(q), k=_bf16(k), w=_bf16(w), topk=g["topk"],
                     batch=B, q_len=T1, k_len=T2, n_heads=1, head_dim=D, layout_q="TND",
                     layout_k="TND", mask_mode=3,
                     max_seqlen_q=max(cu_q[i + 1] - cu_q[i] for i in range(B)),
                     max_seqlen_k=max(cu_k[i + 1] - cu_k[i] for i in range(B)),
                     cu_seqlens_q=torch.tensor(cu_q, dtype=torch.int32),
                     cu_seqlens_k=torch.tensor(cu_k, dtype=torch.int32),
                     seqused_q=None if su is None else torch.tensor(su, dtype=torch.int32))
        out.append((pb,) + _expected(c["idx"], c["val"]))
    return out


FIXTURES = {
    "hand_single_head.txt": _single_key_dim,
    "hand_negative_weight.txt": _single_key_dim,
    "hand_ties.txt": _single_key_dim,
    "hand_two_heads.txt": _single_key_dim,
    "hand_paged_offset.txt": _paged,
    "hand_varlen.txt": _varlen,
}


def all_cases():
    """[(problem, expected_idx, expected_val)] over every fixture and case."""
    out = []
    for fname, fn in FIXTURES.items():
        out.extend(fn(load(fname), fname[:-4]))
    return out
