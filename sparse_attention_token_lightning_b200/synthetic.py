"""Seeded synthetic inputs for the Lightning Indexer forward pass.

This module only draws and lays out inputs; it holds none of the indexer's arithmetic, so the
CUDA path and the CPU oracle can both be fed from it. Every workload is synthetic (the pages
name no dataset): q and k are N(0, 1) and w is N(0, 1/N1), drawn in fp32 from a seeded CPU
``torch.Generator`` and rounded to bf16 (round-to-nearest-even). Shapes follow the pages:

* q: BSND (B, S1, N1, D) or TND (T1, N1, D)
* k: BSND (B, S2, 1, D), TND (T2, 1, D) or PA_BSND (num_blocks, block_size, 1, D)
* w: (B, S1, N1) or (T1, N1)

Draw order (fixed, so a seed names one input): structure first (lengths, cut points), then q,
k, w, then the paged block permutation.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional

import torch

D_DEFAULT = 128


@dataclass
class Problem:
    """One indexer invocation: inputs plus the scalar arguments of the call."""

    name: str
    q: torch.Tensor
    k: torch.Tensor
    w: torch.Tensor
    topk: int
    batch: int
    q_len: int                      # BSND: S1; TND: T1
    k_len: int                      # BSND: S2; TND: T2; PA_BSND: 0
    n_heads: int
    head_dim: int = D_DEFAULT
    layout_q: str = "BSND"
    layout_k: str = "BSND"
    mask_mode: int = 3
    max_seqlen_q: int = 0
    max_seqlen_k: int = 0
    cu_seqlens_q: Optional[torch.Tensor] = None
    cu_seqlens_k: Optional[torch.Tensor] = None
    seqused_q: Optional[torch.Tensor] = None
    seqused_k: Optional[torch.Tensor] = None
    block_table: Optional[torch.Tensor] = None
    output_idx_offset: Optional[torch.Tensor] = None
    num_blocks: int = 0
    block_size: int = 0
    cmp_ratio: int = 1                 # original tokens per key (1: keys not compressed)
    cmp_residual_k: Optional[torch.Tensor] = None   # [B] tokens past the last whole key
    q_descale: Optional[torch.Tensor] = None   # fp8 q: fp32, shaped like w
    k_descale: Optional[torch.Tensor] = None   # fp8 k: fp32, one per key row (k without D)
    meta: dict = field(default_factory=dict)

    TENSORS = ("q", "k", "w", "cu_seqlens_q", "cu_seqlens_k", "seqused_q", "seqused_k",
               "block_table", "output_idx_offset", "cmp_residual_k", "q_descale", "k_descale")

    @property
    def rows(self) -> int:
        """Number of query rows (B*S1 for BSND, T1 for TND)."""
        return self.q_len if self.layout_q == "TND" else self.batch * self.q_len

    def to(self, device) -> "Problem":
        kw = {}
        for f in self.TENSORS:
            t = getattr(self, f)
            kw[f] = None if t is None else t.to(device)
        return dataclasses.replace(self, **kw)

    def replace(self, **kw) -> "Problem":
        return dataclasses.replace(self, **kw)

    def nbytes(self) -> int:
        return sum(getattr(self, f).numel() * getattr(self, f).element_size()
                   for f in self.TENSORS if getattr(self, f) is not None)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std=1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def _integer_valued(g, shape, kind) -> torch.Tensor:
    """Values whose products and sums are exact in fp32: q,k in {-2..2}; w in {+-1/2,+-1,+-2}."""
    if kind == "qk":
        x = torch.randint(-2, 3, shape, generator=g).to(torch.float32)
    else:
        mag = torch.tensor([0.5, 1.0, 2.0])[torch.randint(0, 3, shape, generator=g)]
        sgn = torch.randint(0, 2, shape, generator=g).to(torch.float32) * 2 - 1
        x = mag * sgn
    return x.to(torch.bfloat16)


def _qkw(g, q_shape, k_shape, w_shape, n_heads, integer):
    if integer:
        return (_integer_valued(g, q_shape, "qk"), _integer_valued(g, k_shape, "qk"),
                _integer_valued(g, w_shape, "w"))
    return (_normal(g, q_shape), _normal(g, k_shape),
            _normal(g, w_shape, std=1.0 / math.sqrt(n_heads)))


def _i32(x) -> torch.Tensor:
    return torch.as_tensor(x, dtype=torch.int32)


def compressed(pb: Problem, cmp_ratio: int, residual) -> Problem:
    """The same problem with its keys read as compressed keys: each stands for cmp_ratio
    original tokens, and batch b's sequence has residual[b] (< cmp_ratio) more tokens than its
    whole keys cover (lightning_indexer, "Prototype": cmp_ratio, cmp_residual_k)."""
    return pb.replace(cmp_ratio=int(cmp_ratio),
                      cmp_residual_k=None if residual is None else _i32(residual),
                      name=f"{pb.name}_cmp{cmp_ratio}")


_DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def with_dtypes(pb: Problem, qk: str = "bf16", w: str = "bf16") -> Problem:
    """The same problem with q, k converted to qk (bf16 or fp16) and w to w (bf16, fp16 or fp32),
    each value rounded once to the new type (lightning_indexer, "Constraints": q and k share a
    type; the single-operator example uses fp16 q, k and fp32 w)."""
    return pb.replace(q=pb.q.float().to(_DT[qk]), k=pb.k.float().to(_DT[qk]),
                      w=pb.w.float().to(_DT[w]), name=f"{pb.name}_{qk}_{w}")


def quantized(pb: Problem, unit_scales: bool = False) -> Problem:
    """The same problem with q and k as fp8 e4m3 codes plus q_descale (per row and head, shaped
    like w) and k_descale (per key row): each q head row and each key row is divided by its own
    scale, max|x| / 448 (the largest e4m3 value), and rounded once to e4m3. unit_scales keeps
    every scale at 1 (integer-valued inputs are exact in e4m3)."""
    q = pb.q.float()
    k = pb.k.float()
    if unit_scales:
        qs = torch.ones(q.shape[:-1])
        ks = torch.ones(k.shape[:-1])
    else:
        qs = (q.abs().amax(dim=-1) / 448.0).clamp_min(1e-12)
        ks = (k.abs().amax(dim=-1) / 448.0).clamp_min(1e-12)
    qc = (q / qs.unsqueeze(-1)).to(torch.float8_e4m3fn)
    kc = (k / ks.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return pb.replace(q=qc, k=kc, q_descale=qs.reshape(pb.w.shape).contiguous(),
                      k_descale=ks.reshape(k.shape[:-2] if k.dim() == 4 and k.shape[-2] == 1
                                           else k.shape[:-1]).contiguous(),
                      name=f"{pb.name}_fp8")


def bsnd(B, S1, S2, N1, topk, mask_mode=3, seed=0, D=D_DEFAULT, integer=False, name="bsnd",
         seqused_q=None, seqused_k=None, output_idx_offset=None) -> Problem:
    """Dense batch: q (B,S1,N1,D), k (B,S2,1,D), w (B,S1,N1)."""
    g = _gen(seed)
    q, k, w = _qkw(g, (B, S1, N1, D), (B, S2, 1, D), (B, S1, N1), N1, integer)
    return Problem(name=name, q=q, k=k, w=w, topk=topk, batch=B, q_len=S1, k_len=S2,
                   n_heads=N1, head_dim=D, layout_q="BSND", layout_k="BSND",
                   mask_mode=mask_mode, max_seqlen_q=S1, max_seqlen_k=S2,
                   seqused_q=None if seqused_q is None else _i32(seqused_q),
                   seqused_k=None if seqused_k is None else _i32(seqused_k),
                   output_idx_offset=None if output_idx_offset is None else _i32(output_idx_offset))


def tnd(lens_q, lens_k, N1, topk, mask_mode=3, seed=0, D=D_DEFAULT, integer=False, name="tnd",
        seqused_q=None, output_idx_offset=None, layout_k="TND") -> Problem:
    """Packed varlen: q (T1,N1,D), k (T2,1,D), w (T1,N1) with cumulative cu_seqlens."""
    g = _gen(seed)
    lens_q = [int(x) for x in lens_q]
    lens_k = [int(x) for x in lens_k]
    B = len(lens_q)
    cu_q = [0]
    for x in lens_q:
        cu_q.append(cu_q[-1] + x)
    cu_k = [0]
    for x in lens_k:
        cu_k.append(cu_k[-1] + x)
    T1, T2 = cu_q[-1], cu_k[-1]
    if layout_k == "BSND":
        S2 = max(lens_k) if lens_k else 0
        q, k, w = _qkw(g, (T1, N1, D), (B, S2, 1, D), (T1, N1), N1, integer)
        return Problem(name=name, q=q, k=k, w=w, topk=topk, batch=B, q_len=T1, k_len=S2,
                       n_heads=N1, head_dim=D, layout_q="TND", layout_k="BSND",
                       mask_mode=mask_mode, max_seqlen_q=max(lens_q) if lens_q else 0,
                       max_seqlen_k=S2, cu_seqlens_q=_i32(cu_q),
                       seqused_k=_i32(lens_k),
                       seqused_q=None if seqused_q is None else _i32(seqused_q),
                       output_idx_offset=None if output_idx_offset is None
                       else _i32(output_idx_offset))
    q, k, w = _qkw(g, (T1, N1, D), (T2, 1, D), (T1, N1), N1, integer)
    return Problem(name=name, q=q, k=k, w=w, topk=topk, batch=B, q_len=T1, k_len=T2,
                   n_heads=N1, head_dim=D, layout_q="TND", layout_k="TND", mask_mode=mask_mode,
                   max_seqlen_q=max(lens_q) if lens_q else 0,
                   max_seqlen_k=max(lens_k) if lens_k else 0,
                   cu_seqlens_q=_i32(cu_q), cu_seqlens_k=_i32(cu_k),
                   seqused_q=None if seqused_q is None else _i32(seqused_q),
                   output_idx_offset=None if output_idx_offset is None
                   else _i32(output_idx_offset))


def paged(seqused_k, S1, N1, topk, block_size=64, table_width=None, mask_mode=3, seed=0,
          D=D_DEFAULT, integer=False, name="paged", layout_q="BSND", lens_q=None,
          output_idx_offset=None, spare_blocks=0) -> Problem:
    """Paged key cache PA_BSND (num_blocks, block_size, 1, D) addressed through block_table.

    Batch b owns ceil(seqused_k[b] / block_size) physical blocks, taken from a seeded random
    permutation of all blocks; unused table entries are -1. ``spare_blocks`` adds physical
    blocks no batch uses (the cache need not be dense)."""
    g = _gen(seed)
    seqused_k = [int(x) for x in seqused_k]
    B = len(seqused_k)
    nb = [max(0, -(-L // block_size)) for L in seqused_k]
    NB = sum(nb) + int(spare_blocks)
    width = table_width if table_width is not None else max(1, max(nb) if nb else 1)
    if layout_q == "TND":
        lens_q = [int(x) for x in lens_q]
        cu_q = [0]
        for x in lens_q:
            cu_q.append(cu_q[-1] + x)
        T1 = cu_q[-1]
        q_shape, w_shape = (T1, N1, D), (T1, N1)
    else:
        q_shape, w_shape = (B, S1, N1, D), (B, S1, N1)
    q, k, w = _qkw(g, q_shape, (max(NB, 1), block_size, 1, D), w_shape, N1, integer)
    perm = torch.randperm(max(NB, 1), generator=g)[:NB]
    table = torch.full((B, width), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        table[b, : nb[b]] = perm[pos: pos + nb[b]].to(torch.int32)
        pos += nb[b]
    pb = Problem(name=name, q=q, k=k, w=w, topk=topk, batch=B,
                 q_len=T1 if layout_q == "TND" else S1, k_len=0, n_heads=N1, head_dim=D,
                 layout_q=layout_q, layout_k="PA_BSND", mask_mode=mask_mode,
                 max_seqlen_q=(max(lens_q) if layout_q == "TND" else S1),
                 max_seqlen_k=max(seqused_k) if seqused_k else 0,
                 seqused_k=_i32(seqused_k), block_table=table, num_blocks=max(NB, 1),
                 block_size=block_size,
                 output_idx_offset=None if output_idx_offset is None else _i32(output_idx_offset))
    if layout_q == "TND":
        pb.cu_seqlens_q = _i32(cu_q)
    return pb


# ---------------------------------------------------------------------------------------------
# The named workloads. Sizes and distributions follow the indexer's target configurations:
# q, k ~ N(0,1), w ~ N(0, 1/N1), D = 128, one key head.
# ---------------------------------------------------------------------------------------------

def varlen_lengths(total=32768, n_seq=8, seed=0):
    """n_seq lengths >= 1 summing to total: n_seq-1 distinct cut points uniform in [1,total-1]."""
    g = _gen(seed)
    cuts = (torch.randperm(total - 1, generator=g)[: n_seq - 1] + 1).sort().values.tolist()
    pts = [0] + cuts + [total]
    return [pts[i + 1] - pts[i] for i in range(n_seq)], g


def config(name: str, seed: int = 0, integer: bool = False) -> Problem:
    if name == "tiny":
        return bsnd(1, 256, 256, 4, 32, 3, seed, integer=integer, name=name)
    if name == "causal_prefill":
        return bsnd(1, 4096, 4096, 64, 2048, 3, seed, integer=integer, name=name)
    if name == "paged_decode":
        g = _gen(seed)
        lens = torch.randint(4096, 32769, (64,), generator=g).tolist()
        return paged(lens, 1, 64, 2048, block_size=64, table_width=512, mask_mode=3,
                     seed=seed + 1, integer=integer, name=name)
    if name == "varlen":
        lens, _ = varlen_lengths(32768, 8, seed)
        return tnd(lens, lens, 64, 2048, 3, seed + 1, integer=integer, name=name)
    if name == "long_2048":
        return bsnd(1, 65536, 65536, 64, 2048, 3, seed, integer=integer, name=name)
    if name == "long_8192":
        return bsnd(1, 65536, 65536, 64, 8192, 3, seed, integer=integer, name=name)
    if name == "cmp_prefill":
        # causal prefill over 4096 original tokens whose keys are compressed 4:1 (1024 keys)
        return compressed(bsnd(1, 4096, 1024, 64, 512, 3, seed, integer=integer, name=name), 4,
                          [0])
    if name == "fp16_prefill":
        # the causal prefill in the types of the pages' single-operator example: fp16 q, k and
        # fp32 w
        return with_dtypes(bsnd(1, 4096, 4096, 64, 2048, 3, seed, integer=integer, name=name),
                           "fp16", "fp32").replace(name=name)
    if name == "fp8_prefill":
        return quantized(config("causal_prefill", seed, integer)).replace(name=name)
    if name == "fp8_decode":
        return quantized(config("paged_decode", seed, integer)).replace(name=name)
    if name == "long_row_decode":
        # one decode row over 2^20 keys (256 MB of keys); split by key range across GPUs
        return paged([1 << 20], 1, 64, 2048, block_size=64, mask_mode=3, seed=seed + 1,
                     integer=integer, name=name)
    if name == "pages_example":
        # The shape of the pages' worked example (B=2, S1=64, N1=16, topk=32) with the key
        # length it compresses to (130 // 4 = 32), taken uncompressed.
        return bsnd(2, 64, 32, 16, 32, 3, seed, integer=integer, name=name)
    raise KeyError(name)


CONFIGS = ("tiny", "causal_prefill", "paged_decode", "varlen", "long_2048", "long_8192",
           "cmp_prefill", "fp16_prefill", "long_row_decode", "fp8_prefill", "fp8_decode")


# ---- indexer backward with the KL loss ------------------------------------------------------------

@dataclass
class KLProblem:
    """Inputs of the indexer backward with the KL loss (torch_npu.npu_sparse_lightning_indexer_
    grad_kl_loss): the main attention's query and key (one key head, optional rope parts), the
    indexer's query_index, key_index and weights, the selected keys of every row (positions in
    the row's batch, -1 padded), and the main attention's softmax statistics over those keys."""

    name: str
    q: torch.Tensor                 # (B, S1, G, Dm)
    k: torch.Tensor                 # (B, S2, 1, Dm)
    q_rope: Optional[torch.Tensor]  # (B, S1, G, Dr) or None
    k_rope: Optional[torch.Tensor]  # (B, S2, 1, Dr) or None
    qi: torch.Tensor                # (B, S1, H, Di)
    ki: torch.Tensor                # (B, S2, 1, Di)
    w: torch.Tensor                 # (B, S1, H)
    sparse_indices: torch.Tensor    # (B, S1, 1, topk) int32
    key_base: torch.Tensor          # (B * S1,) int64: key row of position 0 of the row's batch
    softmax_max: torch.Tensor       # (B, 1, S1, G) fp32
    softmax_sum: torch.Tensor       # (B, 1, S1, G) fp32
    scale: float

    TENSORS = ("q", "k", "q_rope", "k_rope", "qi", "ki", "w", "sparse_indices", "key_base",
               "softmax_max", "softmax_sum")

    def to(self, device) -> "KLProblem":
        kw = {f: (None if getattr(self, f) is None else getattr(self, f).to(device))
              for f in self.TENSORS}
        return dataclasses.replace(self, **kw)

    def replace(self, **kw) -> "KLProblem":
        return dataclasses.replace(self, **kw)


def kl_bsnd(B, S, G, Dm, Dr, H, topk, seed=0, Di=D_DEFAULT, dtype=torch.bfloat16,
            name="kl") -> KLProblem:
    """A causal BSND problem (S1 = S2 = S): inputs N(0, 1) (w N(0, 1/H)) rounded to `dtype`;
    row i selects min(topk, i + 1) distinct keys of its causal window at random (in random
    order, -1 padded); softmax_max / softmax_sum are the main attention's forward statistics
    over the selected keys, per head, taken in fp64 and rounded to fp32: the max of
    scale * (q . k + q_rope . k_rope) and the sum of exp(x - max); scale = 1 / sqrt(Dm + Dr)."""
    g = _gen(seed)
    q = torch.randn(B, S, G, Dm, generator=g).to(dtype)
    k = torch.randn(B, S, 1, Dm, generator=g).to(dtype)
    q_rope = torch.randn(B, S, G, Dr, generator=g).to(dtype) if Dr else None
    k_rope = torch.randn(B, S, 1, Dr, generator=g).to(dtype) if Dr else None
    qi = torch.randn(B, S, H, Di, generator=g).to(dtype)
    ki = torch.randn(B, S, 1, Di, generator=g).to(dtype)
    w = (torch.randn(B, S, H, generator=g) / math.sqrt(H)).to(dtype)
    idx = torch.full((B, S, 1, topk), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(S):
            m = min(topk, i + 1)
            idx[b, i, 0, :m] = torch.randperm(i + 1, generator=g)[:m].to(torch.int32)
    scale = 1.0 / math.sqrt(Dm + Dr)
    smax = torch.zeros(B, 1, S, G, dtype=torch.float32)
    ssum = torch.zeros(B, 1, S, G, dtype=torch.float32)
    for b in range(B):
        for i in range(S):
            sel = idx[b, i, 0]
            sel = sel[sel >= 0].long()
            x = q[b, i].double() @ k[b, sel, 0].double().T
            if Dr:
                x = x + q_rope[b, i].double() @ k_rope[b, sel, 0].double().T
            x = x * scale
            mx = x.max(dim=1).values
            smax[b, 0, i] = mx.float()
            ssum[b, 0, i] = torch.exp(x - mx[:, None]).sum(dim=1).float()
    key_base = (torch.arange(B, dtype=torch.int64) * S).repeat_interleave(S)
    return KLProblem(name=name, q=q, k=k, q_rope=q_rope, k_rope=k_rope, qi=qi, ki=ki, w=w,
                     sparse_indices=idx, key_base=key_base, softmax_max=smax, softmax_sum=ssum,
                     scale=scale)


def kl_config(name: str, seed: int = 0) -> KLProblem:
    if name == "kl_backward":
        # causal rows over 2048 tokens, 1024 selected keys per row, a 16-head main attention of
        # 512 + 64 dims and a 64-head indexer
        return kl_bsnd(1, 2048, 16, 512, 64, 64, 1024, seed=seed, name=name)
    raise KeyError(name)


def kl_rows(kp: KLProblem, a: int, b: int) -> KLProblem:
    """Rows [a, b) of a one-batch backward problem (all keys kept)."""
    assert kp.q.shape[0] == 1
    sl = lambda t: None if t is None else t[:, a:b].contiguous()
    return kp.replace(q=sl(kp.q), q_rope=sl(kp.q_rope), qi=sl(kp.qi), w=sl(kp.w),
                      sparse_indices=sl(kp.sparse_indices), key_base=kp.key_base[a:b].contiguous(),
                      softmax_max=kp.softmax_max[:, :, a:b].contiguous(),
                      softmax_sum=kp.softmax_sum[:, :, a:b].contiguous())


# ---- sparse attention over the selected keys ------------------------------------------------------

@dataclass
class AttnProblem:
    """Inputs of the attention over each row's selected keys (values = keys): the main attention's
    query and key (one key head, optional rope parts) and the selected keys of every row
    (positions in the row's batch, -1 = none)."""

    name: str
    q: torch.Tensor                 # (B, S1, G, Dm)
    k: torch.Tensor                 # (B, S2, 1, Dm)
    q_rope: Optional[torch.Tensor]  # (B, S1, G, Dr) or None
    k_rope: Optional[torch.Tensor]  # (B, S2, 1, Dr) or None
    sparse_indices: torch.Tensor    # (B, S1, 1, topk) int32
    key_base: torch.Tensor          # (B * S1,) int64: key row of position 0 of the row's batch
    scale: float
    # paged keys: k / k_rope are caches (num_blocks, block_size, 1, D) read through block_table
    # (B, width); s2 is the logical key count per batch. None / 0 for dense keys.
    block_table: Optional[torch.Tensor] = None
    s2: int = 0

    TENSORS = ("q", "k", "q_rope", "k_rope", "sparse_indices", "key_base", "block_table")

    def to(self, device) -> "AttnProblem":
        kw = {f: (None if getattr(self, f) is None else getattr(self, f).to(device))
              for f in self.TENSORS}
        return dataclasses.replace(self, **kw)

    def replace(self, **kw) -> "AttnProblem":
        return dataclasses.replace(self, **kw)

    def rows(self, rows) -> "AttnProblem":
        """The same problem restricted to the given global query rows (all keys kept), as one
        batch of len(rows) rows; key_base keeps each row's batch."""
        B, S1 = self.q.shape[:2]
        r = torch.as_tensor(rows, dtype=torch.int64)
        take = lambda t: None if t is None else t.reshape(B * S1, *t.shape[2:])[r].unsqueeze(0)
        return self.replace(q=take(self.q), q_rope=take(self.q_rope),
                            sparse_indices=take(self.sparse_indices),
                            key_base=self.key_base[r].contiguous())


def attn_bsnd(B, S1, S2, G, Dm, Dr, topk, seed=0, causal=True, scale=None, name="attn",
              dtype=torch.bfloat16) -> AttnProblem:
    """q, k (and rope parts) N(0, 1) rounded to `dtype`. Row i of a batch selects
    min(topk, window) distinct keys of its window at random (causal: keys 0..i + S2 - S1; else
    all S2 keys), listed in random order and followed by -1 padding, as the indexer's output
    would be; scale = 1 / sqrt(Dm + Dr) unless given."""
    g = _gen(seed)
    q = torch.randn(B, S1, G, Dm, generator=g).to(dtype)
    k = torch.randn(B, S2, 1, Dm, generator=g).to(dtype)
    q_rope = torch.randn(B, S1, G, Dr, generator=g).to(dtype) if Dr else None
    k_rope = torch.randn(B, S2, 1, Dr, generator=g).to(dtype) if Dr else None
    # random keys of each row's window: the first topk of a random score over the window
    u = torch.rand(B, S1, S2, generator=g)
    if causal:
        i = torch.arange(S1).view(1, S1, 1)
        j = torch.arange(S2).view(1, 1, S2)
        u = torch.where(j <= i + (S2 - S1), u, torch.full_like(u, -1.0))
    kk = min(topk, S2)
    val, idx = torch.topk(u, kk, dim=-1)
    idx = torch.where(val >= 0, idx, torch.full_like(idx, -1)).to(torch.int32)
    sel = torch.full((B, S1, 1, topk), -1, dtype=torch.int32)
    sel[:, :, 0, :kk] = idx
    key_base = (torch.arange(B, dtype=torch.int64) * S2).repeat_interleave(S1)
    return AttnProblem(name=name, q=q, k=k, q_rope=q_rope, k_rope=k_rope, sparse_indices=sel,
                       key_base=key_base,
                       scale=float(scale) if scale is not None else 1.0 / math.sqrt(Dm + Dr))


def attn_paged(ap: AttnProblem, block_size: int, seed: int = 0, spare_blocks: int = 0) -> AttnProblem:
    """The same problem with its keys in a paged cache: batch b's ceil(S2 / block_size) blocks are
    taken from a seeded random permutation of all physical blocks (plus `spare_blocks` unused
    ones); key position v of batch b sits in block block_table[b, v // block_size] at row
    v % block_size. Positions past S2 in a batch's last block are zero."""
    g = _gen(seed)
    B, S2 = ap.k.shape[0], ap.k.shape[1]
    nb = -(-S2 // block_size)
    NB = B * nb + int(spare_blocks)
    perm = torch.randperm(NB, generator=g)[: B * nb].reshape(B, nb).to(torch.int32)

    def page(t):
        if t is None:
            return None
        D = t.shape[-1]
        cache = torch.zeros((NB, block_size, 1, D), dtype=t.dtype)
        flat = torch.zeros((B, nb * block_size, 1, D), dtype=t.dtype)
        flat[:, :S2] = t
        cache[perm.reshape(-1).long()] = flat.reshape(B * nb, block_size, 1, D)
        return cache

    return ap.replace(k=page(ap.k), k_rope=page(ap.k_rope), block_table=perm, s2=S2,
                      name=ap.name + f"_paged{block_size}")


def attn_config(name: str, seed: int = 0) -> AttnProblem:
    if name == "sparse_attention":
        # the causal prefill's selection shape (4096 rows, 2048 keys each once the window allows)
        # consumed by a 16-head main attention of 512 + 64 dims
        return attn_bsnd(1, 4096, 4096, 16, 512, 64, 2048, seed=seed, name=name)
    raise KeyError(name)
