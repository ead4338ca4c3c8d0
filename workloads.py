"""Seeded synthetic inputs for the sharded linear block.

This module only draws random tensors with the shapes, value distributions and
seeds of the five benchmark workloads; it contains none of the block's
arithmetic (no products, sums, activations or slicing into shards). Both the CPU
oracle (``oracle/``) and the CUDA path (``tensor_sharded_linear_columnparallel_b200``)
receive the tensors produced here, so the two sides see the same bf16 inputs.

Conventions
-----------
* Every tensor is returned on the CPU as ``torch.bfloat16``.
* Weights are returned in the math orientation of the pages, ``W[k, n]`` for
  ``Y = X W`` (rows = input features, columns = output features).
* "N(0, s)" means a normal distribution with standard deviation ``s``; the fp32
  draw is converted to bf16 by torch's round-to-nearest-even cast.
* Integer workloads draw each value uniformly from ``{-3, ..., 3}``.
* Each tensor has its own generator seeded with
  ``0x7E5A0000 + 256 * workload_id + tensor_index``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_BASE = 0x7E5A0000


def seed_for(workload_id: int, tensor_index: int) -> int:
    return SEED_BASE + 256 * workload_id + tensor_index


def gen_normal(shape, std: float, seed: int) -> torch.Tensor:
    """bf16 tensor with N(0, std) entries (fp32 draw, RNE cast to bf16)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def gen_int(shape, lo: int, hi: int, seed: int) -> torch.Tensor:
    """bf16 tensor of integers drawn uniformly from [lo, hi] inclusive."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randint(lo, hi + 1, tuple(shape), generator=g, dtype=torch.int32)
    return t.to(torch.bfloat16)


@dataclass
class Workload:
    """Shapes and tensors of one workload; ``tensors`` holds bf16 CPU tensors."""

    name: str
    wid: int
    dims: dict
    tps: tuple
    tensors: dict = field(default_factory=dict)
    description: str = ""


def int_pair(m: int = 4, k: int = 64, n: int = 256, tp: int = 2, wid: int = 1) -> Workload:
    """Two-layer column->row pair without activation, small integers in [-3, 3].

    X [m, k], W [k, n] (column-parallel), V [n, k] (row-parallel, maps n back
    to k features), plus integer biases for the column (``b_col`` [n]) and row
    (``b_row`` [k]) layers.
    """
    t = {
        "X": gen_int((m, k), -3, 3, seed_for(wid, 0)),
        "W": gen_int((k, n), -3, 3, seed_for(wid, 1)),
        "V": gen_int((n, k), -3, 3, seed_for(wid, 2)),
        "b_col": gen_int((n,), -3, 3, seed_for(wid, 3)),
        "b_row": gen_int((k,), -3, 3, seed_for(wid, 4)),
    }
    return Workload("int_pair", wid, dict(m=m, k=k, n=n), (tp,), t,
                    "column->row pair, integer inputs in [-3,3], tp=%d" % tp)


def gelu_mlp(m: int = 512, hidden: int = 1024, inter: int = 4096, wid: int = 2) -> Workload:
    """Megatron GELU MLP: fc1 hidden->inter (column), GELU, fc2 inter->hidden (row)."""
    t = {
        "X": gen_normal((m, hidden), 1.0, seed_for(wid, 0)),
        "W1": gen_normal((hidden, inter), 0.02, seed_for(wid, 1)),
        "W2": gen_normal((inter, hidden), 0.02, seed_for(wid, 2)),
    }
    return Workload("gelu_mlp", wid, dict(m=m, H=hidden, I=inter), (1, 2, 4, 8), t,
                    "GELU MLP H=%d I=%d m=%d" % (hidden, inter, m))


def gated_decode(m_max: int = 64, hidden: int = 4096, inter: int = 14336, wid: int = 3) -> Workload:
    """Llama-style gated MLP at decode sizes; callers take the first m rows of X."""
    t = {
        "X": gen_normal((m_max, hidden), 1.0, seed_for(wid, 0)),
        "Wg": gen_normal((hidden, inter), 1.0 / math.sqrt(hidden), seed_for(wid, 1)),
        "Wu": gen_normal((hidden, inter), 1.0 / math.sqrt(hidden), seed_for(wid, 2)),
        "Wd": gen_normal((inter, hidden), 1.0 / math.sqrt(inter), seed_for(wid, 3)),
    }
    return Workload("gated_decode", wid, dict(m_list=(1, 8, 32, 64), H=hidden, I=inter), (8,), t,
                    "gated MLP decode H=%d I=%d tp=8" % (hidden, inter))


def gqa_proj(m: int = 2048, hidden: int = 4096, hq: int = 32, hkv: int = 8, d: int = 128,
             wid: int = 4) -> Workload:
    """GQA attention projections: QKV column-parallel by head, o_proj row-parallel on A."""
    t = {
        "X": gen_normal((m, hidden), 1.0, seed_for(wid, 0)),
        "Wq": gen_normal((hidden, hq * d), 0.02, seed_for(wid, 1)),
        "Wk": gen_normal((hidden, hkv * d), 0.02, seed_for(wid, 2)),
        "Wv": gen_normal((hidden, hkv * d), 0.02, seed_for(wid, 3)),
        "Wo": gen_normal((hq * d, hidden), 0.02, seed_for(wid, 4)),
        "A": gen_normal((m, hq * d), 1.0, seed_for(wid, 5)),
    }
    return Workload("gqa_proj", wid, dict(m=m, H=hidden, hq=hq, hkv=hkv, d=d), (4, 8, 16), t,
                    "GQA projections H=%d hq=%d hkv=%d d=%d m=%d" % (hidden, hq, hkv, d, m))


def layer70b(m: int = 8192, hidden: int = 8192, inter: int = 28672, hq: int = 64, hkv: int = 8,
             d: int = 128, wid: int = 5) -> Workload:
    """70B-layer-shaped linears: QKV, o_proj, gate/up, down at tp=8."""
    s_h = 1.0 / math.sqrt(hidden)
    t = {
        "X": gen_normal((m, hidden), 1.0, seed_for(wid, 0)),
        "Wq": gen_normal((hidden, hq * d), s_h, seed_for(wid, 1)),
        "Wk": gen_normal((hidden, hkv * d), s_h, seed_for(wid, 2)),
        "Wv": gen_normal((hidden, hkv * d), s_h, seed_for(wid, 3)),
        "Wo": gen_normal((hq * d, hidden), 1.0 / math.sqrt(hq * d), seed_for(wid, 4)),
        "Wg": gen_normal((hidden, inter), s_h, seed_for(wid, 5)),
        "Wu": gen_normal((hidden, inter), s_h, seed_for(wid, 6)),
        "Wd": gen_normal((inter, hidden), 1.0 / math.sqrt(inter), seed_for(wid, 7)),
        "A": gen_normal((m, hq * d), 1.0, seed_for(wid, 8)),
    }
    return Workload("layer70b", wid, dict(m=m, H=hidden, I=inter, hq=hq, hkv=hkv, d=d), (8,), t,
                    "70B-layer linears H=%d I=%d hq=%d hkv=%d m=%d tp=8" % (hidden, inter, hq, hkv, m))


def lm_head(m_max: int = 64, hidden: int = 4096, vocab: int = 128256, wid: int = 6) -> Workload:
    """Greedy decoding over a vocab-parallel lm_head (the next step of the block on
    the pages' "lm_head" section): hidden states X [m, H] ~ N(0, 1) and the head
    W [H, V] ~ N(0, 1/sqrt(H)); a Llama-3-sized vocabulary, split over tp = 8."""
    t = {
        "X": gen_normal((m_max, hidden), 1.0, seed_for(wid, 0)),
        "W": gen_normal((hidden, vocab), 1.0 / math.sqrt(hidden), seed_for(wid, 1)),
    }
    return Workload("lm_head", wid, dict(m_list=(1, 8, 32, 64), H=hidden, V=vocab), (8,), t,
                    "X ~ N(0,1), W ~ N(0,1/sqrt(H)), bf16")


def gqa_attention(cols: int, nseq: int = 1, S: int = 2048, wid: int = 7) -> Workload:
    """Input of the attention on local heads: a QKV-projection output of nseq
    sequences of S tokens with `cols` columns (the caller's shard layout for
    hq = 32, hkv = 8, d = 128), entries ~ N(0, 1) so that q.k / sqrt(d) ~ N(0, 1)."""
    t = {"qkv": gen_normal((nseq * S, cols), 1.0, seed_for(wid, 0))}
    return Workload("gqa_attention", wid, dict(nseq=nseq, S=S, cols=cols), (8,), t, "qkv ~ N(0,1), bf16")


BUILDERS = {
    "int_pair": int_pair,
    "gelu_mlp": gelu_mlp,
    "gated_decode": gated_decode,
    "gqa_proj": gqa_proj,
    "layer70b": layer70b,
    "lm_head": lm_head,
    "gqa_attention": gqa_attention,
}


def make(name: str, **kw) -> Workload:
    return BUILDERS[name](**kw)
