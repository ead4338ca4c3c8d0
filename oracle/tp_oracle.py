"""Plain fp64 restatement of the column/row tensor-parallel linear block.

Test infrastructure only (see the package docstring). Every function works on
float64 numpy arrays holding the exact values of the bf16 inputs; library matmul
(`@`) and `scipy.special.erf` are the only library steps. No blocking, fusion or
reordering is done beyond what each definition states: each shard is computed
on its own slice, column results are concatenated, row partials are summed in
shard order 0..tp-1, and a row bias is added once after the sum.

Page short names used in the citations below:

* [mini-vLLM TP] = "Tensor Parallel：当一张 GPU 放不下一个大模型"
* [Megatron→vLLM] = "张量并行（Tensor Parallelism）推理部署实战：从 Megatron-LM 切分原理到 vLLM 多卡配置与性能调优"
* [TP 深入解析] = "Tensor Parallel 深入解析：多加 GPU，推理为什么可能更慢"
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "DivisibilityError", "to_f64", "linear", "split_columns", "split_rows", "split_last_dim",
    "column_parallel", "row_parallel", "gelu", "silu", "silu_mul", "bf16_round",
    "mlp_gelu", "mlp_gelu_sharded", "mlp_gated", "mlp_gated_sharded", "int_pair_sharded",
    "head_map", "qkv_shard_columns", "qkv_sharded", "qkv_unsharded", "attn_proj_sharded",
    "valid_tp_sizes", "vocab_parallel_argmax", "attention_head", "gqa_attention",
    "gqa_attention_sharded", "row_parallel_bf16_allreduce",
]


class DivisibilityError(ValueError):
    """A shard count that does not divide the split dimension (no uneven shards)."""


def to_f64(a) -> np.ndarray:
    """Exact float64 copy of a numpy array or torch tensor (bf16 values are exact in fp64)."""
    if hasattr(a, "detach"):
        import torch  # local import: torch only marshals tensors here
        return a.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Plain linear layer: Y = X W (+ b).
# [mini-vLLM TP] §"Column Parallel Linear：按输出维度切": X [batch, in], W [in, out].
# [TP 深入解析] §"两张卡如何共同算出一层": X is a row vector, rows of W are input
# features, columns are output features.
# ---------------------------------------------------------------------------
def linear(X, W, b=None) -> np.ndarray:
    X, W = to_f64(X), to_f64(W)
    Y = X @ W
    if b is not None:
        Y = Y + to_f64(b)[None, :]
    return Y


def _check_div(total: int, tp: int, what: str) -> int:
    if tp <= 0 or total % tp != 0:
        raise DivisibilityError(f"{what}={total} is not divisible by tp={tp}")
    return total // tp


def split_columns(W, tp: int):
    """W [k, n] -> [W_0, ..., W_{tp-1}], W_i = W[:, i*n/tp:(i+1)*n/tp].

    [mini-vLLM TP] §"Column Parallel Linear：按输出维度切" (W = [W0, W1], each
    [in, out/2]); [Megatron→vLLM] §1.1 (A: (k,n) -> N blocks of (k, n/N)).
    """
    W = to_f64(W)
    ns = _check_div(W.shape[1], tp, "out_features")
    return [W[:, i * ns:(i + 1) * ns] for i in range(tp)]


def split_rows(V, tp: int):
    """V [k, n] -> [V_0; ...; V_{tp-1}], V_i = V[i*k/tp:(i+1)*k/tp, :].

    [mini-vLLM TP] §"Row Parallel Linear：按输入维度切" (W = [W0; W1]);
    [Megatron→vLLM] §1.2 (A_i: (k/N, n)).
    """
    V = to_f64(V)
    ks = _check_div(V.shape[0], tp, "in_features")
    return [V[i * ks:(i + 1) * ks, :] for i in range(tp)]


def split_last_dim(X, tp: int):
    """X [m, k] -> [X_0, ..., X_{tp-1}] along the last dim ([Megatron→vLLM] §1.2, X_i: (m, k/N))."""
    X = to_f64(X)
    ks = _check_div(X.shape[1], tp, "in_features")
    return [X[:, i * ks:(i + 1) * ks] for i in range(tp)]


def column_parallel(X, W, tp: int, b=None):
    """Column-parallel linear: Y_i = X W_i (+ b_i) per shard, Y = concat(Y_i).

    X is replicated on every shard and no communication is needed
    ([mini-vLLM TP] §"Column Parallel Linear：按输出维度切"; [Megatron→vLLM] §1.1,
    whose snippet stores the shard bias with the shard: bias of size out/N).
    Returns (Y, [Y_0, ..., Y_{tp-1}]).
    """
    X = to_f64(X)
    Ws = split_columns(W, tp)
    ns = Ws[0].shape[1]
    bs = None if b is None else [to_f64(b)[i * ns:(i + 1) * ns] for i in range(tp)]
    Ys = [linear(X, Ws[i], None if bs is None else bs[i]) for i in range(tp)]
    return np.concatenate(Ys, axis=1), Ys


def row_parallel(X, V, tp: int, b=None):
    """Row-parallel linear: P_i = X_i V_i, Y = P_0 + P_1 + ... + P_{tp-1} (+ b once).

    The partial results are summed, not concatenated ([mini-vLLM TP] §"Row
    Parallel Linear：按输入维度切"; [TP 深入解析] §"两张卡如何共同算出一层": 39 + 131 = 170).
    The sum runs in shard order 0..tp-1 ("all-reduce" semantics: the sum, which
    every participant receives). [Megatron→vLLM] §1.2 declares a full-size bias
    but never applies it; here it is added exactly once, after the sum.
    Returns (Y, [P_0, ..., P_{tp-1}]).
    """
    Xs = split_last_dim(X, tp)
    Vs = split_rows(V, tp)
    Ps = [Xs[i] @ Vs[i] for i in range(tp)]
    Y = Ps[0].copy()
    for i in range(1, tp):
        Y = Y + Ps[i]
    if b is not None:
        Y = Y + to_f64(b)[None, :]
    return Y, Ps


# ---------------------------------------------------------------------------
# Activations. [Megatron→vLLM] §二 uses nn.GELU() (the exact erf form);
# [mini-vLLM TP] §"MLP 里的 tensor parallel": hidden_i = activation(gate_i) * up_i,
# with the activation taken to be SiLU.
# ---------------------------------------------------------------------------
def gelu(x) -> np.ndarray:
    """GELU(x) = x * Phi(x) = 0.5 x (1 + erf(x / sqrt(2)))."""
    x = to_f64(x)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def silu(x) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    x = to_f64(x)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def silu_mul(g, u) -> np.ndarray:
    return silu(g) * to_f64(u)


# ---------------------------------------------------------------------------
# bf16 rounding, written from the IEEE-754 definition: round to the nearest
# number with an 8-bit significand (1 implicit + 7 stored bits) and an 8-bit
# exponent (normal range 2^-126 .. 2^127, subnormal spacing 2^-133), ties to
# the even significand, overflow to infinity. Used only where the stored
# intermediate is bf16 (the activation h between the two layers).
# ---------------------------------------------------------------------------
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(x) -> np.ndarray:
    x = to_f64(x)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0.0)
    ax = np.abs(x[fin])
    _, e = np.frexp(ax)                      # 2^(e-1) <= ax < 2^e
    ulp_exp = np.maximum(e - 1 - 7, -133)    # spacing of bf16 numbers in that binade
    q = np.ldexp(ax, -ulp_exp)               # exact: a power-of-two scale
    r = np.rint(q)                           # round half to even
    y = np.ldexp(r, ulp_exp)
    y = np.where(y > _BF16_MAX, np.inf, y)
    out[fin] = np.copysign(y, x[fin])
    return out


# ---------------------------------------------------------------------------
# MLP blocks: column-parallel first layer, local activation, row-parallel second
# layer and one reduction ([Megatron→vLLM] §二 MegatronMLP: fc1 column k->4k/N,
# GELU, fc2 row 4k/N->k, one All-Reduce; Dropout(0) is the identity at inference;
# [mini-vLLM TP] §"MLP 里的 tensor parallel" for the gated form).
# round_h=True rounds the stored intermediate h to bf16 before the second layer.
# ---------------------------------------------------------------------------
def mlp_gelu(X, W1, W2, b1=None, b2=None) -> np.ndarray:
    """Unsharded GELU(X W1 + b1) W2 + b2."""
    return linear(gelu(linear(X, W1, b1)), W2, b2)


def mlp_gelu_sharded(X, W1, W2, tp: int, b1=None, b2=None, round_h: bool = False):
    """Per shard h_i = GELU(X W1_i + b1_i), P_i = h_i W2_i; Y = sum_i P_i + b2.

    Returns (Y, h) with h = concat(h_i) as the column layer writes it.
    """
    _, Ys = column_parallel(X, W1, tp, b1)
    hs = [gelu(y) for y in Ys]
    if round_h:
        hs = [bf16_round(h) for h in hs]
    h = np.concatenate(hs, axis=1)
    Y, _ = row_parallel(h, W2, tp, b2)
    return Y, h


def mlp_gated(X, Wg, Wu, Wd) -> np.ndarray:
    """Unsharded (SiLU(X Wg) * (X Wu)) Wd."""
    return linear(silu_mul(linear(X, Wg), linear(X, Wu)), Wd)


def mlp_gated_sharded(X, Wg, Wu, Wd, tp: int, round_h: bool = False):
    """gate_i = X Wg_i, up_i = X Wu_i, h_i = SiLU(gate_i) * up_i, Y = sum_i h_i Wd_i.

    Returns (Y, h) with h = concat(h_i).
    """
    _, gs = column_parallel(X, Wg, tp)
    _, us = column_parallel(X, Wu, tp)
    hs = [silu_mul(gs[i], us[i]) for i in range(tp)]
    if round_h:
        hs = [bf16_round(h) for h in hs]
    h = np.concatenate(hs, axis=1)
    Y, _ = row_parallel(h, Wd, tp)
    return Y, h


def int_pair_sharded(X, W, V, tp: int, b_col=None, b_row=None, round_h: bool = True):
    """Column layer then row layer with no activation in between.

    [TP 深入解析] §"两张卡如何共同算出一层": the column shards' outputs feed the row
    shards directly (first layer's left half -> second layer's upper half).
    With round_h the stored intermediate is rounded to bf16 as the GPU stores it.
    Returns (Y, h).
    """
    _, Ys = column_parallel(X, W, tp, b_col)
    if round_h:
        Ys = [bf16_round(y) for y in Ys]
    h = np.concatenate(Ys, axis=1)
    Y, _ = row_parallel(h, V, tp, b_row)
    return Y, h


# ---------------------------------------------------------------------------
# Attention projections split by head.
# [mini-vLLM TP] §"Attention 里的 tensor parallel": 32 heads over tp=4 gives GPU g
# the contiguous heads [8g, 8g+8); q/k/v are column-parallel by head, o_proj is
# row-parallel over the same heads.
# [TP 深入解析] §"权重变小，不代表所有显存都按比例变小": with GQA (fewer KV heads than
# query heads) query heads are sharded and KV heads may be replicated, so going
# from tp=8 to tp=16 with 32 q / 8 kv heads no longer halves the per-card KV heads.
# Reading taken where the lost table is silent: shard r holds KV heads
# [r*hkv/tp, (r+1)*hkv/tp) when tp divides hkv, else (hkv divides tp) the single
# head floor(r*hkv/tp), replicated tp/hkv times.
# [Megatron→vLLM] §6.3: tp must divide the number of attention heads.
# ---------------------------------------------------------------------------
def valid_tp_sizes(num_heads: int):
    """tp values that divide the head count ([Megatron→vLLM] §6.3)."""
    return [t for t in range(1, num_heads + 1) if num_heads % t == 0]


def head_map(hq: int, hkv: int, tp: int):
    """Returns (q_heads, kv_heads): per shard r, the list of query / KV head indices."""
    if tp <= 0 or hq % tp != 0:
        raise DivisibilityError(f"hq={hq} is not divisible by tp={tp}")
    if hkv <= 0 or hq % hkv != 0:
        raise DivisibilityError(f"hq={hq} is not a multiple of hkv={hkv}")
    qs = hq // tp
    q_heads = [list(range(r * qs, (r + 1) * qs)) for r in range(tp)]
    if hkv % tp == 0:
        ks = hkv // tp
        kv_heads = [list(range(r * ks, (r + 1) * ks)) for r in range(tp)]
    elif tp % hkv == 0:
        kv_heads = [[(r * hkv) // tp] for r in range(tp)]
    else:
        raise DivisibilityError(f"neither tp={tp} divides hkv={hkv} nor hkv divides tp")
    return q_heads, kv_heads


def qkv_shard_columns(hq: int, hkv: int, d: int, tp: int):
    """Per shard r, the columns of [Wq | Wk | Wv] that shard r computes, in its order
    [q heads of r | k heads of r | v heads of r] (each head = d consecutive columns)."""
    q_heads, kv_heads = head_map(hq, hkv, tp)
    off_k, off_v = hq * d, hq * d + hkv * d
    cols = []
    for r in range(tp):
        c = [h * d + j for h in q_heads[r] for j in range(d)]
        c += [off_k + h * d + j for h in kv_heads[r] for j in range(d)]
        c += [off_v + h * d + j for h in kv_heads[r] for j in range(d)]
        cols.append(c)
    return cols


def qkv_unsharded(X, Wq, Wk, Wv) -> np.ndarray:
    """[Q | K | V] = X [Wq | Wk | Wv]."""
    return linear(X, np.concatenate([to_f64(Wq), to_f64(Wk), to_f64(Wv)], axis=1))


def qkv_sharded(X, Wq, Wk, Wv, hq: int, hkv: int, d: int, tp: int):
    """Column-parallel QKV by head: shard r computes X Wq_r, X Wk_r, X Wv_r on its own
    (replicated KV slices are recomputed on every shard that holds them).
    Returns (concat over shards of [Q_r | K_r | V_r], list of per-shard blocks)."""
    X = to_f64(X)
    q_heads, kv_heads = head_map(hq, hkv, tp)
    Wq, Wk, Wv = to_f64(Wq), to_f64(Wk), to_f64(Wv)
    blocks = []
    for r in range(tp):
        qc = [h * d + j for h in q_heads[r] for j in range(d)]
        kc = [h * d + j for h in kv_heads[r] for j in range(d)]
        blocks.append(np.concatenate([X @ Wq[:, qc], X @ Wk[:, kc], X @ Wv[:, kc]], axis=1))
    return np.concatenate(blocks, axis=1), blocks


def attn_proj_sharded(X, A, Wq, Wk, Wv, Wo, hq: int, hkv: int, d: int, tp: int):
    """QKV column-parallel by head on X, and o_proj row-parallel on the attention
    output A [m, hq*d] (shard r owns A's columns of its query heads).
    Returns (qkv_sharded_layout, Y)."""
    qkv, _ = qkv_sharded(X, Wq, Wk, Wv, hq, hkv, d, tp)
    Y, _ = row_parallel(A, Wo, tp)
    return qkv, Y


def vocab_parallel_argmax(X, W, tp: int):
    """Greedy decoding over a vocab-parallel lm_head ([mini-vLLM TP], section
    "lm_head 怎么处理"): the lm_head W [H, V] is split by vocab (column parallel),
    shard r computes the logits of its vocab slice X W_r, finds its largest logit
    (np.argmax: the first occurrence within the slice), and the largest over the
    shards is taken in shard order, a tie keeping the earlier shard -- so ties go
    to the lowest vocab index. Returns (indices int64 [m], largest logits fp64 [m])."""
    Xf = to_f64(X)
    m = Xf.shape[0]
    best_v = np.full(m, -np.inf)
    best_i = np.zeros(m, dtype=np.int64)
    offset = 0
    for Wr in split_columns(W, tp):
        logits = Xf @ Wr
        local_i = np.argmax(logits, axis=1)
        local_v = logits[np.arange(m), local_i]
        take = local_v > best_v
        best_v = np.where(take, local_v, best_v)
        best_i = np.where(take, local_i + offset, best_i)
        offset += Wr.shape[1]
    return best_i, best_v



def attention_head(Q, K, V, causal: bool) -> np.ndarray:
    """One attention head of one sequence: O = softmax(Q K^T / sqrt(d)) V, the
    softmax taken over the keys of each query row (scaled dot-product attention;
    the pages name the operation but print no formula: the 1/sqrt(d) scale is the
    standard one). causal: query i sees keys 0..i only (decoder self-attention).
    Q [S, d], K [S, d], V [S, d] -> O [S, d], fp64."""
    Q, K, V = to_f64(Q), to_f64(K), to_f64(V)
    d = Q.shape[1]
    scores = (Q @ K.T) / math.sqrt(d)
    if causal:
        n = scores.shape[0]
        hidden = np.triu(np.ones((n, K.shape[0]), dtype=bool), k=1)
        scores = np.where(hidden, -np.inf, scores)
    mx = scores.max(axis=1, keepdims=True)
    w = np.exp(scores - mx)
    w = w / w.sum(axis=1, keepdims=True)
    return w @ V


def gqa_attention(Q, K, V, hq: int, hkv: int, d: int, nseq: int, S: int, causal: bool) -> np.ndarray:
    """Unsharded grouped-query attention: query head h reads KV head h // (hq/hkv);
    sequences (S consecutive token rows each) attend only within themselves.
    Q [nseq*S, hq*d], K and V [nseq*S, hkv*d] -> O [nseq*S, hq*d]."""
    Q, K, V = to_f64(Q), to_f64(K), to_f64(V)
    grp = hq // hkv
    out = np.zeros((nseq * S, hq * d))
    for b in range(nseq):
        rows = slice(b * S, (b + 1) * S)
        for h in range(hq):
            g = h // grp
            out[rows, h * d:(h + 1) * d] = attention_head(Q[rows, h * d:(h + 1) * d], K[rows, g * d:(g + 1) * d],
                                                          V[rows, g * d:(g + 1) * d], causal)
    return out


def gqa_attention_sharded(qkv, hq: int, hkv: int, d: int, tp: int, nseq: int, S: int, causal: bool) -> np.ndarray:
    """Attention on local heads ([mini-vLLM TP], section "Attention 里的 tensor
    parallel": each rank keeps the q/k/v of its own heads and computes their
    attention locally; the outputs stay split by head and go to the row-parallel
    o_proj). qkv is the column-parallel QKV output in the shard-major layout of
    qkv_sharded: shard r's block is [q heads of r | k heads of r | v heads of r].
    Shard r computes each of its query heads against the KV head of that head's
    group (head_map gives r's KV heads; a replicated KV head appears in every
    shard that holds it). Returns A [nseq*S, hq*d] with query head h at columns
    [h*d, (h+1)*d)."""
    qkv = to_f64(qkv)
    q_heads, kv_heads = head_map(hq, hkv, tp)
    grp = hq // hkv
    m = nseq * S
    out = np.zeros((m, hq * d))
    col = 0
    for r in range(tp):
        qs, kvs = len(q_heads[r]), len(kv_heads[r])
        block = qkv[:, col:col + (qs + 2 * kvs) * d]
        col += (qs + 2 * kvs) * d
        for j, h in enumerate(q_heads[r]):
            lk = kv_heads[r].index(h // grp)
            Qh = block[:, j * d:(j + 1) * d]
            Kh = block[:, (qs + lk) * d:(qs + lk + 1) * d]
            Vh = block[:, (qs + kvs + lk) * d:(qs + kvs + lk + 1) * d]
            for b in range(nseq):
                rows = slice(b * S, (b + 1) * S)
                out[rows, h * d:(h + 1) * d] = attention_head(Qh[rows], Kh[rows], Vh[rows], causal)
    if col != qkv.shape[1]:
        raise ValueError(f"qkv has {qkv.shape[1]} columns, the shard layout {col}")
    return out


def row_parallel_bf16_allreduce(X, V, tp: int, b=None):
    """Row-parallel linear with the partial sums exchanged in bf16, the way a
    tensor-parallel deployment all-reduces its bf16 activations ([Megatron→vLLM]
    §5.1: the all-reduce runs in NCCL on the activation tensors; the pages give no
    summation order or precision, so the plainest one is taken): every shard's
    partial P_i = X_i V_i is rounded to bf16, then the partials are added in shard
    order 0..tp-1 with a bf16 rounding after every addition, and a bias is added
    once at the end with one more rounding. Returns (Y, [bf16(P_0), ...])."""
    _, Ps = row_parallel(X, V, tp)
    Pr = [bf16_round(P) for P in Ps]
    Y = Pr[0].copy()
    for i in range(1, tp):
        Y = bf16_round(Y + Pr[i])
    if b is not None:
        Y = bf16_round(Y + to_f64(b)[None, :])
    return Y, Pr
