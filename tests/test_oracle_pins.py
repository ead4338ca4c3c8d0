"""Pins of the CPU oracle to facts outside itself.

Each test ties an oracle function to something the oracle does not compute:
values printed on the pages (fixtures under tests/golden/, each with its
citation), pure-Python brute-force loops on tiny integer inputs, textbook values
and odd-part identities of GELU/SiLU, torch's own bf16 cast, hand-picked bf16
ties, and exhaustive properties of the GQA head map. The last section plants
plausible mistakes in copies of oracle functions (on the CPU) and checks that the
pins reject them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- worked example
def _worked_example_ok(column_fn, row_fn):
    g = load("worked_example.json")
    X, W, V = np.array(g["X"], float), np.array(g["W"], float), np.array(g["V"], float)
    Y, Ys = column_fn(X, W, 2)
    ok = np.array_equal(Y, np.array(g["Y_full"], float))
    ok &= all(np.array_equal(Ys[i], np.array(g["Y_shards_tp2"][i], float)) for i in range(2))
    Z, Ps = row_fn(Y, V, 2)
    ok &= all(np.array_equal(Ps[i], np.array(g["row_partials_tp2"][i], float)) for i in range(2))
    ok &= np.array_equal(Z, np.array(g["row_sum"], float))
    return bool(ok)


def test_worked_example():
    assert _worked_example_ok(O.column_parallel, O.row_parallel)
    g = load("worked_example.json")
    assert np.array_equal(O.linear(g["X"], g["W"]), np.array(g["Y_full"], float))
    # the row partials are summed, never concatenated: concat would give two outputs
    _, Ps = O.row_parallel(np.array(g["Y_full"], float), g["V"], 2)
    assert np.concatenate(Ps, axis=1).shape == (1, 2)
    assert O.row_parallel(np.array(g["Y_full"], float), g["V"], 2)[0].shape == (1, 1)


# ---------------------------------------------------------------- brute force
def _bf_matmul(X, W):
    m, k = len(X), len(X[0])
    n = len(W[0])
    return [[sum(X[r][j] * W[j][c] for j in range(k)) for c in range(n)] for r in range(m)]


def _rand_int(rng, shape):
    return rng.integers(-3, 4, size=shape).astype(np.float64)


@pytest.mark.parametrize("m,k,n", [(1, 16, 16), (3, 16, 32), (3, 32, 16), (1, 32, 32)])
def test_column_parallel_brute_force_all_divisors(m, k, n):
    rng = np.random.default_rng(1000 + m * 100 + k + n)
    X, W, b = _rand_int(rng, (m, k)), _rand_int(rng, (k, n)), _rand_int(rng, (n,))
    full = np.array(_bf_matmul(X.tolist(), W.tolist())) + b[None, :]
    for tp in [t for t in range(1, n + 1) if n % t == 0]:
        Y, Ys = O.column_parallel(X, W, tp, b)
        assert np.array_equal(Y, full), tp
        ns = n // tp
        for i in range(tp):
            Wi = [row[i * ns:(i + 1) * ns] for row in W.tolist()]
            ref_i = np.array(_bf_matmul(X.tolist(), Wi)) + b[None, i * ns:(i + 1) * ns]
            assert np.array_equal(Ys[i], ref_i)


@pytest.mark.parametrize("m,k,n", [(1, 16, 16), (3, 16, 32), (3, 32, 16), (1, 32, 32)])
def test_row_parallel_brute_force_all_divisors(m, k, n):
    rng = np.random.default_rng(2000 + m * 100 + k + n)
    X, V, b = _rand_int(rng, (m, k)), _rand_int(rng, (k, n)), _rand_int(rng, (n,))
    full = np.array(_bf_matmul(X.tolist(), V.tolist())) + b[None, :]
    for tp in [t for t in range(1, k + 1) if k % t == 0]:
        Y, Ps = O.row_parallel(X, V, tp, b)
        assert np.array_equal(Y, full), tp
        ks = k // tp
        for i in range(tp):
            Xi = [row[i * ks:(i + 1) * ks] for row in X.tolist()]
            Vi = V.tolist()[i * ks:(i + 1) * ks]
            assert np.array_equal(Ps[i], np.array(_bf_matmul(Xi, Vi)))


def test_tp1_is_plain_gemm():
    rng = np.random.default_rng(7)
    X, W = _rand_int(rng, (3, 16)), _rand_int(rng, (16, 32))
    ref = np.array(_bf_matmul(X.tolist(), W.tolist()))
    assert np.array_equal(O.column_parallel(X, W, 1)[0], ref)
    assert np.array_equal(O.row_parallel(X, W, 1)[0], ref)


@pytest.mark.parametrize("tp", [1, 2, 4, 8, 16])
def test_concat_and_sum_invariants(tp):
    """[mini-vLLM TP] validation recipe: column concat == full, row sum == full."""
    rng = np.random.default_rng(tp)
    X, W = _rand_int(rng, (5, 64)), _rand_int(rng, (64, 256))
    assert np.array_equal(O.column_parallel(X, W, tp)[0], X @ W)
    assert np.array_equal(O.row_parallel(X, W, tp)[0], X @ W)
    Xf, Wf = rng.standard_normal((5, 64)), rng.standard_normal((64, 256))
    assert np.allclose(O.column_parallel(Xf, Wf, tp)[0], Xf @ Wf, rtol=0, atol=1e-12)
    assert np.allclose(O.row_parallel(Xf, Wf, tp)[0], Xf @ Wf, rtol=0, atol=1e-12)


def test_divisibility_errors():
    W = np.zeros((8, 12))
    with pytest.raises(O.DivisibilityError):
        O.column_parallel(np.zeros((1, 8)), W, 5)
    with pytest.raises(O.DivisibilityError):
        O.row_parallel(np.zeros((1, 8)), W, 3)
    with pytest.raises(O.DivisibilityError):
        O.head_map(32, 8, 3)


def test_valid_tp_sizes_fixture():
    for case in load("valid_tp_sizes.json")["cases"]:
        assert O.valid_tp_sizes(case["num_heads"]) == case["valid"]
        for t in case.get("invalid", []):
            with pytest.raises(O.DivisibilityError):
                O.head_map(case["num_heads"], case["num_heads"], t)


# ---------------------------------------------------------------- activations
def test_gelu_textbook_values_and_identities():
    # GELU(x) = x * Phi(x); Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    assert abs(O.gelu(np.array([-1.0]))[0] + 0.15865525393145707) < 1e-15
    assert abs(O.gelu(np.array([2.0]))[0] - 2 * 0.9772498680518208) < 1e-15
    x = np.random.default_rng(3).standard_normal(1000) * 4
    assert np.allclose(O.gelu(x) - O.gelu(-x), x, rtol=0, atol=1e-13)   # odd part is x/2
    assert abs(O.gelu(np.array([12.0]))[0] - 12.0) < 1e-12
    assert abs(O.gelu(np.array([-12.0]))[0]) < 1e-12
    ref = torch.nn.functional.gelu(torch.tensor(x, dtype=torch.float64)).numpy()
    assert np.allclose(O.gelu(x), ref, rtol=1e-14, atol=1e-15)
    ref_py = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in x])
    assert np.allclose(O.gelu(x), ref_py, rtol=1e-14, atol=1e-15)


def test_silu_textbook_values_and_identities():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([1.0]))[0] - 0.7310585786300049) < 1e-15   # sigmoid(1)
    x = np.random.default_rng(4).standard_normal(1000) * 6
    assert np.allclose(O.silu(x) - O.silu(-x), x, rtol=0, atol=1e-12)
    ref = torch.nn.functional.silu(torch.tensor(x, dtype=torch.float64)).numpy()
    assert np.allclose(O.silu(x), ref, rtol=1e-14, atol=1e-15)
    assert O.silu(np.array([-800.0]))[0] == 0.0 or abs(O.silu(np.array([-800.0]))[0]) < 1e-300
    g, u = np.array([1.0, -2.0]), np.array([3.0, 0.5])
    assert np.allclose(O.silu_mul(g, u), [3 * 0.7310585786300049, 0.5 * -2 / (1 + math.e ** 2)])


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_hand_picked():
    e = 2.0 ** -8
    cases = {
        1.0 + e: 1.0,                          # tie -> even (1.0)
        1.0 + 3 * e: 1.0 + 2.0 ** -6,          # tie -> even (upper)
        1.0 + e + 2.0 ** -20: 1.0 + 2.0 ** -7,  # just above the tie
        -(1.0 + e): -1.0,
        255.0: 255.0, 256.0: 256.0, 257.0: 256.0, 258.0: 258.0, 259.0: 260.0, 577.0: 576.0,
        2.0 ** -133: 2.0 ** -133,               # smallest subnormal
        2.0 ** -134: 0.0,                      # tie between 0 and 2^-133 -> 0
        3 * 2.0 ** -134: 2.0 ** -132,           # tie between 1 and 2 subnormal steps -> 2
        (2 - 2.0 ** -7) * 2.0 ** 127: (2 - 2.0 ** -7) * 2.0 ** 127,
        (2 - 2.0 ** -8) * 2.0 ** 127: math.inf,  # tie at the top -> overflow
        0.0: 0.0,
    }
    xs = np.array(list(cases.keys()))
    want = np.array(list(cases.values()))
    got = O.bf16_round(xs)
    assert np.array_equal(got, want), list(zip(xs, got, want))


def test_bf16_matches_torch_cast_on_fp32_values():
    rng = np.random.default_rng(5)
    a = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 100,
        (rng.integers(0, 2 ** 31, 20000, dtype=np.int64).astype(np.uint32)).view(np.float32),
    ])
    a = a[np.isfinite(a)]
    ref = torch.tensor(a).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(a.astype(np.float64))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- GQA head map
def test_head_map_page_fixture():
    g = load("head_split_32x4.json")
    q, _ = O.head_map(g["num_heads"], g["num_heads"], g["tp"])
    assert [[h[0], h[-1]] for h in q] == g["heads_per_gpu"]


def test_head_map_kv_replication_fixture():
    g = load("gqa_kv_per_card.json")
    for c in g["per_card"]:
        q, kv = O.head_map(g["hq"], g["hkv"], c["tp"])
        assert all(len(x) == c["q_heads"] for x in q)
        assert all(len(x) == c["kv_heads"] for x in kv)
    _, kv16 = O.head_map(32, 8, 16)
    for j in range(8):
        assert [r for r in range(16) if j in kv16[r]] == [2 * j, 2 * j + 1]


def test_head_map_exhaustive_properties():
    n = 0
    for hq in range(1, 65):
        for hkv in [h for h in range(1, hq + 1) if hq % h == 0]:
            group = hq // hkv
            for tp in [t for t in range(1, hq + 1) if hq % t == 0]:
                if not (hkv % tp == 0 or tp % hkv == 0):
                    with pytest.raises(O.DivisibilityError):
                        O.head_map(hq, hkv, tp)
                    continue
                q, kv = O.head_map(hq, hkv, tp)
                n += 1
                # query heads: a contiguous, disjoint cover of [0, hq)
                assert list(itertools.chain(*q)) == list(range(hq))
                assert all(len(x) == hq // tp for x in q)
                # each shard holds the KV head of every query head it owns
                for r in range(tp):
                    for h in q[r]:
                        assert h // group in kv[r]
                    assert len(kv[r]) == max(1, hkv // tp)
                # every KV head is held, max(1, tp/hkv) times
                counts = [sum(j in kv[r] for r in range(tp)) for j in range(hkv)]
                assert counts == [max(1, tp // hkv)] * hkv
    assert n > 200


def test_qkv_sharded_brute_force():
    rng = np.random.default_rng(11)
    hq, hkv, d, H, m = 4, 2, 2, 8, 3
    X = _rand_int(rng, (m, H))
    Wq, Wk, Wv = _rand_int(rng, (H, hq * d)), _rand_int(rng, (H, hkv * d)), _rand_int(rng, (H, hkv * d))
    Q = np.array(_bf_matmul(X.tolist(), Wq.tolist()))
    K = np.array(_bf_matmul(X.tolist(), Wk.tolist()))
    Vv = np.array(_bf_matmul(X.tolist(), Wv.tolist()))
    for tp in (1, 2, 4):
        qkv, blocks = O.qkv_sharded(X, Wq, Wk, Wv, hq, hkv, d, tp)
        qs = hq // tp
        for r in range(tp):
            kvh = [(r * hkv) // tp] if tp > hkv else list(range(r * hkv // tp, (r + 1) * hkv // tp))
            want = np.concatenate(
                [Q[:, r * qs * d:(r + 1) * qs * d]]
                + [K[:, h * d:(h + 1) * d] for h in kvh] + [Vv[:, h * d:(h + 1) * d] for h in kvh], axis=1)
            assert np.array_equal(blocks[r], want)
        full = O.qkv_unsharded(X, Wq, Wk, Wv)
        cols = O.qkv_shard_columns(hq, hkv, d, tp)
        assert np.array_equal(qkv, full[:, list(itertools.chain(*cols))])


# ---------------------------------------------------------------- MLP blocks
def _bf_gelu_mlp(X, W1, W2):
    h = [[0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in row] for row in _bf_matmul(X, W1)]
    return np.array(_bf_matmul(h, W2))


def _bf_gated_mlp(X, Wg, Wu, Wd):
    g, u = _bf_matmul(X, Wg), _bf_matmul(X, Wu)
    h = [[gv / (1 + math.exp(-gv)) * uv for gv, uv in zip(gr, ur)] for gr, ur in zip(g, u)]
    return np.array(_bf_matmul(h, Wd))


@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_mlp_blocks_brute_force(tp):
    rng = np.random.default_rng(20 + tp)
    X = rng.standard_normal((3, 16))
    W1, W2 = rng.standard_normal((16, 32)) * 0.3, rng.standard_normal((32, 16)) * 0.3
    Y, _ = O.mlp_gelu_sharded(X, W1, W2, tp)
    assert np.allclose(Y, _bf_gelu_mlp(X.tolist(), W1.tolist(), W2.tolist()), rtol=1e-12, atol=1e-12)
    Wg, Wu, Wd = (rng.standard_normal(s) * 0.3 for s in ((16, 32), (16, 32), (32, 16)))
    Y, _ = O.mlp_gated_sharded(X, Wg, Wu, Wd, tp)
    assert np.allclose(Y, _bf_gated_mlp(X.tolist(), Wg.tolist(), Wu.tolist(), Wd.tolist()),
                       rtol=1e-12, atol=1e-12)
    assert np.allclose(O.mlp_gated(X, Wg, Wu, Wd), Y, rtol=1e-12, atol=1e-12)


def test_int_pair_contract_mode_rounds_only_h():
    # intermediate values above 256 are not all bf16 integers: 257 -> 256, 259 -> 260
    X = np.array([[1.0]])
    W = np.array([[257.0, 259.0]])
    V = np.array([[1.0], [1.0]])
    Y, h = O.int_pair_sharded(X, W, V, 2, round_h=True)
    assert np.array_equal(h, [[256.0, 260.0]]) and Y[0, 0] == 516.0
    Y, h = O.int_pair_sharded(X, W, V, 2, round_h=False)
    assert np.array_equal(h, [[257.0, 259.0]]) and Y[0, 0] == 516.0


# ---------------------------------------------------------------- planted mistakes
def _mut_row_concat(X, V, tp, b=None):
    Y, Ps = O.row_parallel(X, V, tp, b)
    return np.concatenate(Ps, axis=1)[:, :Y.shape[1]], Ps


def _mut_row_drop_last(X, V, tp, b=None):
    Y, Ps = O.row_parallel(X, V, tp, b)
    return Y - Ps[-1], Ps


def _mut_row_swapped_slices(X, V, tp, b=None):
    Xs, Vs = O.split_last_dim(X, tp), O.split_rows(V, tp)
    Ps = [Xs[i] @ Vs[tp - 1 - i] for i in range(tp)]
    return sum(Ps), Ps


def _mut_col_transposed(X, W, tp, b=None):
    Wt = O.to_f64(W).T.reshape(O.to_f64(W).shape)
    return O.column_parallel(X, Wt, tp, b)


def _mut_col_bias_twice(X, W, tp, b=None):
    Y, Ys = O.column_parallel(X, W, tp, b)
    return Y + 1.0, [y + 1.0 for y in Ys]


@pytest.mark.parametrize("mut", [_mut_row_concat, _mut_row_drop_last, _mut_row_swapped_slices])
def test_planted_row_mistakes_fail_pins(mut):
    assert not _worked_example_ok(O.column_parallel, mut)


@pytest.mark.parametrize("mut", [_mut_col_transposed, _mut_col_bias_twice])
def test_planted_column_mistakes_fail_pins(mut):
    assert not _worked_example_ok(mut, O.row_parallel)


def test_planted_activation_mistakes_fail_pins():
    wrong_gelu = lambda x: 0.5 * x * (1 + np.tanh(x))            # noqa: E731  wrong inner scale
    wrong_silu = lambda x: x / (1 + np.exp(x))                   # noqa: E731  sign flip
    assert abs(wrong_gelu(1.0) - 0.8413447460685429) > 1e-3
    assert abs(wrong_silu(1.0) - 0.7310585786300049) > 1e-3


# ============================================================ vocab-parallel greedy argmax
def _argmax_brute(X, W, tp):
    """Python loops: per shard, the first largest logit of its vocab slice; then
    shards in order, a later shard replacing the best only when strictly larger."""
    X, W = O.to_f64(X), O.to_f64(W)
    m, k = X.shape
    V = W.shape[1]
    vs = V // tp
    idx, val = [], []
    for r in range(m):
        best_v, best_i = -math.inf, -1
        for s in range(tp):
            lv, li = -math.inf, -1
            for c in range(s * vs, (s + 1) * vs):
                logit = sum(X[r, j] * W[j, c] for j in range(k))
                if logit > lv:
                    lv, li = logit, c
            if lv > best_v:
                best_v, best_i = lv, li
        idx.append(best_i)
        val.append(best_v)
    return np.array(idx), np.array(val)


def test_argmax_worked_example_every_tp():
    """The worked example's logits [11, 14, 17, 20]: the greedy token is vocab 3
    (logit 20) whatever the split."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    X, W = np.array(g["X"], float), np.array(g["W"], float)
    for tp in (1, 2, 4):
        i, v = O.vocab_parallel_argmax(X, W, tp)
        assert i.tolist() == [3] and v.tolist() == [20.0]


@pytest.mark.parametrize("m,k,V", [(3, 5, 12), (2, 4, 24)])
def test_argmax_brute_force_all_divisors(m, k, V):
    rng = np.random.default_rng(7 + V)
    X = rng.integers(-3, 4, size=(m, k)).astype(float)
    W = rng.integers(-3, 4, size=(k, V)).astype(float)   # small integers: many exact ties
    for tp in [d for d in range(1, V + 1) if V % d == 0]:
        i, v = O.vocab_parallel_argmax(X, W, tp)
        bi, bv = _argmax_brute(X, W, tp)
        assert np.array_equal(i, bi) and np.array_equal(v, bv)


def test_argmax_equals_unsharded_first_argmax():
    """Shard-local argmax then the max over shards (ties to the earlier shard) is
    the first argmax of the full logits, for every divisor tp."""
    rng = np.random.default_rng(11)
    X = rng.integers(-2, 3, size=(64, 6)).astype(float)
    W = rng.integers(-2, 3, size=(6, 96)).astype(float)
    full = X @ W
    for tp in (1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 48, 96):
        i, v = O.vocab_parallel_argmax(X, W, tp)
        assert np.array_equal(i, np.argmax(full, axis=1))
        assert np.array_equal(v, full.max(axis=1))


def test_argmax_ties_go_to_the_lowest_index():
    X = np.array([[1.0]])
    W = np.array([[5.0, 1.0, 5.0, 5.0, 2.0, 5.0]])   # max 5 at 0, 2, 3, 5
    for tp in (1, 2, 3, 6):
        assert O.vocab_parallel_argmax(X, W, tp)[0].tolist() == [0]
    W = np.array([[1.0, 4.0, 2.0, 4.0]])             # equal maxima in shard 0 and shard 1 at tp=2
    assert O.vocab_parallel_argmax(X, W, 2)[0].tolist() == [1]


def _mut_argmax_no_offset(X, W, tp):
    """Planted mistake: shard-local index returned without the shard's vocab offset."""
    Xf = O.to_f64(X)
    best_v = np.full(Xf.shape[0], -np.inf)
    best_i = np.zeros(Xf.shape[0], dtype=np.int64)
    for Wr in O.split_columns(W, tp):
        L = Xf @ Wr
        li = np.argmax(L, axis=1)
        lv = L[np.arange(len(li)), li]
        take = lv > best_v
        best_v, best_i = np.where(take, lv, best_v), np.where(take, li, best_i)
    return best_i, best_v


def _mut_argmax_last_shard_wins_ties(X, W, tp):
    """Planted mistake: a later shard replaces the best on equal logits."""
    Xf = O.to_f64(X)
    best_v = np.full(Xf.shape[0], -np.inf)
    best_i = np.zeros(Xf.shape[0], dtype=np.int64)
    off = 0
    for Wr in O.split_columns(W, tp):
        L = Xf @ Wr
        li = np.argmax(L, axis=1)
        lv = L[np.arange(len(li)), li]
        take = lv >= best_v
        best_v, best_i = np.where(take, lv, best_v), np.where(take, li + off, best_i)
        off += Wr.shape[1]
    return best_i, best_v


@pytest.mark.parametrize("mut", [_mut_argmax_no_offset, _mut_argmax_last_shard_wins_ties])
def test_planted_argmax_mistakes_fail_pins(mut):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    X, W = np.array(g["X"], float), np.array(g["W"], float)
    ok_example = all(mut(X, W, tp)[0].tolist() == [3] for tp in (1, 2, 4))
    Xt, Wt = np.array([[1.0]]), np.array([[1.0, 4.0, 2.0, 4.0]])
    ok_ties = mut(Xt, Wt, 2)[0].tolist() == [1]
    assert not (ok_example and ok_ties)


# ============================================================ local per-shard GQA attention
def _sdpa(Q, K, V, causal, enable_gqa=False):
    """torch's scaled_dot_product_attention in fp64 on [heads, S, d] arrays."""
    q, k, v = (torch.tensor(np.asarray(a, dtype=np.float64))[None] for a in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal,
                                                            enable_gqa=enable_gqa)[0].numpy()


def _head_pins_hold(head_fn):
    """Closed forms and library agreement that any correct single-head attention meets."""
    rng = np.random.default_rng(11)
    S, d = 9, 8
    V = rng.standard_normal((S, d))
    K = rng.standard_normal((S, d))
    ok = True
    # Q = 0: uniform weights -> the mean of the visible values (prefix means when causal)
    Z = np.zeros((S, d))
    ok &= np.allclose(head_fn(Z, K, V, False), np.tile(V.mean(axis=0), (S, 1)), atol=1e-12)
    prefix = np.cumsum(V, axis=0) / np.arange(1, S + 1)[:, None]
    ok &= np.allclose(head_fn(Z, K, V, True), prefix, atol=1e-12)
    # one key: the output is that key's value
    ok &= np.allclose(head_fn(rng.standard_normal((1, d)), K[:1], V[:1], True), V[:1], atol=1e-12)
    # a dominant score selects one value row: K = I, Q = 60 * permutation -> scores 30 * delta
    perm = np.array([2, 0, 3, 1])
    Kd = np.eye(4)
    Qd = 60.0 * np.eye(4)[perm]
    Vd = rng.standard_normal((4, 4))
    ok &= np.allclose(head_fn(Qd, Kd, Vd, False), Vd[perm], atol=1e-9)
    # the library routine on random inputs, both masks
    Q = rng.standard_normal((S, d))
    for c in (False, True):
        ok &= np.allclose(head_fn(Q, K, V, c), _sdpa(Q[None], K[None], V[None], c)[0], atol=1e-12)
    return bool(ok)


def test_attention_head_pins():
    assert _head_pins_hold(O.attention_head)


def _gqa_pins_hold(gqa_fn):
    """GQA grouping against torch's own grouped attention, and sequence independence."""
    rng = np.random.default_rng(12)
    nseq, S, d = 2, 6, 8
    ok = True
    for hq, hkv in ((4, 4), (4, 2), (6, 1), (8, 2)):
        Q = rng.standard_normal((nseq * S, hq * d))
        K = rng.standard_normal((nseq * S, hkv * d))
        V = rng.standard_normal((nseq * S, hkv * d))
        for c in (False, True):
            got = gqa_fn(Q, K, V, hq, hkv, d, nseq, S, c)
            for b in range(nseq):
                rows = slice(b * S, (b + 1) * S)
                q = Q[rows].reshape(S, hq, d).transpose(1, 0, 2)
                k = K[rows].reshape(S, hkv, d).transpose(1, 0, 2)
                v = V[rows].reshape(S, hkv, d).transpose(1, 0, 2)
                ref = _sdpa(q, k, v, c, enable_gqa=True).transpose(1, 0, 2).reshape(S, hq * d)
                ok &= np.allclose(got[rows], ref, atol=1e-12)
    # changing sequence 0 leaves sequence 1 unchanged
    Q = rng.standard_normal((nseq * S, 2 * d))
    K = rng.standard_normal((nseq * S, d))
    V = rng.standard_normal((nseq * S, d))
    a = gqa_fn(Q, K, V, 2, 1, d, nseq, S, True)
    V2 = V.copy()
    V2[:S] += 5.0
    b = gqa_fn(Q, K, V2, 2, 1, d, nseq, S, True)
    ok &= np.array_equal(a[S:], b[S:]) and not np.allclose(a[:S], b[:S])
    return bool(ok)


def test_gqa_attention_pins():
    assert _gqa_pins_hold(O.gqa_attention)


def _shard_layout(Q, K, V, hq, hkv, d, tp):
    """[Q | K | V] gathered into the shard-major QKV layout by the (separately
    pinned) column lists of qkv_shard_columns."""
    full = np.concatenate([Q, K, V], axis=1)
    return np.concatenate([full[:, c] for c in O.qkv_shard_columns(hq, hkv, d, tp)], axis=1)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 2), (8, 1), (6, 3), (32, 8)])
def test_gqa_attention_sharded_equals_unsharded_every_tp(hq, hkv):
    """Attention on local heads gives the unsharded result for every valid tp, the
    page's 32 heads over tp = 4 included, with KV heads replicated when tp > hkv."""
    rng = np.random.default_rng(13)
    nseq, S, d = 2, 5, 8
    Q = rng.standard_normal((nseq * S, hq * d))
    K = rng.standard_normal((nseq * S, hkv * d))
    V = rng.standard_normal((nseq * S, hkv * d))
    ref = O.gqa_attention(Q, K, V, hq, hkv, d, nseq, S, True)
    n = 0
    for tp in O.valid_tp_sizes(hq):
        if hkv % tp and tp % hkv:
            continue
        got = O.gqa_attention_sharded(_shard_layout(Q, K, V, hq, hkv, d, tp), hq, hkv, d, tp, nseq, S, True)
        assert np.allclose(got, ref, atol=1e-12), tp
        n += 1
    assert n >= 2


def _mut_head_no_scale(Q, K, V, causal):
    """Planted mistake: the 1/sqrt(d) scale left out."""
    return O.attention_head(np.asarray(Q) * math.sqrt(np.asarray(Q).shape[1]), K, V, causal)


def _mut_head_mask_diagonal(Q, K, V, causal):
    """Planted mistake: the causal mask also hides a query's own key (first row sees
    nothing, so it is given the first value row)."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    if not causal:
        return O.attention_head(Q, K, V, False)
    out = np.zeros_like(Q @ np.zeros((Q.shape[1], V.shape[1])))
    out[0] = V[0]
    for i in range(1, Q.shape[0]):
        out[i] = O.attention_head(Q[i:i + 1], K[:i], V[:i], False)[0]
    return out


def _mut_gqa_modulo_map(Q, K, V, hq, hkv, d, nseq, S, causal):
    """Planted mistake: query head h reads KV head h % hkv instead of h // (hq/hkv)."""
    out = np.zeros((nseq * S, hq * d))
    for b in range(nseq):
        r = slice(b * S, (b + 1) * S)
        for h in range(hq):
            g = h % hkv
            out[r, h * d:(h + 1) * d] = O.attention_head(Q[r, h * d:(h + 1) * d], K[r, g * d:(g + 1) * d],
                                                         V[r, g * d:(g + 1) * d], causal)
    return out


def _mut_gqa_sequences_joined(Q, K, V, hq, hkv, d, nseq, S, causal):
    """Planted mistake: all token rows treated as one sequence."""
    return O.gqa_attention(Q, K, V, hq, hkv, d, 1, nseq * S, causal)


@pytest.mark.parametrize("mut", [_mut_head_no_scale, _mut_head_mask_diagonal])
def test_planted_attention_head_mistakes_fail_pins(mut):
    assert not _head_pins_hold(mut)


@pytest.mark.parametrize("mut", [_mut_gqa_modulo_map, _mut_gqa_sequences_joined])
def test_planted_gqa_mistakes_fail_pins(mut):
    assert not _gqa_pins_hold(mut)


# ============================================================ bf16 partials, summed in bf16
def test_bf16_allreduce_worked_example():
    """The page's worked example: partials 39 and 131 are exact in bf16 and so is
    their sum 170 (8 significant bits)."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    H, V = np.array(g["Y_full"], float), np.array(g["V"], float)   # the example's row layer
    Y, Pr = O.row_parallel_bf16_allreduce(H, V, 2)
    assert [P.tolist() for P in Pr] == g["row_partials_tp2"]
    assert Y.tolist() == g["row_sum"]


def test_bf16_allreduce_rounds_after_every_addition():
    """Hand-computed: partials 256, 1, 1 (each exact in bf16). In bf16, 256 + 1 = 257
    lies halfway between 256 and 258 and rounds to even (256), twice; an fp32 or fp64
    sum gives 258. In the other shard order (1, 1, 256) the sum is 2 + 256 = 258."""
    X = np.array([[1.0, 1.0, 1.0]])
    for V, want in ((np.array([[256.0], [1.0], [1.0]]), 256.0), (np.array([[1.0], [1.0], [256.0]]), 258.0)):
        Y, _ = O.row_parallel_bf16_allreduce(X, V, 3)
        assert Y[0, 0] == want
        assert O.row_parallel(X, V, 3)[0][0, 0] == 258.0


def test_bf16_allreduce_rounds_each_partial_first():
    """Hand-computed: partials 1 + 2^-8 and 2^-8. The first is a tie between 1 and
    1 + 2^-7 in bf16 and rounds to 1 (even); 1 + 2^-8 is again a tie and gives 1.
    Summing the unrounded partials would give 1 + 2^-7, a bf16 value."""
    X = np.array([[1.0 + 2.0 ** -8, 2.0 ** -8]])
    V = np.array([[1.0], [1.0]])
    Y, Pr = O.row_parallel_bf16_allreduce(X, V, 2)
    assert Pr[0][0, 0] == 1.0 and Pr[1][0, 0] == 2.0 ** -8
    assert Y[0, 0] == 1.0
    assert O.bf16_round(O.row_parallel(X, V, 2)[0])[0, 0] == 1.0 + 2.0 ** -7


def test_bf16_allreduce_is_the_exact_sum_when_nothing_rounds():
    """Small integers: every partial and every running sum is below 256 in magnitude,
    hence exact in bf16; the result equals the exact row-parallel sum for every tp."""
    rng = np.random.default_rng(21)
    X = rng.integers(-2, 3, size=(6, 32)).astype(float)
    V = rng.integers(-2, 3, size=(32, 16)).astype(float)
    for tp in (1, 2, 4, 8, 16, 32):
        Y, _ = O.row_parallel_bf16_allreduce(X, V, tp)
        assert np.array_equal(Y, X @ V)


def _mut_bf16_single_rounding(X, V, tp, b=None):
    """Planted mistake: partials summed in full precision, rounded once."""
    Y, Ps = O.row_parallel(X, V, tp, b)
    return O.bf16_round(Y), Ps


def _mut_bf16_reverse_order(X, V, tp, b=None):
    """Planted mistake: partials added from the last shard to the first."""
    _, Ps = O.row_parallel(X, V, tp)
    Pr = [O.bf16_round(P) for P in Ps]
    Y = Pr[-1].copy()
    for P in reversed(Pr[:-1]):
        Y = O.bf16_round(Y + P)
    return Y, Pr


def _mut_bf16_partials_unrounded(X, V, tp, b=None):
    """Planted mistake: partials added in bf16 but not rounded before the exchange."""
    _, Ps = O.row_parallel(X, V, tp)
    Y = Ps[0].copy()
    for P in Ps[1:]:
        Y = O.bf16_round(Y + P)
    return Y, Ps


@pytest.mark.parametrize("mut", [_mut_bf16_single_rounding, _mut_bf16_reverse_order, _mut_bf16_partials_unrounded])
def test_planted_bf16_allreduce_mistakes_fail_pins(mut):
    X1, V1 = np.array([[1.0, 1.0, 1.0]]), np.array([[256.0], [1.0], [1.0]])
    X2, V2 = np.array([[1.0 + 2.0 ** -8, 2.0 ** -8]]), np.array([[1.0], [1.0]])
    ok1 = mut(X1, V1, 3)[0][0, 0] == 256.0
    ok2 = mut(X2, V2, 2)[0][0, 0] == 1.0
    assert not (ok1 and ok2)


# ============================================================ the whole attention block
@pytest.mark.parametrize("hq,hkv,tp", [(8, 2, 1), (8, 2, 2), (8, 2, 4), (8, 2, 8), (4, 4, 4)])
def test_sharded_attention_block_equals_single_device(hq, hkv, tp):
    """The validation the mini-vLLM page prescribes ("如何验证 tensor parallel 正确":
    the tensor-parallel result must match the single-GPU one): QKV column-parallel by
    head, attention on local heads, o_proj row-parallel with the partials summed,
    against the unsharded block softmax(X Wq (X Wk)^T / sqrt(d)) X Wv Wo."""
    rng = np.random.default_rng(31 + tp)
    nseq, S, d, H = 2, 5, 4, 16
    X = rng.standard_normal((nseq * S, H))
    Wq = rng.standard_normal((H, hq * d)) * 0.3
    Wk = rng.standard_normal((H, hkv * d)) * 0.3
    Wv = rng.standard_normal((H, hkv * d)) * 0.3
    Wo = rng.standard_normal((hq * d, H)) * 0.3
    qkv, _ = O.qkv_sharded(X, Wq, Wk, Wv, hq, hkv, d, tp)
    A = O.gqa_attention_sharded(qkv, hq, hkv, d, tp, nseq, S, True)
    _, Y = O.attn_proj_sharded(X, A, Wq, Wk, Wv, Wo, hq, hkv, d, tp)
    ref = O.gqa_attention(X @ Wq, X @ Wk, X @ Wv, hq, hkv, d, nseq, S, True) @ Wo
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


# ============================================================ randomized properties (hypothesis)
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(m=st.integers(1, 4), k=st.integers(1, 6), per=st.integers(1, 6), tp=st.sampled_from([1, 2, 3, 4]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_property_column_concat_and_row_sum(m, k, per, tp, seed):
    """For any shapes that divide: concat of column shards = X W and the sum of row
    partials = X V (small integers, exact in fp64)."""
    rng = np.random.default_rng(seed)
    X = rng.integers(-3, 4, size=(m, k * tp)).astype(float)
    W = rng.integers(-3, 4, size=(k * tp, per * tp)).astype(float)
    Y, shards = O.column_parallel(X, W, tp)
    assert np.array_equal(Y, X @ W) and len(shards) == tp
    Yr, parts = O.row_parallel(X, W, tp)
    assert np.array_equal(Yr, X @ W) and len(parts) == tp


@settings(max_examples=40, deadline=None)
@given(m=st.integers(1, 5), H=st.integers(1, 5), per=st.integers(1, 8), tp=st.sampled_from([1, 2, 3, 4, 6]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_property_argmax_equals_unsharded_first_maximum(m, H, per, tp, seed):
    """Greedy over a vocab split in tp: the first maximum of the full logits row, ties
    included (small integers make ties frequent)."""
    rng = np.random.default_rng(seed)
    X = rng.integers(-2, 3, size=(m, H)).astype(float)
    W = rng.integers(-2, 3, size=(H, per * tp)).astype(float)
    idx, val = O.vocab_parallel_argmax(X, W, tp)
    L = X @ W
    assert np.array_equal(idx, np.argmax(L, axis=1))
    assert np.array_equal(val, L.max(axis=1))


@settings(max_examples=25, deadline=None)
@given(nseq=st.integers(1, 3), S=st.integers(1, 6), grp=st.sampled_from([1, 2, 4]), hkv=st.sampled_from([1, 2]),
       causal=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
def test_property_attention_sharded_equals_unsharded(nseq, S, grp, hkv, causal, seed):
    """Attention on local heads equals the unsharded grouped attention for every tp
    the head map admits."""
    rng = np.random.default_rng(seed)
    d, hq = 4, grp * hkv
    Q = rng.standard_normal((nseq * S, hq * d))
    K = rng.standard_normal((nseq * S, hkv * d))
    V = rng.standard_normal((nseq * S, hkv * d))
    ref = O.gqa_attention(Q, K, V, hq, hkv, d, nseq, S, causal)
    for tp in O.valid_tp_sizes(hq):
        if hkv % tp and tp % hkv:
            continue
        got = O.gqa_attention_sharded(_shard_layout(Q, K, V, hq, hkv, d, tp), hq, hkv, d, tp, nseq, S, causal)
        assert np.allclose(got, ref, atol=1e-12)
