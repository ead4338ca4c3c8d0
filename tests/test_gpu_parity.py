"""GPU parity of the CUDA path (through the C ABI) against the CPU fp64 oracle.

Bar: bit-exact on integer-valued inputs (fp32 accumulation is exact there) and
for the packer (a bit copy); for random bf16 inputs with fp32 accumulation the
relative Frobenius error must be <= 5e-3 and the max elementwise error
<= 1e-2 * max|ref|. Integer-valued intermediates are compared in "contract" mode:
the oracle rounds the stored bf16 intermediate h exactly where the GPU stores it.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
REL_MAX = 1e-2
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tensor_sharded_linear_columnparallel_b200 as T
    return T


@pytest.fixture(autouse=True)
def _reset_plan(T):
    T.tps_set_plan_override(0)
    yield
    T.tps_set_plan_override(0)
    torch.cuda.synchronize()
    assert T.tps_device_error() == T.TPS_OK


def cuda(t):
    return t.to("cuda").contiguous()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(y, ref, what=""):
    y = f64(y) if isinstance(y, torch.Tensor) else np.asarray(y, np.float64)
    assert y.shape == ref.shape, (what, y.shape, ref.shape)
    assert np.isfinite(y).all(), what
    d = y - ref
    nref = np.linalg.norm(ref)
    fro = np.linalg.norm(d) / (nref if nref > 0 else 1.0)
    mx = np.abs(d).max() if d.size else 0.0
    amax = np.abs(ref).max() if ref.size else 0.0
    assert fro <= REL_FRO, f"{what}: rel Frobenius {fro:.3e}"
    assert mx <= REL_MAX * max(amax, 1e-30), f"{what}: max err {mx:.3e} vs {REL_MAX}*{amax:.3e}"


def assert_exact(y, ref, what=""):
    y = f64(y)
    assert y.shape == ref.shape, (what, y.shape, ref.shape)
    bad = np.argwhere(y != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first {bad[:3].tolist()} " \
                          f"{[(y[tuple(b)], ref[tuple(b)]) for b in bad[:3]]}"


def ws_for(T, fn, m, n, k, tp):
    return T.workspace(fn, m, n, k, tp)


# token-major / weight-major, forced / forbidden split-K, CTA-pair tiles (256 and 128 wide),
# cluster split-K (row-parallel) in both orientations
CSPLIT = 1 << 16   # plan-override bit: prefer cluster split-K (row-parallel)
PLANS = [0, 1, 2, 1 | 16, 2 | 16, 1 | 32, 2 | 32, 1 | 64, 1 | 64 | (4 << 8), 1 | CSPLIT, 2 | CSPLIT,
         1 | CSPLIT | (3 << 8), 1 | CSPLIT | (4 << 8), 2 | CSPLIT | (1 << 8),
         1 | CSPLIT | (1 << 12), 1 | CSPLIT | (3 << 12), 2 | CSPLIT | (1 << 12), 2 | CSPLIT | (3 << 12)]


def unpack(pk, tp, R, Kp):
    """Packed shards [tp][RB][KB][128][64] (layout of include/tps.h) -> [tp][R][Kp]."""
    RB, KB = (R + 127) // 128, (Kp + 63) // 64
    a = f64(pk).reshape(tp, RB, KB, 128, 64).transpose(0, 1, 3, 2, 4).reshape(tp, RB * 128, KB * 64)
    assert not a[:, R:, :].any() and not a[:, :, Kp:].any(), "padding must be zero"
    return a[:, :R, :Kp]


# ============================================================ packer (bit copy)
@pytest.mark.parametrize("transposed", [False, True])
def test_pack_column_and_row_bit_exact(T, transposed):
    k, n, tp = 96, 320, 4
    W = WL.gen_normal((k, n), 1.0, 11)
    src = W.t().contiguous() if transposed else W
    pk = T.tp_shard_weights(T.KIND_COLUMN, cuda(src), tp, transposed=transposed).cpu()
    shards = O.split_columns(W, tp)
    got = unpack(pk, tp, n // tp, k)
    for i in range(tp):
        assert np.array_equal(got[i], shards[i].T)
    pk = T.tp_shard_weights(T.KIND_ROW, cuda(src), tp, transposed=transposed).cpu()
    rows = O.split_rows(W, tp)
    got = unpack(pk, tp, n, k // tp)
    for i in range(tp):
        assert np.array_equal(got[i], rows[i].T)


@pytest.mark.parametrize("tp", [4, 8, 16])
@pytest.mark.parametrize("transposed", [False, True])
def test_pack_qkv_bit_exact(T, tp, transposed):
    hq, hkv, d, k = 32, 8, 16, 64
    W = WL.gen_normal((k, (hq + 2 * hkv) * d), 1.0, 12)
    src = W.t().contiguous() if transposed else W
    pk = T.tp_shard_weights(T.KIND_QKV, cuda(src), tp, heads=T.Heads(hq, hkv, d), transposed=transposed)
    cols = O.qkv_shard_columns(hq, hkv, d, tp)
    got = unpack(pk, tp, len(cols[0]), k)
    Wf = O.to_f64(W)
    for r in range(tp):
        assert np.array_equal(got[r], Wf[:, cols[r]].T)


@pytest.mark.parametrize("I,tp", [(14336, 8), (400, 2), (256, 1)])
def test_pack_gate_up_bit_exact(T, I, tp):
    k = 64
    Wg, Wu = WL.gen_normal((k, I), 1.0, 13), WL.gen_normal((k, I), 1.0, 14)
    W = torch.cat([Wg, Wu], dim=1)
    pk = T.tp_shard_weights(T.KIND_GATE_UP, cuda(W), tp)
    Is = I // tp
    nb = (Is + 127) // 128
    got = unpack(pk, tp, nb * 256, k).reshape(tp, nb, 2, 128, k)
    gs, us = O.split_columns(Wg, tp), O.split_columns(Wu, tp)
    for r in range(tp):
        for b in range(nb):
            lo, hi = b * 128, min(Is, b * 128 + 128)
            assert np.array_equal(got[r, b, 0, :hi - lo], gs[r][:, lo:hi].T)
            assert np.array_equal(got[r, b, 1, :hi - lo], us[r][:, lo:hi].T)
            assert not got[r, b, :, hi - lo:].any()


# ============================================================ worked example
def test_worked_example_padded(T):
    """The two-GPU hand example, zero-padded to k = 16 and 8 columns per shard."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    X = torch.zeros(1, 16)
    X[0, :2] = torch.tensor(g["X"][0], dtype=torch.float32)
    Wx = np.array(g["W"], float)
    W = torch.zeros(16, 16)
    W[:2, 0:2] = torch.tensor(Wx[:, 0:2])        # left half -> shard 0
    W[:2, 8:10] = torch.tensor(Wx[:, 2:4])       # right half -> shard 1
    V = torch.zeros(16, 8)
    Vx = np.array(g["V"], float)
    V[0:2, 0] = torch.tensor(Vx[0:2, 0])         # upper half -> shard 0
    V[8:10, 0] = torch.tensor(Vx[2:4, 0])        # lower half -> shard 1
    X, W, V = (cuda(t.to(torch.bfloat16)) for t in (X, W, V))
    for plan in PLANS:
        T.tps_set_plan_override(plan)
        Y = T.column_parallel_forward(X, T.tp_shard_weights(T.KIND_COLUMN, W, 2), T.KIND_COLUMN, 16, 2,
                                      y_dtype=torch.float32)
        y = f64(Y)[0]
        assert list(y[0:2]) == g["Y_shards_tp2"][0][0] and list(y[8:10]) == g["Y_shards_tp2"][1][0]
        P = torch.empty(2, 1, 8, dtype=torch.float32, device="cuda")
        Z = T.row_parallel_forward(Y.to(torch.bfloat16), T.tp_shard_weights(T.KIND_ROW, V, 2), 8, 2,
                                   reduce_mode=T.REDUCE_PARTIALS, partials=P, y_dtype=torch.float32)
        assert f64(P)[0, 0, 0] == g["row_partials_tp2"][0][0][0]
        assert f64(P)[1, 0, 0] == g["row_partials_tp2"][1][0][0]
        assert f64(Z)[0, 0] == g["row_sum"][0][0]
        Z = T.row_parallel_forward(Y.to(torch.bfloat16), T.tp_shard_weights(T.KIND_ROW, V, 2), 8, 2,
                                   y_dtype=torch.float32)
        assert f64(Z)[0, 0] == g["row_sum"][0][0]


# ============================================================ integer pair: bit-exact
@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_int_pair_bit_exact(T, plan, ydt):
    wl = WL.int_pair()
    m, k, n = wl.dims["m"], wl.dims["k"], wl.dims["n"]
    tp = 2
    t = {key: cuda(v) for key, v in wl.tensors.items()}
    T.tps_set_plan_override(plan)
    ws = ws_for(T, T.FN_ROW, m, k, n, tp)
    for use_bias in (False, True):
        bc, br = (t["b_col"], t["b_row"]) if use_bias else (None, None)
        pw = T.tp_shard_weights(T.KIND_COLUMN, t["W"], tp)
        pv = T.tp_shard_weights(T.KIND_ROW, t["V"], tp)
        h = T.column_parallel_forward(t["X"], pw, T.KIND_COLUMN, n, tp, bias=bc, ws=ws)   # bf16 h
        Y = T.row_parallel_forward(h, pv, k, tp, bias=br, y_dtype=ydt, ws=ws)
        Yo, ho = O.int_pair_sharded(wl.tensors["X"], wl.tensors["W"], wl.tensors["V"], tp,
                                    None if bc is None else wl.tensors["b_col"],
                                    None if br is None else wl.tensors["b_row"], round_h=True)
        assert_exact(h, ho, "h")
        assert_exact(Y, Yo if ydt == torch.float32 else O.bf16_round(Yo), "Y")
        # unrounded column output in fp32 equals the unsharded product exactly
        Yc = T.column_parallel_forward(t["X"], pw, T.KIND_COLUMN, n, tp, bias=bc, y_dtype=torch.float32, ws=ws)
        assert_exact(Yc, O.linear(wl.tensors["X"], wl.tensors["W"], None if bc is None else wl.tensors["b_col"]),
                     "column fp32")


@pytest.mark.parametrize("tp", [1, 2, 4, 8, 16])
def test_int_concat_and_sum_invariants_every_tp(T, tp):
    """Column concat == unsharded and row sum == unsharded, bit-exact, for tp in {1,...,16}."""
    wl = WL.int_pair()
    X, W, V = (cuda(wl.tensors[key]) for key in ("X", "W", "V"))
    n, k = wl.dims["n"], wl.dims["k"]
    Yc = T.column_parallel_forward(X, T.tp_shard_weights(T.KIND_COLUMN, W, tp), T.KIND_COLUMN, n, tp,
                                   y_dtype=torch.float32)
    assert_exact(Yc, O.linear(wl.tensors["X"], wl.tensors["W"]), "column")
    # row layer on integer bf16 input [m, n] (values <= 256 in magnitude stay exact)
    Xr = cuda(WL.gen_int((5, n), -3, 3, 77))
    ws = ws_for(T, T.FN_ROW, 5, k, n, tp)
    for mode in (T.REDUCE_FUSED, T.REDUCE_PARTIALS):
        for plan in (0, 2 | 16, 2 | CSPLIT, 1 | CSPLIT):
            T.tps_set_plan_override(plan)
            Yr = T.row_parallel_forward(Xr, T.tp_shard_weights(T.KIND_ROW, V, tp), k, tp, reduce_mode=mode,
                                        y_dtype=torch.float32, ws=ws)
            assert_exact(Yr, O.row_parallel(Xr.cpu(), wl.tensors["V"], tp)[0], f"row mode={mode} plan={plan}")


# ============================================================ GELU MLP
@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_gelu_mlp_full_size(T, tp):
    wl = WL.gelu_mlp()
    m, H, I = wl.dims["m"], wl.dims["H"], wl.dims["I"]
    X, W1, W2 = (cuda(wl.tensors[key]) for key in ("X", "W1", "W2"))
    p1 = T.tp_shard_weights(T.KIND_COLUMN, W1, tp)
    p2 = T.tp_shard_weights(T.KIND_ROW, W2, tp)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    Y, h = T.sharded_mlp_forward(X, H, I, tp, T.ACT_GELU, p1, p2, ws=ws)
    Yo, ho = O.mlp_gelu_sharded(wl.tensors["X"], wl.tensors["W1"], wl.tensors["W2"], tp)
    assert_close(h, ho, "h")
    assert_close(Y, Yo, "Y")
    Yu = O.mlp_gelu(wl.tensors["X"], wl.tensors["W1"], wl.tensors["W2"])
    assert_close(Y, Yu, "Y vs unsharded")


FUSED_MLP = 1 << 18      # plan-override bit: the one-launch MLP kernel, an error if it cannot run
NO_FUSED_MLP = 1 << 19   # plan-override bit: column and row GEMMs as two launches


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("m", [1, 77, 300])
def test_gelu_mlp_ragged_every_plan(T, plan, m):
    wl = WL.gelu_mlp(m=m, hidden=256, inter=1024)
    H, I, tp = 256, 1024, 4
    X, W1, W2 = (cuda(wl.tensors[key]) for key in ("X", "W1", "W2"))
    T.tps_set_plan_override(plan | NO_FUSED_MLP)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    Y, h = T.sharded_mlp_forward(X, H, I, tp, T.ACT_GELU, T.tp_shard_weights(T.KIND_COLUMN, W1, tp),
                                 T.tp_shard_weights(T.KIND_ROW, W2, tp), ws=ws, y_dtype=torch.float32)
    Yo, ho = O.mlp_gelu_sharded(wl.tensors["X"], wl.tensors["W1"], wl.tensors["W2"], tp)
    assert_close(h, ho, "h")
    assert_close(Y, Yo, "Y")


@pytest.mark.parametrize("m,H,I,tp", [(512, 1024, 4096, 8), (512, 1024, 4096, 1), (300, 256, 1024, 4),
                                      (77, 256, 1024, 2), (1000, 256, 2048, 8), (1, 256, 1024, 4), (129, 512, 512, 2)])
def test_fused_mlp_one_launch(T, m, H, I, tp):
    """The one-launch MLP (fc1 tiles, then cluster split-K fc2 tiles gated by
    per-shard readiness flags): parity with the oracle, the same bits on a second
    call (the flags are re-zeroed by the kernel) and no device error."""
    wl = WL.gelu_mlp(m=m, hidden=H, inter=I)
    X, W1, W2 = (cuda(wl.tensors[key]) for key in ("X", "W1", "W2"))
    p1 = T.tp_shard_weights(T.KIND_COLUMN, W1, tp)
    p2 = T.tp_shard_weights(T.KIND_ROW, W2, tp)
    T.tps_set_plan_override(FUSED_MLP)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    outs = []
    for _ in range(3):
        Y, h = T.sharded_mlp_forward(X, H, I, tp, T.ACT_GELU, p1, p2, ws=ws, y_dtype=torch.float32)
        outs.append((Y.clone(), h.clone()))
    assert T.tps_device_error() == T.TPS_OK
    Yo, ho = O.mlp_gelu_sharded(wl.tensors["X"], wl.tensors["W1"], wl.tensors["W2"], tp)
    assert_close(outs[0][1], ho, "h")
    assert_close(outs[0][0], Yo, "Y")
    for Yr, hr in outs[1:]:
        assert torch.equal(Yr, outs[0][0]) and torch.equal(hr, outs[0][1])
    # the workspace's flag region is left zero for the next user
    assert int(ws.view(torch.int32).count_nonzero()) == 0


# ============================================================ gated decode
@pytest.mark.parametrize("m", [1, 8, 32, 64])
def test_gated_decode_full_size(T, m):
    wl = getattr(test_gated_decode_full_size, "_wl", None)
    if wl is None:
        wl = WL.gated_decode()
        test_gated_decode_full_size._wl = wl
    H, I, tp = wl.dims["H"], wl.dims["I"], 8
    key = "_packed"
    pk = getattr(test_gated_decode_full_size, key, None)
    if pk is None:
        Wgu = torch.cat([wl.tensors["Wg"], wl.tensors["Wu"]], dim=1)
        pk = (T.tp_shard_weights(T.KIND_GATE_UP, cuda(Wgu), tp), T.tp_shard_weights(T.KIND_ROW, cuda(wl.tensors["Wd"]), tp))
        test_gated_decode_full_size._packed = pk
    X = cuda(wl.tensors["X"][:m])
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    Y, h = T.sharded_mlp_forward(X, H, I, tp, T.ACT_SILU_MUL, pk[0], pk[1], ws=ws)
    Yo, ho = O.mlp_gated_sharded(wl.tensors["X"][:m], wl.tensors["Wg"], wl.tensors["Wu"], wl.tensors["Wd"], tp)
    assert_close(h, ho, "h")
    assert_close(Y, Yo, "Y")


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("m,I,tp", [(5, 400, 2), (33, 2048, 8), (130, 1024, 4)])
def test_gated_mlp_ragged_every_plan(T, plan, m, I, tp):
    H = 128
    X = WL.gen_normal((m, H), 1.0, 31)
    Wg, Wu = WL.gen_normal((H, I), H ** -0.5, 32), WL.gen_normal((H, I), H ** -0.5, 33)
    Wd = WL.gen_normal((I, H), I ** -0.5, 34)
    T.tps_set_plan_override(plan | NO_FUSED_MLP)
    pgu = T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([Wg, Wu], 1)), tp)
    pd = T.tp_shard_weights(T.KIND_ROW, cuda(Wd), tp)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    Y, h = T.sharded_mlp_forward(cuda(X), H, I, tp, T.ACT_SILU_MUL, pgu, pd, ws=ws)
    Yo, ho = O.mlp_gated_sharded(X, Wg, Wu, Wd, tp)
    assert_close(h, ho, "h")
    assert_close(Y, Yo, "Y")


SK_MLP = 1 << 22        # plan-override bit: the stream-K form of the one-launch gated MLP
NO_SK_MLP = 1 << 23     # plan-override bit: the cluster form


@pytest.mark.parametrize("form", [SK_MLP, NO_SK_MLP])
@pytest.mark.parametrize("m,H,I,tp", [(64, 4096, 14336, 8), (1, 4096, 14336, 8), (33, 4096, 14336, 8),
                                      (5, 128, 400, 2), (17, 256, 2048, 4), (64, 512, 1024, 1),
                                      (40, 1024, 3072, 3)])
def test_fused_gated_mlp_one_launch(T, m, H, I, tp, form):
    """The one-launch gated MLP for decode-sized m in both forms -- stream-K over
    both layers on one CTA per SM (phase-1 tiles finished by the last CTA of each,
    down iterations gated by per-shard readiness flags), and weight-major gate/up
    pairs followed by the cluster split-K down projection: oracle parity, the same
    bits on repeats, workspace (tile counters and flags) left zero."""
    X = WL.gen_normal((m, H), 1.0, 61)
    Wg, Wu = WL.gen_normal((H, I), H ** -0.5, 62), WL.gen_normal((H, I), H ** -0.5, 63)
    Wd = WL.gen_normal((I, H), I ** -0.5, 64)
    pgu = T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([Wg, Wu], 1)), tp)
    pd = T.tp_shard_weights(T.KIND_ROW, cuda(Wd), tp)
    T.tps_set_plan_override(FUSED_MLP | form)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    outs = []
    for _ in range(3):
        Y, h = T.sharded_mlp_forward(cuda(X), H, I, tp, T.ACT_SILU_MUL, pgu, pd, ws=ws, y_dtype=torch.float32)
        outs.append((Y.clone(), h.clone()))
    assert T.tps_device_error() == T.TPS_OK
    Yo, ho = O.mlp_gated_sharded(X, Wg, Wu, Wd, tp)
    assert_close(outs[0][1], ho, "h")
    assert_close(outs[0][0], Yo, "Y")
    for Yr, hr in outs[1:]:
        assert torch.equal(Yr, outs[0][0]) and torch.equal(hr, outs[0][1])
    assert_ws_state_zero(ws)


@pytest.mark.parametrize("act,m,H,I,tp", [("gelu", 300, 1024, 4096, 8), ("gated", 37, 512, 1600, 4)])
def test_one_launch_mlp_writes_only_its_outputs(T, act, m, H, I, tp):
    """The one-launch MLP kernels (both forms) write h and Y and nothing else: the
    epilogue warps' early dry passes through the epilogue code store nothing, so the
    rows past m of oversized h and Y buffers keep their sentinel, and the results
    match the oracle."""
    X = WL.gen_normal((m, H), 1.0, 71)
    pad = 64
    if act == "gelu":
        W1, W2 = WL.gen_normal((H, I), 0.02, 72), WL.gen_normal((I, H), 0.02, 73)
        pu = T.tp_shard_weights(T.KIND_COLUMN, cuda(W1), tp)
        pd = T.tp_shard_weights(T.KIND_ROW, cuda(W2), tp)
        code = T.ACT_GELU
    else:
        Wg, Wu = WL.gen_normal((H, I), H ** -0.5, 74), WL.gen_normal((H, I), H ** -0.5, 75)
        Wd = WL.gen_normal((I, H), I ** -0.5, 76)
        pu = T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([Wg, Wu], 1)), tp)
        pd = T.tp_shard_weights(T.KIND_ROW, cuda(Wd), tp)
        code = T.ACT_SILU_MUL
    sentinel = -12345.0
    hbuf = torch.full((m + pad, I), sentinel, dtype=torch.bfloat16, device="cuda")
    ybuf = torch.full((m + pad, H), sentinel, dtype=torch.bfloat16, device="cuda")
    T.tps_set_plan_override(FUSED_MLP)
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    Y, h = T.sharded_mlp_forward(cuda(X), H, I, tp, code, pu, pd, h_ws=hbuf[:m], out=ybuf[:m], ws=ws)
    torch.cuda.synchronize()
    assert T.tps_device_error() == T.TPS_OK
    assert bool((hbuf[m:] == sentinel).all()) and bool((ybuf[m:] == sentinel).all())
    if act == "gelu":
        Yo, ho = O.mlp_gelu_sharded(X, W1, W2, tp)
    else:
        Yo, ho = O.mlp_gated_sharded(X, Wg, Wu, Wd, tp)
    assert_close(h, ho, "h")
    assert_close(Y, Yo, "Y")


def assert_ws_state_zero(ws):
    """The workspace's status header, tile counters and readiness flags are zero
    after a completed call (the split-K segment slots between them hold partials
    that every call writes before it reads them)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    slots_end = 256 + 2 * sms * 128 * 256 * 4
    b = ws.view(torch.uint8)
    assert int(b[:256].count_nonzero()) == 0
    assert int(b[slots_end:].count_nonzero()) == 0


# ============================================================ vocab-parallel greedy argmax
@pytest.mark.parametrize("m,H,V,tp", [(1, 4096, 32000, 8), (8, 4096, 32000, 8), (64, 1024, 16000, 4),
                                      (300, 512, 8192, 4), (129, 256, 2000, 2)])
def test_vocab_parallel_argmax_random(T, m, H, V, tp):
    """Random logits: the chosen token's (fp64) logit is a maximum within the fp32
    accumulation's rounding, the returned value matches, and wherever the maximum
    is unique beyond rounding the token is the oracle's."""
    X = WL.gen_normal((m, H), 1.0, 71)
    W = WL.gen_normal((H, V), H ** -0.5, 72)
    idx, val = T.vocab_parallel_argmax(cuda(X), H, V, tp, T.tp_shard_weights(T.KIND_COLUMN, cuda(W), tp))
    torch.cuda.synchronize()
    oi, ov = O.vocab_parallel_argmax(X, W, tp)
    L = O.linear(X, W)
    gi = idx.cpu().numpy().astype(np.int64)
    gv = val.cpu().numpy().astype(np.float64)
    tol = 1e-4 * (1.0 + np.abs(ov))
    assert np.all((gi >= 0) & (gi < V))
    assert np.all(L[np.arange(m), gi] >= ov - tol)
    assert np.all(np.abs(gv - ov) <= tol)
    second = np.sort(L, axis=1)[:, -2]
    unique = (ov - second) > 2 * tol
    assert np.array_equal(gi[unique], oi[unique])
    assert unique.sum() >= 0.75 * m   # near-ties (top-two gap within rounding) are rare but do occur


def test_vocab_parallel_argmax_full_size_lm_head(T):
    """The greedy lm_head the bench times (H=4096, V=128256, tp=8, m=64 and the
    decode sizes below it), every token against the oracle, with the plan and
    launch configuration the bench uses (no override)."""
    wl = WL.lm_head()
    X, W = wl.tensors["X"], wl.tensors["W"]
    H, V = wl.dims["H"], wl.dims["V"]
    pw = T.tp_shard_weights(T.KIND_COLUMN, cuda(W), 8)
    L = O.linear(X, W)
    for m in wl.dims["m_list"]:
        idx, val = T.vocab_parallel_argmax(cuda(X[:m]), H, V, 8, pw)
        torch.cuda.synchronize()
        Lm = L[:m]
        oi = np.argmax(Lm, axis=1)
        ov = Lm[np.arange(m), oi]
        gi = idx.cpu().numpy().astype(np.int64)
        gv = val.cpu().numpy().astype(np.float64)
        tol = 1e-4 * (1.0 + np.abs(ov))
        assert np.all((gi >= 0) & (gi < V))
        assert np.all(Lm[np.arange(m), gi] >= ov - tol)
        assert np.all(np.abs(gv - ov) <= tol)
        second = np.sort(Lm, axis=1)[:, -2]
        unique = (ov - second) > 2 * tol
        assert np.array_equal(gi[unique], oi[unique])
    assert T.tps_device_error() == T.TPS_OK


@pytest.mark.parametrize("plan", [0, 1, 2, 1 | (3 << 8), 1 | (5 << 8), 2 | (1 << 8), 2 | (4 << 8)])
def test_vocab_parallel_argmax_integer_ties_exact(T, plan):
    """Small integers: every logit is exact in fp32 and ties are frequent, so the
    token (lowest vocab index among the maxima) and the value must be bit-exact."""
    m, H, V, tp = 40, 64, 2048, 4
    X = WL.gen_int((m, H), -2, 2, 81)
    W = WL.gen_int((H, V), -2, 2, 82)
    T.tps_set_plan_override(plan)
    idx, val = T.vocab_parallel_argmax(cuda(X), H, V, tp, T.tp_shard_weights(T.KIND_COLUMN, cuda(W), tp))
    oi, ov = O.vocab_parallel_argmax(X, W, tp)
    assert np.array_equal(idx.cpu().numpy().astype(np.int64), oi)
    assert np.array_equal(val.cpu().numpy().astype(np.float64), ov)


def test_vocab_parallel_argmax_errors(T):
    X = cuda(WL.gen_normal((4, 64), 1.0, 91))
    pw = T.tp_shard_weights(T.KIND_COLUMN, cuda(WL.gen_normal((64, 256), 0.1, 92)), 2)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(T.TpsError) as e:
        T.vocab_parallel_argmax(X, 64, 256, 2, pw, ws=small)
    assert e.value.status == T.TPS_ERR_WORKSPACE
    empty = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    idx, _ = T.vocab_parallel_argmax(empty, 64, 256, 2, pw)
    assert idx.numel() == 0


def test_gate_up_bias(T):
    m, H, I, tp = 40, 64, 512, 4
    X = WL.gen_normal((m, H), 1.0, 41)
    W = WL.gen_normal((H, 2 * I), 0.1, 42)
    b = WL.gen_normal((2 * I,), 0.5, 43)
    for plan in (1, 2):
        T.tps_set_plan_override(plan)
        h = T.column_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_GATE_UP, cuda(W), tp), T.KIND_GATE_UP,
                                      2 * I, tp, bias=cuda(b), act=T.ACT_SILU_MUL, y_dtype=torch.float32)
        Wf, bf = O.to_f64(W), O.to_f64(b)
        ref = O.silu_mul(O.linear(X, Wf[:, :I], bf[:I]), O.linear(X, Wf[:, I:], bf[I:]))
        assert_close(h, ref, f"plan {plan}")


# ============================================================ GQA attention projections
@pytest.mark.parametrize("tp", [4, 8, 16])
@pytest.mark.parametrize("m", [1, 200])
def test_gqa_proj_every_tp(T, tp, m):
    hq, hkv, d, H = 32, 8, 32, 512
    X = WL.gen_normal((m, H), 1.0, 51)
    Wq, Wk, Wv = (WL.gen_normal((H, c * d), 0.05, 52 + i) for i, c in enumerate((hq, hkv, hkv)))
    Wo = WL.gen_normal((hq * d, H), 0.05, 55)
    A = WL.gen_normal((m, hq * d), 1.0, 56)
    heads = T.Heads(hq, hkv, d)
    pq = T.tp_shard_weights(T.KIND_QKV, cuda(torch.cat([Wq, Wk, Wv], 1)), tp, heads=heads)
    po = T.tp_shard_weights(T.KIND_ROW, cuda(Wo), tp)
    ws = ws_for(T, T.FN_ATTN, m, H, hq * d, tp)
    for plan in (0, 1, 2 | 16, 1 | 64):
        T.tps_set_plan_override(plan)
        Y, qkv = T.sharded_attn_proj_forward(cuda(X), cuda(A), H, heads, tp, pq, po, ws=ws)
        qo, Yo = O.attn_proj_sharded(X, A, Wq, Wk, Wv, Wo, hq, hkv, d, tp)
        assert_close(qkv, qo, "qkv")
        assert_close(Y, Yo, "Y")
        # replicated KV slices equal the unsharded head's columns
        full = O.qkv_unsharded(X, Wq, Wk, Wv)
        cols = O.qkv_shard_columns(hq, hkv, d, tp)
        flat = [c for cs in cols for c in cs]
        assert_close(qkv, full[:, flat], "qkv vs unsharded")


def test_qkv_bias(T):
    hq, hkv, d, H, tp, m = 8, 2, 16, 64, 4, 20
    X = WL.gen_normal((m, H), 1.0, 61)
    W = WL.gen_normal((H, (hq + 2 * hkv) * d), 0.1, 62)
    b = WL.gen_normal(((hq + 2 * hkv) * d,), 0.5, 63)
    heads = T.Heads(hq, hkv, d)
    y = T.column_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_QKV, cuda(W), tp, heads=heads), T.KIND_QKV,
                                  (hq + 2 * hkv) * d, tp, heads=heads, bias=cuda(b), y_dtype=torch.float32)
    full = O.linear(X, W, b)
    flat = [c for cs in O.qkv_shard_columns(hq, hkv, d, tp) for c in cs]
    assert_close(y, full[:, flat], "qkv+bias")


def test_gqa_full_size_every_row(T):
    """GQA projections at the bench's full size (m = 2048), every element of the
    QKV output and of o_proj against the fp64 oracle, for tp = 4, 8 and 16 (KV
    heads replicated at 16), with the plans the entry point picks by itself."""
    wl = WL.gqa_proj()
    m, H, hq, hkv, d = (wl.dims[x] for x in ("m", "H", "hq", "hkv", "d"))
    heads = T.Heads(hq, hkv, d)
    tt = wl.tensors
    Wqkv = cuda(torch.cat([tt["Wq"], tt["Wk"], tt["Wv"]], 1))
    for tp in (4, 8, 16):
        pq = T.tp_shard_weights(T.KIND_QKV, Wqkv, tp, heads=heads)
        po = T.tp_shard_weights(T.KIND_ROW, cuda(tt["Wo"]), tp)
        Y, qkv = T.sharded_attn_proj_forward(cuda(tt["X"]), cuda(tt["A"]), H, heads, tp, pq, po,
                                             ws=ws_for(T, T.FN_ATTN, m, H, hq * d, tp))
        qo, Yo = O.attn_proj_sharded(tt["X"], tt["A"], tt["Wq"], tt["Wk"], tt["Wv"], tt["Wo"], hq, hkv, d, tp)
        assert_close(qkv, qo, f"qkv tp={tp}")
        assert_close(Y, Yo, f"Y tp={tp}")


def tile_rows(m: int) -> np.ndarray:
    """Token rows that hit every output tile of any plan: the first and last row
    of every 128-token tile (so both halves of every 256-token CTA-pair tile and
    every pair boundary 256j - 1, 256j), one interior row per 128-token tile at a
    position that moves from tile to tile (every TMEM lane quarter is visited),
    and the last row m - 1."""
    rows = set()
    for t in range((m + 127) // 128):
        lo, hi = t * 128, min(m, t * 128 + 128) - 1
        rows.update((lo, hi, min(hi, lo + 1 + (t * 37) % 126)))
    rows.add(m - 1)
    return np.array(sorted(rows))


def assert_close_tiles(y, ref, rows, what):
    """assert_close on all sampled rows, then on each 128-token tile's rows alone,
    so that a tile-indexed mistake cannot hide in the global norm."""
    y = f64(y)
    assert_close(y, ref, what)
    for t in np.unique(rows // 128):
        sel = (rows // 128) == t
        assert_close(y[sel], ref[sel], f"{what} tile {t}")


def test_tile_rows_cover_every_tile():
    rows = tile_rows(8192)
    for width in (128, 256):
        assert set(rows // width) == set(range(8192 // width))
    # both 128-row halves of every 256-token pair tile, and every TMEM lane quarter
    assert {(r // 128) % 2 for r in rows} == {0, 1}
    assert {(r % 128) // 32 for r in rows} == {0, 1, 2, 3}
    assert 0 in rows and 8191 in rows and all(r in rows for r in (255, 256, 4095, 4096))


# ============================================================ 70B-layer shapes, a row in every tile
def test_layer70b_full_size_every_tile(T):
    """The 70B-layer linears at the bench's full size (m = 8192, tp = 8) through the
    entry points the bench calls, compared with the oracle on the rows of
    tile_rows(): every column of QKV, o_proj, h = SiLU(gate)*up and down, and at
    least three rows of every 128-token tile (so every output tile of every plan
    the planner may pick is checked)."""
    wl = WL.layer70b()
    tt = wl.tensors
    m, H, I, hq, hkv, d = (wl.dims[x] for x in ("m", "H", "I", "hq", "hkv", "d"))
    tp = 8
    heads = T.Heads(hq, hkv, d)
    rows = tile_rows(m)
    ridx = torch.as_tensor(rows, device="cuda")
    X, A = cuda(tt["X"]), cuda(tt["A"])
    ws = ws_for(T, T.FN_MLP, m, H, I, tp)
    pq = T.tp_shard_weights(T.KIND_QKV, cuda(torch.cat([tt["Wq"], tt["Wk"], tt["Wv"]], 1)), tp, heads=heads)
    po = T.tp_shard_weights(T.KIND_ROW, cuda(tt["Wo"]), tp)
    Y, qkv = T.sharded_attn_proj_forward(X, A, H, heads, tp, pq, po, ws=ws)
    qo, Yo = O.attn_proj_sharded(tt["X"][rows], tt["A"][rows], tt["Wq"], tt["Wk"], tt["Wv"], tt["Wo"],
                                 hq, hkv, d, tp)
    assert_close_tiles(qkv[ridx], qo, rows, "qkv")
    assert_close_tiles(Y[ridx], Yo, rows, "o_proj")
    del pq, po, qkv, Y
    pgu = T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([tt["Wg"], tt["Wu"]], 1)), tp)
    pd = T.tp_shard_weights(T.KIND_ROW, cuda(tt["Wd"]), tp)
    Y, h = T.sharded_mlp_forward(X, H, I, tp, T.ACT_SILU_MUL, pgu, pd, ws=ws)
    Yo, ho = O.mlp_gated_sharded(tt["X"][rows], tt["Wg"], tt["Wu"], tt["Wd"], tp)
    assert_close_tiles(h[ridx], ho, rows, "h")
    assert_close_tiles(Y[ridx], Yo, rows, "down")


# ============================================================ wide CTA-pair tiles
WIDE = 1 | 64 | (1 << 20)   # token-major, CTA pairs, wide tiles (256 tokens x 512 weight rows)


@pytest.mark.parametrize("m", [129, 300, 1000])
def test_wide_pair_tiles_every_kind(T, m):
    """Wide pair tiles (two MMA halves of 256 weight rows per 256-token tile, one
    accumulator buffer) on ragged token counts and K: column with GELU and bias,
    gate/up with SiLU(gate)*up, row-parallel with the K loop over the shards (64-wide
    shard K ranges, and ragged ones read through the 3-D view), against the oracle;
    integer inputs bit-exact."""
    T.tps_set_plan_override(WIDE)
    k, n, tp = 200, 1024, 2                      # 512 columns per shard = one wide tile
    X, W, b = WL.gen_normal((m, k), 1.0, 701), WL.gen_normal((k, n), 0.05, 702), WL.gen_normal((n,), 0.5, 703)
    pw = T.tp_shard_weights(T.KIND_COLUMN, cuda(W), tp)
    y = T.column_parallel_forward(cuda(X), pw, T.KIND_COLUMN, n, tp, bias=cuda(b), act=T.ACT_GELU,
                                  y_dtype=torch.float32)
    assert_close(y, O.gelu(O.column_parallel(X, W, tp, b)[0]), "column + GELU")
    H, I, tp = 192, 2048, 4                      # 512 gate + 512 up columns per shard = two wide tiles
    Wg, Wu = WL.gen_normal((H, I), H ** -0.5, 704), WL.gen_normal((H, I), H ** -0.5, 705)
    Xg = WL.gen_normal((m, H), 1.0, 706)
    h = T.column_parallel_forward(cuda(Xg), T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([Wg, Wu], 1)), tp),
                                  T.KIND_GATE_UP, 2 * I, tp, act=T.ACT_SILU_MUL, y_dtype=torch.float32)
    assert_close(h, O.silu_mul(O.linear(Xg, Wg), O.linear(Xg, Wu)), "gate/up")
    for k, n, tp in [(2048, 512, 4), (288, 1024, 4)]:   # shard K 512 (2-D map) and 72 (3-D view)
        Xr, V = WL.gen_normal((m, k), 1.0, 707), WL.gen_normal((k, n), k ** -0.5, 708)
        yr = T.row_parallel_forward(cuda(Xr), T.tp_shard_weights(T.KIND_ROW, cuda(V), tp), n, tp,
                                    y_dtype=torch.float32)
        assert_close(yr, O.row_parallel(Xr, V, tp)[0], f"row k={k}")
    Xi, Wi = WL.gen_int((m, 128), -3, 3, 709), WL.gen_int((128, 1024), -3, 3, 710)
    yi = T.column_parallel_forward(cuda(Xi), T.tp_shard_weights(T.KIND_COLUMN, cuda(Wi), 2), T.KIND_COLUMN, 1024, 2,
                                   y_dtype=torch.float32)
    assert_exact(yi, O.linear(Xi, Wi), "integer column")


# ============================================================ bf16 exchange of the partial sums
# TPS_REDUCE_BF16: every shard's partial rounded to bf16, summed in shard order with
# a rounding after every addition, the bias once with one more rounding -- the
# oracle's row_parallel_bf16_allreduce. Fused for any tp: a cluster of tp CTAs per
# tile (tp in {2, 4, 8}, few tiles) or the shard chain (one CTA per tile walking the
# shards in order; plan-override bit 30 forces it); two kernels with a partials
# buffer.
CHAIN = 1 << 30
CLUSTER = 1 << 14   # plan-override bit: the cluster form (tp = 2, 4, 8)
BF16_PLANS = [0, 1, 2, 1 | (3 << 8), 2 | (1 << 8), 2 | (4 << 8),
              CHAIN, CHAIN | 1, CHAIN | 2, CHAIN | 1 | (3 << 8), CHAIN | 2 | (2 << 8)]


def _bf16_exchange(T, X, pv, n, tp, bias, ydt, partials=None, ws=None):
    return T.row_parallel_forward(X, pv, n, tp, bias=bias, reduce_mode=T.REDUCE_BF16, partials=partials,
                                  y_dtype=ydt, ws=ws)


@pytest.mark.parametrize("plan", BF16_PLANS)
@pytest.mark.parametrize("tp", [1, 2, 4, 8])
def test_bf16_exchange_integer_bit_exact(T, tp, plan):
    """Integer inputs: every fp32 partial is exact and reaches past 256, where bf16
    rounds, so the result depends on every rounding and on the shard order; it must
    equal the oracle bit for bit (fused form, every plan), with and without bias,
    for fp32 and bf16 outputs, and the same through the two-kernel form."""
    m, k, n = 37, 128 * tp if tp > 1 else 256, 200
    # X integers in [-20, 20] (exact in bf16): shard partials of std ~270, often past
    # 256 where the bf16 spacing exceeds 1, and below 2^24 where fp32 stays exact
    Xc = WL.gen_int((m, k), -20, 20, 620 + tp)
    Vc = WL.gen_int((k, n), -3, 3, 630 + tp)
    bc = WL.gen_int((n,), -3, 3, 640)
    X, pv, b = cuda(Xc), T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp), cuda(bc)
    P = torch.empty(tp, m, n, dtype=torch.float32, device="cuda")
    T.tps_set_plan_override(plan)
    for bias, bref in ((None, None), (b, bc)):
        ref, _ = O.row_parallel_bf16_allreduce(Xc, Vc, tp, bref)
        exact, _ = O.row_parallel(Xc, Vc, tp, bref)
        assert not np.array_equal(ref, exact)   # the roundings matter on these inputs
        for ydt in (torch.float32, torch.bfloat16):
            assert_exact(_bf16_exchange(T, X, pv, n, tp, bias, ydt), ref, f"fused tp={tp} {ydt}")
            assert_exact(_bf16_exchange(T, X, pv, n, tp, bias, ydt, partials=P), ref, f"two kernels tp={tp} {ydt}")


@pytest.mark.parametrize("m", [21, 300])
@pytest.mark.parametrize("tp", [3, 16])
def test_bf16_exchange_other_tp(T, tp, m):
    """Shard counts without a cluster form: the shard chain (no partials buffer, both
    tile orientations) and the two-kernel form (fp32 partials, then
    shard_partial_reduce_bf16) are bit-exact on integers whose partials reach past
    256; K per shard (48) is not a whole 64-wide block."""
    k, n = 48 * tp, 200
    Xc, Vc = WL.gen_int((m, k), -20, 20, 650 + m), WL.gen_int((k, n), -3, 3, 651)
    bc = WL.gen_int((n,), -3, 3, 652)
    X, pv, b = cuda(Xc), T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp), cuda(bc)
    P = torch.empty(tp, m, n, dtype=torch.float32, device="cuda")
    ref, _ = O.row_parallel_bf16_allreduce(Xc, Vc, tp, bc)
    for plan in (0, 1, 2):
        T.tps_set_plan_override(plan)
        for ydt in (torch.float32, torch.bfloat16):
            assert_exact(_bf16_exchange(T, X, pv, n, tp, b, ydt), ref, f"chain tp={tp} plan={plan} {ydt}")
    assert_exact(_bf16_exchange(T, X, pv, n, tp, b, torch.float32, partials=P), ref, f"two kernels tp={tp}")


def test_bf16_exchange_ties_in_shard_order(T):
    """Shard partials 256, 1, 1, 0 (tp = 4): in shard order 256 + 1 rounds to 256
    (a tie, to even) and + 1 again to 256, where the exact sum is 258; the
    reversed order would give 258. Both forms and the standalone reduce."""
    tp, k, n = 4, 64, 8
    X = torch.zeros(1, k)
    X[0, :] = 1.0
    V = torch.zeros(k, n)
    V[0, :] = 256.0       # shard 0 (rows 0-15)
    V[16, :] = 1.0        # shard 1
    V[32, :] = 1.0        # shard 2
    Xb, Vb = X.to(torch.bfloat16), V.to(torch.bfloat16)
    ref, _ = O.row_parallel_bf16_allreduce(Xb, Vb, tp)
    assert (ref == 256.0).all()
    pv = T.tp_shard_weights(T.KIND_ROW, cuda(Vb), tp)
    P = torch.empty(tp, 1, n, dtype=torch.float32, device="cuda")
    for plan in (0, 1, 2, CHAIN, CHAIN | 1):
        T.tps_set_plan_override(plan)
        assert_exact(_bf16_exchange(T, cuda(Xb), pv, n, tp, None, torch.float32), ref, f"fused plan {plan}")
        assert_exact(_bf16_exchange(T, cuda(Xb), pv, n, tp, None, torch.float32, partials=P), ref, "two kernels")
    Pc = torch.zeros(tp, 1, n)
    Pc[0], Pc[1], Pc[2] = 256.0, 1.0, 1.0
    assert_exact(T.shard_partial_reduce(cuda(Pc), y_dtype=torch.float32, bf16_exchange=True), ref, "standalone")
    assert f64(T.shard_partial_reduce(cuda(Pc), y_dtype=torch.float32))[0, 0] == 258.0   # the fp32 reduce


@pytest.mark.parametrize("m,k,n,tp", [(512, 4096, 1024, 8), (64, 14336, 4096, 8), (1, 14336, 4096, 8),
                                      (300, 1024, 512, 2), (129, 2048, 384, 4), (2048, 4096, 4096, 8),
                                      (1000, 4096, 1000, 16)])
def test_bf16_exchange_random_matches_oracle(T, m, k, n, tp):
    """bf16 N(0,1) inputs at the workloads' row-layer shapes (fc2 of the GELU MLP,
    the decode down projection, the GQA output projection, where the planner picks
    the shard chain; a ragged tp = 16 case): the fused form as planned, the shard
    chain forced, and the two-kernel form against the oracle's bf16 all-reduce
    within the float tolerance (a partial within an fp32 rounding of a bf16 rounding
    boundary may round the other way), every output value a bf16 number."""
    Xc = WL.gen_normal((m, k), 1.0, 660)
    Vc = WL.gen_normal((k, n), k ** -0.5, 661)
    X, pv = cuda(Xc), T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp)
    P = torch.empty(tp, m, n, dtype=torch.float32, device="cuda")
    ref, _ = O.row_parallel_bf16_allreduce(Xc, Vc, tp)
    fused = _bf16_exchange(T, X, pv, n, tp, None, torch.float32)
    assert_close(fused, ref, "fused")
    T.tps_set_plan_override(CHAIN)
    chained = _bf16_exchange(T, X, pv, n, tp, None, torch.float32)
    T.tps_set_plan_override(0)
    assert_close(chained, ref, "shard chain")
    assert torch.equal(chained, chained.to(torch.bfloat16).float())
    two = _bf16_exchange(T, X, pv, n, tp, None, torch.float32, partials=P)
    assert_close(two, ref, "two kernels")
    # every value is a bf16 number
    assert torch.equal(fused, fused.to(torch.bfloat16).float())


@pytest.mark.parametrize("tp", [2, 4, 8])
@pytest.mark.parametrize("m", [45, 300])
def test_bf16_exchange_chain_equals_cluster(T, tp, m):
    """The cluster form and the shard chain round every shard's fp32 partial to bf16
    and add the rounded partials in shard order with the same roundings, so on any
    input (N(0,1) here, with a bias, ragged m) they agree bit for bit, in both tile
    orientations."""
    k, n = 256 * tp, 200
    Xc = WL.gen_normal((m, k), 1.0, 680 + tp)
    Vc = WL.gen_normal((k, n), k ** -0.5, 681 + tp)
    bc = WL.gen_normal((n,), 1.0, 682)
    X, pv, b = cuda(Xc), T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp), cuda(bc)
    for orient in (1, 2):
        T.tps_set_plan_override(CLUSTER | orient)
        cl = _bf16_exchange(T, X, pv, n, tp, b, torch.float32)
        T.tps_set_plan_override(CHAIN | orient)
        ch = _bf16_exchange(T, X, pv, n, tp, b, torch.float32)
        assert torch.equal(cl.view(torch.int32), ch.view(torch.int32)), (tp, m, orient)


def test_bf16_exchange_form_choice(T, monkeypatch, capfd):
    """The planner's choice of fused bf16 form: a cluster of tp CTAs per tile for
    weight-major tiles and for token-major problems whose exchanges are cheap next to
    walking every shard on one SM (m = 500), the shard chain otherwise (m = 1000, the
    GQA output projection's 16 x 32 tiles), and always for a tp without a cluster
    form."""
    monkeypatch.setenv("TPS_DEBUG_PLAN", "1")
    for m, k, n, tp, want in ((45, 1024, 512, 8, "chain=0"), (2040, 512, 4096, 8, "chain=1"),
                              (45, 768, 512, 16, "chain=1"), (1000, 4096, 1024, 8, "chain=1"),
                              (500, 4096, 1024, 8, "chain=0")):
        Xc, Vc = WL.gen_int((m, k), -3, 3, 670), WL.gen_int((k, n), -3, 3, 671)
        ref, _ = O.row_parallel_bf16_allreduce(Xc, Vc, tp)
        y = _bf16_exchange(T, cuda(Xc), T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp), n, tp, None, torch.float32)
        plans = [ln for ln in capfd.readouterr().err.splitlines() if "bf16 exchange" in ln]
        assert plans and want in plans[-1], (m, tp, plans)
        assert_exact(y, ref, f"m={m} tp={tp}")


# ============================================================ standalone reduce, determinism, edges
@pytest.mark.parametrize("tp,m,n", [(1, 3, 8), (8, 512, 1024), (16, 77, 4100)])
def test_shard_partial_reduce(T, tp, m, n):
    g = torch.Generator().manual_seed(tp * 1000 + m)
    P = torch.randn(tp, m, n, generator=g)
    b = WL.gen_normal((n,), 1.0, 71)
    for ydt in (torch.float32, torch.bfloat16):
        Y = T.shard_partial_reduce(cuda(P), bias=cuda(b), y_dtype=ydt)
        ref = O.to_f64(P).sum(axis=0) + O.to_f64(b)[None, :]
        assert_close(Y, ref, f"reduce {ydt}")


def test_split_k_reduction_is_deterministic(T):
    m, k, n, tp = 64, 4096, 1024, 8
    X = cuda(WL.gen_normal((m, k), 1.0, 81))
    V = cuda(WL.gen_normal((k, n), 0.02, 82))
    pv = T.tp_shard_weights(T.KIND_ROW, V, tp)
    ws = ws_for(T, T.FN_ROW, m, n, k, tp)
    for plan in (2 | 16, 1 | 16, 1 | CSPLIT, 2 | CSPLIT):
        T.tps_set_plan_override(plan)
        ys = [T.row_parallel_forward(X, pv, n, tp, y_dtype=torch.float32, ws=ws) for _ in range(3)]
        for y in ys[1:]:
            assert torch.equal(y, ys[0])
        assert_close(ys[0], O.row_parallel(X.cpu(), V.cpu(), tp)[0], f"plan {plan}")


def test_empty_and_ragged_k(T):
    X = cuda(WL.gen_normal((0, 64), 1.0, 91))
    W = cuda(WL.gen_normal((64, 64), 1.0, 92))
    out = T.column_parallel_forward(X, T.tp_shard_weights(T.KIND_COLUMN, W, 2), T.KIND_COLUMN, 64, 2)
    assert out.shape == (0, 64)
    # k not a multiple of the 64-wide K block, n/tp not a multiple of the tile
    for (m, k, n, tp) in [(3, 200, 80, 2), (129, 72, 40, 1), (257, 136, 24, 3)]:
        X = WL.gen_normal((m, k), 1.0, 93)
        W = WL.gen_normal((k, n), 0.1, 94)
        for plan in (1, 2, 1 | 16):
            T.tps_set_plan_override(plan)
            y = T.column_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_COLUMN, cuda(W), tp), T.KIND_COLUMN,
                                          n, tp, y_dtype=torch.float32, ws=ws_for(T, T.FN_COLUMN, m, n, k, tp))
            assert_close(y, O.column_parallel(X, W, tp)[0], f"col {m},{k},{n},{tp} plan {plan}")
        V = WL.gen_normal((k, n), 0.1, 95)
        if k % tp == 0 and (k // tp) % 8 == 0:
            y = T.row_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_ROW, cuda(V), tp), n, tp,
                                       y_dtype=torch.float32, ws=ws_for(T, T.FN_ROW, m, n, k, tp))
            assert_close(y, O.row_parallel(X, V, tp)[0], f"row {m},{k},{n},{tp}")


def test_errors_on_device_pointers(T):
    X = cuda(WL.gen_normal((4, 64), 1.0, 96))
    W = cuda(WL.gen_normal((64, 256), 1.0, 97))
    pk = T.tp_shard_weights(T.KIND_COLUMN, W, 2)
    with pytest.raises(T.TpsError) as e:
        T.column_parallel_forward(X, pk, T.KIND_COLUMN, 256, 3)
    assert e.value.status == T.TPS_ERR_DIVISIBILITY
    out = torch.empty(4 * 256 + 1, dtype=torch.bfloat16, device="cuda")
    rc = T.lib.column_parallel_forward(X.data_ptr(), 4, 64, pk.data_ptr(), T.KIND_COLUMN, 256, 2, None, None, 0,
                                       out.data_ptr() + 2, 0, None, 0, None)
    assert rc == T.TPS_ERR_ALIGN


def test_bounded_wait_reports_timeout(T):
    """A device wait on a barrier that nothing completes gives up after its limit
    and reports TPS_ERR_TIMEOUT; the context stays usable."""
    T.tps_debug_wait_timeout(2000)
    assert T.tps_device_error() == T.TPS_ERR_TIMEOUT
    assert T.tps_device_error() == T.TPS_OK        # cleared
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def test_status_word_is_per_workspace(T):
    """A bounded wait that runs out on one stream, with its own workspace, is
    reported through that workspace's status word only: a clean GEMM on another
    stream with another workspace reads TPS_OK from its own word (and still
    matches the oracle). The device-wide word sees the failure as well."""
    m, k, n, tp = 48, 1024, 512, 4
    Xc, Vc = WL.gen_normal((m, k), 1.0, 611), WL.gen_normal((k, n), k ** -0.5, 612)
    pv = T.tp_shard_weights(T.KIND_ROW, cuda(Vc), tp)
    X = cuda(Xc)
    ws_bad = ws_for(T, T.FN_ROW, m, n, k, tp)
    ws_ok = ws_for(T, T.FN_ROW, m, n, k, tp)
    s_bad, s_ok = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    T.tps_set_plan_override(2 | 16)   # stream-K: the clean call really uses its workspace
    T.tps_debug_wait_timeout(3000, ws=ws_bad, stream=s_bad)
    with torch.cuda.stream(s_ok):
        Y = T.row_parallel_forward(X, pv, n, tp, y_dtype=torch.float32, ws=ws_ok, stream=s_ok)
    assert T.tps_sync_status(ws_ok, stream=s_ok) == T.TPS_OK
    assert T.tps_sync_status(ws_bad, stream=s_bad) == T.TPS_ERR_TIMEOUT
    assert T.tps_sync_status(ws_bad, stream=s_bad) == T.TPS_OK      # read and cleared
    assert T.tps_device_error() == T.TPS_ERR_TIMEOUT                # the device-wide word saw it too
    torch.cuda.synchronize()
    assert_close(Y, O.row_parallel(Xc, Vc, tp)[0], "clean call beside the failed one")
    assert_ws_state_zero(ws_ok)
    assert_ws_state_zero(ws_bad)


# ============================================================ activation accuracy
def _identity_rows(m, k):
    X = torch.zeros(m, k)
    for i in range(m):
        X[i, i % k] = 1.0
    return X.to(torch.bfloat16)


# token-major, weight-major, and the CTA-pair kernel (256-token tiles, m > 128)
ACT_PLANS = [(1, 64), (2, 64), (1 | 64 | (4 << 8), 200)]


@pytest.mark.parametrize("plan,m", ACT_PLANS)
def test_gelu_epilogue_accuracy(T, plan, m):
    """The fused GELU evaluates erf with Abramowitz & Stegun 7.1.28 (|error| <= 3e-7);
    with X = identity rows the column output is GELU(W) itself, checked element by
    element against the oracle's exact erf form."""
    k, n, tp = 64, 512, 2
    X = _identity_rows(m, k)
    ramp = torch.linspace(-12.0, 12.0, k * n).reshape(k, n).to(torch.bfloat16)
    T.tps_set_plan_override(plan)
    y = T.column_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_COLUMN, cuda(ramp), tp), T.KIND_COLUMN, n, tp,
                                  act=T.ACT_GELU, y_dtype=torch.float32)
    pre = O.linear(X, ramp)
    ref = O.gelu(pre)
    err = np.abs(f64(y) - ref)
    bound = 1e-6 * (1.0 + np.abs(pre))
    assert (err <= bound).all(), float((err / bound).max())


@pytest.mark.parametrize("plan,m", [(1, 64), (2, 64), (1 | 64 | (5 << 8), 200)])
def test_silu_mul_epilogue_accuracy(T, plan, m):
    k, I, tp = 64, 512, 2
    X = _identity_rows(m, k)
    g = torch.linspace(-15.0, 15.0, k * I).reshape(k, I).to(torch.bfloat16)
    u = torch.linspace(0.5, 2.0, k * I).reshape(k, I).to(torch.bfloat16)
    T.tps_set_plan_override(plan)
    h = T.column_parallel_forward(cuda(X), T.tp_shard_weights(T.KIND_GATE_UP, cuda(torch.cat([g, u], 1)), tp),
                                  T.KIND_GATE_UP, 2 * I, tp, act=T.ACT_SILU_MUL, y_dtype=torch.float32)
    G, U = O.linear(X, g), O.linear(X, u)
    ref = O.silu_mul(G, U)
    err = np.abs(f64(h) - ref)
    bound = 1e-6 * (1.0 + np.abs(ref))
    assert (err <= bound).all(), float((err / bound).max())


# ============================================================ attention on local heads
def _qkv_cols(hq, hkv, tp, d=128):
    kvs = hkv // tp if hkv % tp == 0 else 1
    return tp * (hq // tp + 2 * kvs) * d


ATTN_CASES = [  # nseq, S, hq, hkv, tp, causal, std of the q/k/v entries
    (1, 128, 2, 1, 1, True, 1.0),
    (1, 256, 8, 2, 2, True, 1.0),
    (2, 200, 4, 4, 4, True, 1.0),     # two ragged sequences
    (1, 130, 8, 8, 8, False, 1.0),    # ragged, no mask
    (3, 77, 4, 1, 2, True, 1.0),      # KV head replicated on both shards, short sequences
    (1, 1, 2, 1, 1, True, 1.0),       # one token
    (2, 640, 16, 4, 4, True, 1.0),
    (1, 384, 8, 2, 4, False, 1.0),
    (1, 300, 32, 8, 4, True, 3.0),    # the page's 32 heads over tp = 4; peaked softmax (scores ~ N(0, 81))
]


# the attention kernel forms: two 128-query blocks per work item (default) and one
ATTN_FORMS = {"two_tiles": 0, "one_tile": 1 << 27}


@pytest.mark.parametrize("form", list(ATTN_FORMS))
@pytest.mark.parametrize("nseq,S,hq,hkv,tp,causal,std", ATTN_CASES)
def test_gqa_attention_parity(T, nseq, S, hq, hkv, tp, causal, std, form):
    d = 128
    qkv = WL.gen_normal((nseq * S, _qkv_cols(hq, hkv, tp)), std, 101)
    T.tps_set_plan_override(ATTN_FORMS[form])
    A = T.sharded_gqa_attention(cuda(qkv), nseq, S, T.Heads(hq, hkv, d), tp, causal)
    torch.cuda.synchronize()
    assert T.tps_device_error() == T.TPS_OK
    ref = O.gqa_attention_sharded(qkv, hq, hkv, d, tp, nseq, S, causal)
    assert_close(A, ref, "attention")
    A2 = T.sharded_gqa_attention(cuda(qkv), nseq, S, T.Heads(hq, hkv, d), tp, causal)
    assert torch.equal(A, A2)


def test_gqa_attention_full_size(T):
    """The bench's attention: one causal sequence of 2048 tokens, 32 query / 8 KV
    heads of 128, tp = 8, every output element of both kernel forms against the
    oracle."""
    nseq, S, hq, hkv, tp, d = 1, 2048, 32, 8, 8, 128
    qkv = WL.gen_normal((nseq * S, _qkv_cols(hq, hkv, tp)), 1.0, 102)
    ref = O.gqa_attention_sharded(qkv, hq, hkv, d, tp, nseq, S, True)
    for form, ov in ATTN_FORMS.items():
        T.tps_set_plan_override(ov)
        A = T.sharded_gqa_attention(cuda(qkv), nseq, S, T.Heads(hq, hkv, d), tp, True)
        torch.cuda.synchronize()
        assert T.tps_device_error() == T.TPS_OK
        assert_close(A, ref, f"attention ({form})")


def test_gqa_attention_errors(T):
    qkv = torch.zeros(4, _qkv_cols(4, 2, 2), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(T.TpsError) as e:
        T.sharded_gqa_attention(torch.zeros(4, 2 * 4 * 64, dtype=torch.bfloat16, device="cuda"), 1, 4,
                                T.Heads(4, 2, 64), 2)
    assert e.value.status == T.TPS_ERR_UNIMPLEMENTED
    with pytest.raises(T.TpsError) as e:
        T.sharded_gqa_attention(qkv, 1, 4, T.Heads(4, 2, 128), 3)
    assert e.value.status == T.TPS_ERR_DIVISIBILITY
    out = T.sharded_gqa_attention(qkv, 0, 4, T.Heads(4, 2, 128), 2)
    assert out.numel() == 0
