"""The allocation-free row-parallel entry point (row_parallel_forward_noalloc).

Some callers cannot allocate device memory or hand the library a workspace (an
engine running under a fixed memory plan, code that must not call the
allocator); this entry point serves them from a scratch array that lives in the
library. This file checks, through the C ABI, that two calls in a row give the
same output as the fp64 oracle and as row_parallel_forward with a caller
workspace, within the parity tolerance of the other tests, that the forced
split-K plan really runs on the static scratch (stream-K slots and counters),
and that sizes beyond the scratch's limit are rejected. It is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process."""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tensor_sharded_linear_columnparallel_b200 as T
    return T


def _rel(y, ref):
    y, ref = y.double().cpu().numpy(), ref.double().cpu().numpy()
    d = y - ref
    return np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30), np.abs(d).max() / max(np.abs(ref).max(), 1e-30)


# plan override 0 = automatic; 2 | 16 = weight-major tiles with stream-K split
def _ok(fro_mx):
    fro, mx = fro_mx
    return fro <= 5e-3 and mx <= 1e-2


# plan override 0 = automatic; 2 | 16 | (1 << 17) = weight-major tiles with a stream-K
# split (cluster split-K, which needs no scratch, forbidden), whose segment partials
# and tile counters then live in the static scratch
@pytest.mark.parametrize("ov", [0, 2 | 16 | (1 << 17)])
@pytest.mark.parametrize("m,k,n,tp", [(64, 14336, 4096, 8), (8, 14336, 4096, 8), (33, 2048, 512, 4), (1, 512, 128, 2)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(T, m, k, n, tp, ov, capfd, monkeypatch):
    monkeypatch.setenv("TPS_DEBUG_PLAN", "1")   # the planner prints its choice to stderr
    prev = T.tps_set_plan_override(ov)
    try:
        _check_noalloc(T, m, k, n, tp)
    finally:
        T.tps_set_plan_override(prev)
    plans = [ln for ln in capfd.readouterr().err.splitlines() if "static_ws=1" in ln]
    assert plans, "the allocation-free calls were not planned on the static scratch"
    if ov & 16:
        # the forced split-K plan really parks its partials in the static array
        assert all(" sk=1 " in ln for ln in plans), plans


def _check_noalloc(T, m, k, n, tp):
    Xc = WL.gen_normal((m, k), 1.0, 501)
    Vc = WL.gen_normal((k, n), k ** -0.5, 502)
    bc = WL.gen_normal((n,), 0.1, 503)
    X, V, b = Xc.cuda(), Vc.cuda(), bc.cuda()
    oracle, _ = O.row_parallel(Xc, Vc, tp, bc)
    oracle = torch.from_numpy(oracle)
    pv = T.tp_shard_weights(T.KIND_ROW, V, tp)
    ws = T.workspace(T.FN_ROW, m, n, k, tp)
    for ydt in (torch.float32, torch.bfloat16):
        ref = T.row_parallel_forward(X, pv, n, tp, bias=b, y_dtype=ydt, ws=ws)
        assert _ok(_rel(ref, oracle))
        for _ in range(2):                       # two calls in a row share the static scratch
            out = torch.full((m, n), float("nan"), dtype=ydt, device="cuda")
            rc = T.lib.row_parallel_forward_noalloc(X.data_ptr(), m, k, pv.data_ptr(), n, tp, b.data_ptr(),
                                                    out.data_ptr(), T.DTYPE_F32 if ydt == torch.float32 else T.DTYPE_BF16,
                                                    torch.cuda.current_stream().cuda_stream)
            assert rc == T.TPS_OK, T.status_string(rc)
            torch.cuda.synchronize()
            assert torch.isfinite(out).all()
            assert _ok(_rel(out, oracle)), _rel(out, oracle)     # against the fp64 oracle
            assert _ok(_rel(out, ref)), _rel(out, ref)           # and against the workspace entry point
    assert T.tps_device_error() == T.TPS_OK


def test_noalloc_rejects_sizes_beyond_its_scratch(T):
    X = WL.gen_normal((65, 256), 1.0, 504).cuda()
    pv = T.tp_shard_weights(T.KIND_ROW, WL.gen_normal((256, 128), 0.1, 505).cuda(), 2)
    out = torch.empty(65, 128, dtype=torch.bfloat16, device="cuda")
    rc = T.lib.row_parallel_forward_noalloc(X.data_ptr(), 65, 256, pv.data_ptr(), 128, 2, None, out.data_ptr(),
                                            T.DTYPE_BF16, None)
    assert rc == T.TPS_ERR_WORKSPACE
