"""The allocation-free row-parallel entry point (row_parallel_forward_noalloc).

Some callers cannot allocate device memory or hand the library a workspace (an
engine running under a fixed memory plan, code that must not call the
allocator); this entry point serves them from a scratch array that lives in the
library. This file checks, through the C ABI, that two calls in a row give the
same output as row_parallel_forward with a caller workspace, within the parity
tolerance of the other tests, and that sizes beyond the scratch's limit are
rejected. It is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process."""

import numpy as np
import pytest
import torch

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
@pytest.mark.parametrize("ov", [0, 2 | 16])
@pytest.mark.parametrize("m,k,n,tp", [(64, 14336, 4096, 8), (8, 14336, 4096, 8), (33, 2048, 512, 4), (1, 512, 128, 2)])
def test_noalloc_matches_workspace_entry_point_twice(T, m, k, n, tp, ov):
    prev = T.tps_set_plan_override(ov)
    try:
        _check_noalloc(T, m, k, n, tp)
    finally:
        T.tps_set_plan_override(prev)


def _check_noalloc(T, m, k, n, tp):
    X = WL.gen_normal((m, k), 1.0, 501).cuda()
    V = WL.gen_normal((k, n), k ** -0.5, 502).cuda()
    b = WL.gen_normal((n,), 0.1, 503).cuda()
    pv = T.tp_shard_weights(T.KIND_ROW, V, tp)
    ws = T.workspace(T.FN_ROW, m, n, k, tp)
    for ydt in (torch.float32, torch.bfloat16):
        ref = T.row_parallel_forward(X, pv, n, tp, bias=b, y_dtype=ydt, ws=ws)
        for _ in range(2):                       # two calls in a row share the static scratch
            out = torch.full((m, n), float("nan"), dtype=ydt, device="cuda")
            rc = T.lib.row_parallel_forward_noalloc(X.data_ptr(), m, k, pv.data_ptr(), n, tp, b.data_ptr(),
                                                    out.data_ptr(), T.DTYPE_F32 if ydt == torch.float32 else T.DTYPE_BF16,
                                                    torch.cuda.current_stream().cuda_stream)
            assert rc == T.TPS_OK, T.status_string(rc)
            torch.cuda.synchronize()
            assert torch.isfinite(out).all()
            fro, mx = _rel(out, ref)
            assert fro <= 5e-3 and mx <= 1e-2, (fro, mx)
    assert T.tps_device_error() == T.TPS_OK


def test_noalloc_rejects_sizes_beyond_its_scratch(T):
    X = WL.gen_normal((65, 256), 1.0, 504).cuda()
    pv = T.tp_shard_weights(T.KIND_ROW, WL.gen_normal((256, 128), 0.1, 505).cuda(), 2)
    out = torch.empty(65, 128, dtype=torch.bfloat16, device="cuda")
    rc = T.lib.row_parallel_forward_noalloc(X.data_ptr(), 65, 256, pv.data_ptr(), 128, 2, None, out.data_ptr(),
                                            T.DTYPE_BF16, None)
    assert rc == T.TPS_ERR_WORKSPACE
