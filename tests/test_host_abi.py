"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol declared in include/tps.h, and its host logic (head map, packed sizes,
workspace bound, argument validation) behaves as documented. No call here
launches a kernel."""

import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tps.h")


def _tps():
    import tensor_sharded_linear_columnparallel_b200 as T
    return T


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^TPS_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_six_entry_points():
    names = declared_functions()
    for n in ("tp_shard_weights", "column_parallel_forward", "row_parallel_forward",
              "shard_partial_reduce", "sharded_mlp_forward", "sharded_attn_proj_forward"):
        assert n in names


def test_library_exports_every_declared_symbol():
    T = _tps()
    lib = ctypes.CDLL(T.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(T.EXPORTED)


def test_status_strings():
    T = _tps()
    for code in range(-9, 1):
        s = T.status_string(code)
        assert s.startswith("TPS_") and "UNKNOWN" not in s
    assert "UNKNOWN" in T.status_string(-100)


@pytest.mark.parametrize("hq,hkv,tp", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (32, 8, 16),
                                       (32, 32, 4), (64, 8, 8), (64, 8, 16), (64, 8, 64), (12, 4, 12),
                                       (12, 4, 2), (8, 1, 8)])
def test_head_map_matches_oracle(hq, hkv, tp):
    T = _tps()
    qf, qc, kf, kc = T.tp_head_map(hq, hkv, tp)
    q_heads, kv_heads = O.head_map(hq, hkv, tp)
    assert [list(range(qf[r], qf[r] + qc[r])) for r in range(tp)] == q_heads
    assert [list(range(kf[r], kf[r] + kc[r])) for r in range(tp)] == kv_heads


@pytest.mark.parametrize("hq,hkv,tp", [(32, 8, 3), (32, 8, 0), (12, 8, 4), (32, 12, 8), (24, 8, 16)])
def test_head_map_rejects(hq, hkv, tp):
    T = _tps()
    a = [(ctypes.c_int32 * max(tp, 1))() for _ in range(4)]
    rc = T.lib.tp_head_map(hq, hkv, tp, *a)
    assert rc in (T.TPS_ERR_DIVISIBILITY, T.TPS_ERR_ARG)


def test_packed_bytes():
    T = _tps()
    assert T.tp_packed_bytes(T.KIND_COLUMN, 64, 256, 2) == 64 * 256 * 2
    # ROW: R = 64 rows padded to one 128-row block, K/tp = 128 = 2 K blocks
    assert T.tp_packed_bytes(T.KIND_ROW, 256, 64, 2) == 2 * 128 * 128 * 2
    assert T.tp_packed_bytes(T.KIND_COLUMN, 72, 80, 2) == 2 * 128 * 128 * 2     # 40 rows, 72 K -> padded
    h = T.Heads(32, 8, 128)
    # tp=16: 2 q heads + 1 k + 1 v head per shard -> 512 rows per shard (KV replicated)
    assert T.tp_packed_bytes(T.KIND_QKV, 4096, (32 + 16) * 128, 16, h) == 16 * 512 * 4096 * 2
    assert T.tp_packed_bytes(T.KIND_QKV, 4096, (32 + 16) * 128, 8, h) == 8 * 768 * 4096 * 2
    # gate/up, I/tp = 1792 = 14 blocks of 128 -> no padding
    assert T.tp_packed_bytes(T.KIND_GATE_UP, 4096, 2 * 14336, 8) == 2 * 14336 * 4096 * 2
    # I/tp = 200 -> 2 blocks of 2x128 rows (zero padded)
    assert T.tp_packed_bytes(T.KIND_GATE_UP, 64, 2 * 400, 2) == 2 * 512 * 64 * 2
    assert T.tp_packed_bytes(T.KIND_COLUMN, 64, 250, 2) == 0       # 125 per shard, not a multiple of 8
    assert T.tp_packed_bytes(T.KIND_COLUMN, 64, 256, 3) == 0       # not divisible
    assert T.tp_packed_bytes(9, 64, 256, 2) == 0


def test_workspace_bound_positive():
    T = _tps()
    assert T.tps_workspace_bytes(T.FN_ROW, 512, 1024, 4096, 8) >= 2 * 148 * 128 * 1024
    assert T.tps_workspace_bytes(T.FN_ROW, 0, 1024, 4096, 8) > 0
    assert T.tps_workspace_bytes(7, 1, 1, 1, 1) == 0


def test_validation_happens_before_any_cuda_call():
    """Invalid arguments return their status without touching a device (this box has none)."""
    T = _tps()
    lib = T.lib
    good = 1 << 20                 # 16-B aligned fake addresses: never dereferenced on the host
    h = T.tps_heads(32, 8, 128)
    # divisibility
    assert lib.column_parallel_forward(good, 4, 64, good, T.KIND_COLUMN, 256, 3, None, None, 0, good, 0,
                                       None, 0, None) == T.TPS_ERR_DIVISIBILITY
    assert lib.row_parallel_forward(good, 4, 64, good, 64, 3, None, 0, None, good, 0, None, 0,
                                    None) == T.TPS_ERR_DIVISIBILITY
    assert lib.column_parallel_forward(good, 4, 4096, good, T.KIND_QKV, 48 * 128, 3, ctypes.byref(h), None, 0,
                                       good, 0, None, 0, None) == T.TPS_ERR_DIVISIBILITY
    # alignment
    assert lib.column_parallel_forward(good + 2, 4, 64, good, T.KIND_COLUMN, 256, 2, None, None, 0, good, 0,
                                       None, 0, None) == T.TPS_ERR_ALIGN
    assert lib.column_parallel_forward(good, 4, 60, good, T.KIND_COLUMN, 256, 2, None, None, 0, good, 0,
                                       None, 0, None) == T.TPS_ERR_ALIGN
    # bad enums / combinations
    assert lib.column_parallel_forward(good, 4, 64, good, T.KIND_COLUMN, 256, 2, None, None,
                                       T.ACT_SILU_MUL, good, 0, None, 0, None) == T.TPS_ERR_ARG
    assert lib.column_parallel_forward(good, 4, 64, good, T.KIND_COLUMN, 256, 2, None, None, 0, good, 7,
                                       None, 0, None) == T.TPS_ERR_DTYPE
    assert lib.row_parallel_forward(good, 4, 64, good, 64, 2, None, 5, None, good, 0, None, 0,
                                    None) == T.TPS_ERR_ARG
    assert lib.row_parallel_forward(good, 4, 64, good, 64, 2, None, T.REDUCE_PARTIALS, None, good, 0, None, 0,
                                    None) == T.TPS_ERR_ARG
    assert lib.column_parallel_forward(None, 4, 64, good, T.KIND_COLUMN, 256, 2, None, None, 0, good, 0,
                                       None, 0, None) == T.TPS_ERR_ARG
    assert lib.shard_partial_reduce(good, 2, 4, 6, None, good, 0, None) == T.TPS_ERR_ALIGN
    assert lib.tp_shard_weights(T.KIND_ROW, good, 0, 64, 256, 3, None, good, 1 << 30, None) == T.TPS_ERR_DIVISIBILITY
    assert lib.tp_shard_weights(T.KIND_ROW, good, 0, 64, 256, 2, None, good, 16, None) == T.TPS_ERR_WORKSPACE
    assert lib.tps_debug_wait_timeout(0, None, 0, None) == T.TPS_ERR_ARG
    assert lib.tps_debug_wait_timeout(1000, good, 128, None) == T.TPS_ERR_WORKSPACE   # smaller than the header
    assert lib.tps_sync_status(None, None) == T.TPS_ERR_ARG
    # m = 0 is a valid empty problem: returns OK without any CUDA call
    assert lib.column_parallel_forward(good, 0, 64, good, T.KIND_COLUMN, 256, 2, None, None, 0, good, 0,
                                       None, 0, None) == T.TPS_OK
    assert lib.row_parallel_forward(good, 0, 64, good, 64, 2, None, 0, None, good, 0, None, 0,
                                    None) == T.TPS_OK


def test_plan_override_roundtrip():
    T = _tps()
    prev = T.tps_set_plan_override(T.PLAN_WEIGHT_MAJOR | T.PLAN_FORCE_SPLITK)
    assert T.tps_set_plan_override(prev) == T.PLAN_WEIGHT_MAJOR | T.PLAN_FORCE_SPLITK


def test_attention_and_argmax_validation_before_any_cuda_call():
    """The two later entry points check their arguments on the host first."""
    T = _tps()
    lib = T.lib
    good = 1 << 20
    hd = T.tps_heads(32, 8, 128)
    # sharded_gqa_attention(qkv, nseq, seqlen, heads, tp, causal, attn_out, stream)
    assert lib.sharded_gqa_attention(good, 1, 16, None, 8, 1, good, None) == T.TPS_ERR_ARG
    assert lib.sharded_gqa_attention(good, 1, 16, ctypes.byref(hd), 3, 1, good, None) == T.TPS_ERR_DIVISIBILITY
    assert lib.sharded_gqa_attention(good, 1, 16, ctypes.byref(T.tps_heads(32, 8, 64)), 8, 1, good,
                                     None) == T.TPS_ERR_UNIMPLEMENTED
    assert lib.sharded_gqa_attention(good, 1, 16, ctypes.byref(hd), 8, 2, good, None) == T.TPS_ERR_ARG
    assert lib.sharded_gqa_attention(good, -1, 16, ctypes.byref(hd), 8, 1, good, None) == T.TPS_ERR_ARG
    assert lib.sharded_gqa_attention(None, 1, 16, ctypes.byref(hd), 8, 1, good, None) == T.TPS_ERR_ARG
    assert lib.sharded_gqa_attention(good + 8, 1, 16, ctypes.byref(hd), 8, 1, good, None) == T.TPS_ERR_ALIGN
    assert lib.sharded_gqa_attention(good, 0, 16, ctypes.byref(hd), 8, 1, good, None) == T.TPS_OK
    assert lib.sharded_gqa_attention(None, 3, 0, ctypes.byref(hd), 8, 1, None, None) == T.TPS_OK
    # vocab_parallel_argmax(X, m, H, packed_w, V, tp, out_idx, out_val, ws, ws_bytes, stream)
    need = T.tps_workspace_bytes(T.FN_ARGMAX, 64, 128256, 4096, 8)
    assert need >= 64 * 8 * 8 * (128256 // 8 // 128)
    assert lib.vocab_parallel_argmax(good, 64, 4096, good, 100, 3, good, good, good, need,
                                     None) == T.TPS_ERR_DIVISIBILITY
    assert lib.vocab_parallel_argmax(good, -1, 4096, good, 128256, 8, good, good, good, need, None) == T.TPS_ERR_ARG
    assert lib.vocab_parallel_argmax(good, 64, 4096, good, 128256, 8, None, good, good, need, None) == T.TPS_ERR_ARG
    assert lib.vocab_parallel_argmax(good + 4, 64, 4096, good, 128256, 8, good, good, good, need,
                                     None) == T.TPS_ERR_ALIGN
    assert lib.vocab_parallel_argmax(good, 64, 4096, good, 128256, 8, good, good, good, need - 8,
                                     None) == T.TPS_ERR_WORKSPACE
    assert lib.vocab_parallel_argmax(good, 0, 4096, good, 128256, 8, good, good, good, 0, None) == T.TPS_OK


def test_plain_c_client_compiles_links_and_runs(tmp_path):
    """A C99 program that includes only include/tps.h and links libtps.so calls the
    host-only entry points (head map, packed sizes, workspace bound, status strings,
    argument validation)."""
    import shutil
    import subprocess
    T = _tps()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "host_calls"
    libdir = os.path.dirname(T.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "host_calls.c"), T.LIB_PATH, f"-Wl,-rpath,{libdir}",
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("all ok")
