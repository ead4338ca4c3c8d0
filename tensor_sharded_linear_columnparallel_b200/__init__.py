"""Python binding of libtps.so, the tensor-sharded (column/row-parallel) linear
block for one B200 (sm_100a).

Argument marshalling only: every function below checks tensor dtypes/devices,
allocates outputs with torch when none are given (PyTorch is the device-memory
and stream plumbing), and calls the C entry point of the same name declared in
include/tps.h. Every step of the block's arithmetic runs in the library's CUDA
kernels. There is no fallback: if libtps.so is missing or cannot be loaded,
importing this package raises.

Weights use the math orientation W[k, n] (Y = X W) unless ``transposed=True``.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtps.so")

# ---------------------------------------------------------------- constants (tps.h)
TPS_OK = 0
TPS_ERR_ARG = -1
TPS_ERR_DIVISIBILITY = -2
TPS_ERR_ALIGN = -3
TPS_ERR_DTYPE = -4
TPS_ERR_WORKSPACE = -5
TPS_ERR_CUDA = -6
TPS_ERR_TIMEOUT = -7
TPS_ERR_UNIMPLEMENTED = -8
TPS_ERR_DEVICE = -9

KIND_COLUMN, KIND_ROW, KIND_QKV, KIND_GATE_UP = 0, 1, 2, 3
ACT_NONE, ACT_GELU, ACT_SILU_MUL = 0, 1, 2
DTYPE_BF16, DTYPE_F32 = 0, 1
REDUCE_FUSED, REDUCE_PARTIALS, REDUCE_BF16 = 0, 1, 2
FN_COLUMN, FN_ROW, FN_MLP, FN_ATTN, FN_ARGMAX = 0, 1, 2, 3, 4

PLAN_AUTO, PLAN_TOKEN_MAJOR, PLAN_WEIGHT_MAJOR = 0, 1, 2
PLAN_FORCE_SPLITK, PLAN_NO_SPLITK = 16, 32


def plan_width(cols: int) -> int:
    """Plan-override bits forcing the tile width (16, 32, 64, 128 or 256 columns)."""
    return {16: 1, 32: 2, 64: 3, 128: 4, 256: 5}[cols] << 8

EXPORTED = (
    "tp_head_map", "tp_packed_bytes", "tp_shard_weights", "column_parallel_forward",
    "row_parallel_forward", "shard_partial_reduce", "sharded_mlp_forward",
    "sharded_attn_proj_forward", "tps_workspace_bytes", "tps_status_string",
    "tps_device_error", "tps_set_plan_override", "tps_debug_wait_timeout",
    "row_parallel_forward_noalloc", "vocab_parallel_argmax", "sharded_gqa_attention", "tps_sync_status",
    "shard_partial_reduce_bf16",
)


class TpsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class tps_heads(ctypes.Structure):
    _fields_ = [("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


@dataclass(frozen=True)
class Heads:
    hq: int
    hkv: int
    head_dim: int

    def c(self) -> tps_heads:
        return tps_heads(self.hq, self.hkv, self.head_dim)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python tensor_sharded_linear_columnparallel_b200/build.py` "
            "(there is no CPU or PyTorch fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    HP = ctypes.POINTER(tps_heads)
    I32P = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "tp_head_map": (I, [I, I, I, I32P, I32P, I32P, I32P]),
        "tp_packed_bytes": (SZ, [I, I64, I64, I, HP]),
        "tp_shard_weights": (I, [I, P, I, I64, I64, I, HP, P, SZ, P]),
        "column_parallel_forward": (I, [P, I64, I64, P, I, I64, I, HP, P, I, P, I, P, SZ, P]),
        "row_parallel_forward": (I, [P, I64, I64, P, I64, I, P, I, P, P, I, P, SZ, P]),
        "shard_partial_reduce": (I, [P, I, I64, I64, P, P, I, P]),
        "shard_partial_reduce_bf16": (I, [P, I, I64, I64, P, P, I, P]),
        "sharded_mlp_forward": (I, [P, I64, I64, I64, I, I, P, P, P, P, I, P, SZ, P]),
        "sharded_attn_proj_forward": (I, [P, P, I64, I64, HP, I, P, P, P, P, I, P, SZ, P]),
        "tps_workspace_bytes": (SZ, [I, I64, I64, I64, I]),
        "tps_status_string": (ctypes.c_char_p, [I]),
        "tps_device_error": (I, [P]),
        "tps_set_plan_override": (I, [I]),
        "tps_debug_wait_timeout": (I, [I, P, SZ, P]),
        "tps_sync_status": (I, [P, P]),
        "row_parallel_forward_noalloc": (I, [P, I64, I64, P, I64, I, P, P, I, P]),
        "vocab_parallel_argmax": (I, [P, I64, I64, P, I64, I, P, P, P, SZ, P]),
        "sharded_gqa_attention": (I, [P, I64, I64, HP, I, I, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


# ---------------------------------------------------------------- helpers
def status_string(status: int) -> str:
    return lib.tps_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != TPS_OK:
        raise TpsError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev(t: torch.Tensor, what: str, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t


def _ydtype(dt) -> int:
    if dt in (torch.bfloat16, DTYPE_BF16):
        return DTYPE_BF16
    if dt in (torch.float32, DTYPE_F32):
        return DTYPE_F32
    raise ValueError(f"unsupported output dtype {dt}")


def _torch_dtype(code: int):
    return torch.bfloat16 if code == DTYPE_BF16 else torch.float32


def _heads_ref(heads):
    if heads is None:
        return None
    h = heads.c() if isinstance(heads, Heads) else heads
    return ctypes.byref(h)


# ---------------------------------------------------------------- host-only queries
def tp_head_map(hq: int, hkv: int, tp: int):
    """(q_first, q_count, kv_first, kv_count) lists of length tp."""
    arrs = [(ctypes.c_int32 * tp)() for _ in range(4)]
    _check(lib.tp_head_map(hq, hkv, tp, *arrs), "tp_head_map")
    return tuple(list(a) for a in arrs)


def tp_packed_bytes(kind: int, k: int, n: int, tp: int, heads=None) -> int:
    h = heads.c() if isinstance(heads, Heads) else heads
    return lib.tp_packed_bytes(kind, k, n, tp, ctypes.byref(h) if h is not None else None)


def tps_workspace_bytes(fn: int, m: int, n: int, k: int, tp: int) -> int:
    return lib.tps_workspace_bytes(fn, m, n, k, tp)


def tps_set_plan_override(plan: int) -> int:
    return lib.tps_set_plan_override(plan)


def tps_device_error(stream=None) -> int:
    return lib.tps_device_error(_stream(stream))


def tps_sync_status(ws: torch.Tensor, stream=None) -> int:
    """Status of the calls given workspace `ws` (its status word, read and cleared)."""
    _dev(ws, "ws")
    return lib.tps_sync_status(_ptr(ws), _stream(stream))


def tps_debug_wait_timeout(timeout_us: int, ws: torch.Tensor | None = None, stream=None) -> None:
    _check(lib.tps_debug_wait_timeout(timeout_us, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                      _stream(stream)), "tps_debug_wait_timeout")


def workspace(fn: int, m: int, n: int, k: int, tp: int, device=None) -> torch.Tensor:
    """Zero-filled workspace buffer of tps_workspace_bytes(...) bytes."""
    nbytes = tps_workspace_bytes(fn, m, n, k, tp)
    return torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------- entry points
def tp_shard_weights(kind: int, W: torch.Tensor, tp: int, heads=None, transposed: bool = False,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Packs W (bf16, [k, n], or [n, k] if transposed) into its tp shards."""
    _dev(W, "W", torch.bfloat16)
    if W.dim() != 2:
        raise ValueError("W must be 2-D")
    k, n = (W.shape[1], W.shape[0]) if transposed else (W.shape[0], W.shape[1])
    nbytes = tp_packed_bytes(kind, k, n, tp, heads)
    if nbytes == 0:
        raise TpsError(TPS_ERR_ARG if kind not in (0, 1, 2, 3) else TPS_ERR_DIVISIBILITY, "tp_packed_bytes")
    if out is None:
        out = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=W.device)
    _dev(out, "out")
    _check(lib.tp_shard_weights(kind, _ptr(W), int(transposed), k, n, tp, _heads_ref(heads), _ptr(out),
                                out.numel() * out.element_size(), _stream(stream)), "tp_shard_weights")
    return out


def column_parallel_forward(X: torch.Tensor, packed_w: torch.Tensor, kind: int, n: int, tp: int,
                            heads=None, bias=None, act: int = ACT_NONE, out=None,
                            y_dtype=torch.bfloat16, ws: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """concat_i act(X W_i + b_i); n is the logical column count of the packed weight."""
    _dev(X, "X", torch.bfloat16)
    _dev(packed_w, "packed_w", torch.bfloat16)
    m, k = X.shape
    yd = _ydtype(y_dtype)
    if out is None:
        if kind == KIND_COLUMN:
            n_out = n
        elif kind == KIND_GATE_UP:
            n_out = n // 2
        else:
            _, qc, _, kc = tp_head_map(heads.hq, heads.hkv, tp)
            n_out = tp * (qc[0] + 2 * kc[0]) * heads.head_dim
        out = torch.empty(m, n_out, dtype=_torch_dtype(yd), device=X.device)
    _dev(out, "out")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    _check(lib.column_parallel_forward(_ptr(X), m, k, _ptr(packed_w), kind, n, tp, _heads_ref(heads), _ptr(bias),
                                       act, _ptr(out), yd, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                       _stream(stream)), "column_parallel_forward")
    return out


def row_parallel_forward(X: torch.Tensor, packed_v: torch.Tensor, n: int, tp: int, bias=None,
                         reduce_mode: int = REDUCE_FUSED, partials: torch.Tensor | None = None, out=None,
                         y_dtype=torch.bfloat16, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """sum_i X_i V_i (+ bias once)."""
    _dev(X, "X", torch.bfloat16)
    _dev(packed_v, "packed_v", torch.bfloat16)
    m, k = X.shape
    yd = _ydtype(y_dtype)
    if out is None:
        out = torch.empty(m, n, dtype=_torch_dtype(yd), device=X.device)
    _dev(out, "out")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    if reduce_mode == REDUCE_PARTIALS and partials is None:
        partials = torch.empty(tp, m, n, dtype=torch.float32, device=X.device)
    if partials is not None:
        _dev(partials, "partials", torch.float32)
    _check(lib.row_parallel_forward(_ptr(X), m, k, _ptr(packed_v), n, tp, _ptr(bias), reduce_mode, _ptr(partials),
                                    _ptr(out), yd, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream)), "row_parallel_forward")
    return out


def shard_partial_reduce(partials: torch.Tensor, bias=None, out=None, y_dtype=torch.bfloat16,
                         stream=None, bf16_exchange: bool = False) -> torch.Tensor:
    """Y = sum over dim 0 of partials [tp, m, n] (fp32, shard order) + bias; with
    bf16_exchange, shard_partial_reduce_bf16 (bf16 partials, rounded after every
    addition)."""
    _dev(partials, "partials", torch.float32)
    tp, m, n = partials.shape
    yd = _ydtype(y_dtype)
    if out is None:
        out = torch.empty(m, n, dtype=_torch_dtype(yd), device=partials.device)
    _dev(out, "out")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    fn = lib.shard_partial_reduce_bf16 if bf16_exchange else lib.shard_partial_reduce
    _check(fn(_ptr(partials), tp, m, n, _ptr(bias), _ptr(out), yd, _stream(stream)),
           "shard_partial_reduce_bf16" if bf16_exchange else "shard_partial_reduce")
    return out


def sharded_mlp_forward(X: torch.Tensor, H: int, I: int, tp: int, act: int, packed_up: torch.Tensor,
                        packed_down: torch.Tensor, h_ws=None, out=None, y_dtype=torch.bfloat16,
                        ws: torch.Tensor | None = None, stream=None):
    """MLP block: h = act(column(X)), Y = row(h). Returns (Y, h)."""
    _dev(X, "X", torch.bfloat16)
    m = X.shape[0]
    yd = _ydtype(y_dtype)
    if h_ws is None:
        h_ws = torch.empty(m, I, dtype=torch.bfloat16, device=X.device)
    if out is None:
        out = torch.empty(m, H, dtype=_torch_dtype(yd), device=X.device)
    _dev(h_ws, "h_ws", torch.bfloat16)
    _dev(out, "out")
    _check(lib.sharded_mlp_forward(_ptr(X), m, H, I, tp, act, _ptr(packed_up), _ptr(packed_down), _ptr(h_ws),
                                   _ptr(out), yd, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream)), "sharded_mlp_forward")
    return out, h_ws


def vocab_parallel_argmax(X: torch.Tensor, H: int, V: int, tp: int, packed_w: torch.Tensor,
                          ws: torch.Tensor | None = None, out_idx=None, out_val=None, stream=None):
    """Greedy token per row of X over a vocab-parallel lm_head (COLUMN pack of
    W[H, V]): each shard's local argmax, then the max over shards. Returns
    (indices int32 [m], max logits fp32 [m])."""
    _dev(X, "X", torch.bfloat16)
    m = X.shape[0]
    if ws is None:
        ws = workspace(FN_ARGMAX, m, V, H, tp, device=X.device)
    if out_idx is None:
        out_idx = torch.empty(m, dtype=torch.int32, device=X.device)
    if out_val is None:
        out_val = torch.empty(m, dtype=torch.float32, device=X.device)
    _check(lib.vocab_parallel_argmax(_ptr(X), m, H, _ptr(packed_w), V, tp, _ptr(out_idx), _ptr(out_val), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "vocab_parallel_argmax")
    return out_idx, out_val


def sharded_gqa_attention(qkv: torch.Tensor, nseq: int, seqlen: int, heads: Heads, tp: int, causal: bool = True,
                          out=None, stream=None):
    """Attention on local heads over a QKV-kind column output (shard-major
    [q | k | v] blocks). Returns attn_out [nseq*seqlen, hq*d] bf16, query head h
    at columns [h*d, (h+1)*d)."""
    _dev(qkv, "qkv", torch.bfloat16)
    m = nseq * seqlen
    if out is None:
        out = torch.empty(m, heads.hq * heads.head_dim, dtype=torch.bfloat16, device=qkv.device)
    _dev(out, "out", torch.bfloat16)
    _check(lib.sharded_gqa_attention(_ptr(qkv), nseq, seqlen, _heads_ref(heads), tp, 1 if causal else 0, _ptr(out),
                                     _stream(stream)), "sharded_gqa_attention")
    return out


def sharded_attn_proj_forward(X: torch.Tensor, attn_out: torch.Tensor, H: int, heads: Heads, tp: int,
                              packed_qkv: torch.Tensor, packed_o: torch.Tensor, qkv_out=None, out=None,
                              y_dtype=torch.bfloat16, ws: torch.Tensor | None = None, stream=None):
    """QKV (column by head) and o_proj (row by head). Returns (Y, qkv_out)."""
    _dev(X, "X", torch.bfloat16)
    _dev(attn_out, "attn_out", torch.bfloat16)
    m = X.shape[0]
    yd = _ydtype(y_dtype)
    if qkv_out is None:
        _, qc, _, kc = tp_head_map(heads.hq, heads.hkv, tp)
        qkv_out = torch.empty(m, tp * (qc[0] + 2 * kc[0]) * heads.head_dim, dtype=torch.bfloat16, device=X.device)
    if out is None:
        out = torch.empty(m, H, dtype=_torch_dtype(yd), device=X.device)
    _dev(qkv_out, "qkv_out", torch.bfloat16)
    _dev(out, "out")
    _check(lib.sharded_attn_proj_forward(_ptr(X), _ptr(attn_out), m, H, _heads_ref(heads), tp, _ptr(packed_qkv),
                                         _ptr(packed_o), _ptr(qkv_out), _ptr(out), yd, _ptr(ws),
                                         0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "sharded_attn_proj_forward")
    return out, qkv_out


def row_parallel_forward_noalloc(X: torch.Tensor, packed_v: torch.Tensor, n: int, tp: int, bias=None, out=None,
                                 y_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """row_parallel_forward for callers that cannot provide a workspace: the
    split-K scratch is the library's own static device array (m <= 64 tokens;
    concurrent calls on unordered streams race on it)."""
    _dev(X, "X", torch.bfloat16)
    _dev(packed_v, "packed_v", torch.bfloat16)
    m, k = X.shape
    yd = _ydtype(y_dtype)
    if out is None:
        out = torch.empty(m, n, dtype=_torch_dtype(yd), device=X.device)
    _dev(out, "out")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    _check(lib.row_parallel_forward_noalloc(_ptr(X), m, k, _ptr(packed_v), n, tp, _ptr(bias), _ptr(out), yd,
                                            _stream(stream)), "row_parallel_forward_noalloc")
    return out
