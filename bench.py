#!/usr/bin/env python
"""Benchmark of the tensor-sharded linear block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--tp TP] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
the column-parallel GEMM with its fused activation epilogue, then the
row-parallel GEMM with the cross-shard reduction fused into it (for the 70B
layer: QKV, o_proj, gate/up and down). Packing the weights is start-up work
(weights are split once) and is not timed. Inputs are resident in HBM before
the timed region; the L2 is flushed between timed steps and
every step is bracketed by CUDA events on the launching stream. The flush writes
a 512 MiB buffer and then reads it back, so the L2 holds only clean lines of the
flush buffer when a step starts (no write-back of the flush inside the timed step). With N > 1
(one process per GPU under torchrun) every rank runs its own replica of the
workload: the block emulates all tp shards on one GPU, so nothing crosses GPUs
and the scaling is weak; the reported time is the max over ranks.

`--impl reference` times the CPU fp64 oracle (the only other program this
file may run) on the host cores, on a bounded sample of the same workload.
One JSON line is printed by rank 0.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FUSED_MLP_OVERRIDE = 1 << 18   # plan-override bit: the one-launch MLP kernel (an error if it cannot run)
METRIC = "sharded linear-block TFLOP/s (prefill) and weight-stream GB/s (decode), 1 B200"
L2_BYTES = 126 << 20          # B200 L2
E2E_BUFS = 4                  # device buffers per input / output in the pipelined end-to-end run
FLUSH_BYTES = 512 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# Device-code files each workload's kernels are compiled from (a change elsewhere,
# e.g. a new kernel or launcher in another file, leaves these kernels unchanged).
KERNEL_SOURCES = {
    "gelu_mlp": ("tps_mlp.cuh", "tps_gemm.cuh", "tps_ptx.cuh"),
    "gated_decode": ("tps_mlp_sk.cuh", "tps_mlp.cuh", "tps_gemm.cuh", "tps_ptx.cuh"),
    "gqa_proj": ("tps_gemm.cuh", "tps_gemm2.cuh", "tps_ptx.cuh"),
    "layer70b": ("tps_gemm.cuh", "tps_gemm2.cuh", "tps_ptx.cuh"),
    "lm_head_greedy": ("tps_gemm.cuh", "tps_ptx.cuh", "tps_kernels.cu"),   # the reduce over shards is in tps_kernels.cu
    "gqa_attention": ("tps_attn.cuh", "tps_gemm.cuh", "tps_ptx.cuh"),
}


def kernel_source_hash(workload: str) -> str:
    """Hash of the code (comments and blank lines removed) of the files the
    workload's kernels are compiled from, which ties a committed ncu traffic figure
    to the kernels it was measured on."""
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[workload]:
        with open(os.path.join(ROOT, "tensor_sharded_linear_columnparallel_b200", "csrc", f)) as fh:
            text = re.sub(r"//[^\n]*", "", fh.read())
        h.update("\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip()).encode())
    return h.hexdigest()[:16]


# ============================================================ workloads
def workload_spec(name: str, tp: int | None, m: int | None):
    """Static description of a bench workload (shapes, units, kernel list)."""
    if name == "gelu_mlp":
        m = m or 512
        tp = tp or 8
        H, I = 1024, 4096
        f1 = 2.0 * m * H * I
        return dict(name=name, m=m, tp=tp, H=H, I=I, unit="TFLOP/s", bound="tensor",
                    step_units=2 * f1,
                    kernels=[("column fc1+GELU", f1), ("row fc2+reduce", f1)],
                    label=f"Megatron GELU MLP H={H} I={I} m={m} tp={tp}")
    if name == "gated_decode":
        m = m or 64
        tp = tp or 8
        H, I = 4096, 14336
        wb = 2.0 * H * I * 2
        xb = m * H * 2.0
        return dict(name=name, m=m, tp=tp, H=H, I=I, unit="GB/s", bound="hbm",
                    step_units=wb + H * I * 2.0 + 2 * xb,
                    kernels=[("gate/up+SiLU*up", wb + xb), ("down+reduce", H * I * 2.0 + xb)],
                    label=f"gated MLP decode H={H} I={I} m={m} tp={tp}")
    if name == "gqa_proj":
        m = m or 2048
        tp = tp or 8
        H, hq, hkv, d = 4096, 32, 8, 128
        fq = 2.0 * m * H * (hq + 2 * hkv) * d
        fo = 2.0 * m * hq * d * H
        return dict(name=name, m=m, tp=tp, H=H, hq=hq, hkv=hkv, d=d, unit="TFLOP/s", bound="tensor",
                    step_units=fq + fo,
                    kernels=[("QKV column by head", fq), ("o_proj row+reduce", fo)],
                    label=f"GQA projections H={H} hq={hq} hkv={hkv} d={d} m={m} tp={tp}")
    if name == "layer70b":
        m = m or 8192
        tp = tp or 8
        H, I, hq, hkv, d = 8192, 28672, 64, 8, 128
        fq = 2.0 * m * H * (hq + 2 * hkv) * d
        fo = 2.0 * m * hq * d * H
        fgu = 2.0 * m * H * 2 * I
        fd = 2.0 * m * I * H
        return dict(name=name, m=m, tp=tp, H=H, I=I, hq=hq, hkv=hkv, d=d, unit="TFLOP/s", bound="tensor",
                    step_units=fq + fo + fgu + fd,
                    kernels=[("QKV column by head", fq), ("o_proj row+reduce", fo),
                             ("gate/up+SiLU*up", fgu), ("down+reduce", fd)],
                    label=f"70B-layer linears H={H} I={I} hq={hq} hkv={hkv} d={d} m={m} tp={tp}")
    if name == "lm_head_greedy":
        m = m or 64
        tp = tp or 8
        H, V = 4096, 128256
        wb = 2.0 * H * V
        return dict(name=name, m=m, tp=tp, H=H, V=V, unit="GB/s", bound="hbm",
                    step_units=wb + m * H * 2.0 + m * 8.0,
                    kernels=[("lm_head GEMM with shard argmax epilogue + max over shards", wb + m * H * 2.0 + m * 8.0)],
                    label=f"vocab-parallel lm_head greedy H={H} V={V} m={m} tp={tp}")
    if name == "gqa_attention":
        nseq, S = 1, (m or 2048)
        tp = tp or 8
        hq, hkv, d = 32, 8, 128
        flops = 4.0 * d * hq * nseq * S * (S + 1) / 2   # QK^T and PV over the visible (causal) pairs
        return dict(name=name, m=nseq * S, nseq=nseq, S=S, tp=tp, hq=hq, hkv=hkv, d=d, unit="TFLOP/s",
                    bound="tensor", step_units=flops, kernels=[("attention on local heads (causal)", flops)],
                    label=f"causal GQA attention on local heads S={S} hq={hq} hkv={hkv} d={d} tp={tp}")
    raise SystemExit(f"unknown workload {name}")


class GpuStep:
    """Device tensors, packed weights and the launches of one step."""

    def __init__(self, spec, device):
        import torch
        import tensor_sharded_linear_columnparallel_b200 as T
        import workloads as WL
        self.T, self.torch, self.spec = T, torch, spec
        tp, m = spec["tp"], spec["m"]
        name = spec["name"]
        cuda = lambda t: t.to(device).contiguous()  # noqa: E731
        self.bufs = {}
        if name == "gelu_mlp":
            wl = WL.gelu_mlp(m=m)
            t = wl.tensors
            self.X = cuda(t["X"])
            self.p_up = T.tp_shard_weights(T.KIND_COLUMN, cuda(t["W1"]), tp)
            self.p_down = T.tp_shard_weights(T.KIND_ROW, cuda(t["W2"]), tp)
            self.h = torch.empty(m, spec["I"], dtype=torch.bfloat16, device=device)
            self.Y = torch.empty(m, spec["H"], dtype=torch.bfloat16, device=device)
            self.ws = T.workspace(T.FN_MLP, m, spec["H"], spec["I"], tp, device=device)
            self.act, self.kind_up, self.n_up = T.ACT_GELU, T.KIND_COLUMN, spec["I"]
        elif name == "gated_decode":
            wl = WL.gated_decode(m_max=max(m, 1))
            t = wl.tensors
            self.X = cuda(t["X"][:m])
            Wgu = torch.cat([t["Wg"], t["Wu"]], dim=1)
            self.p_up = T.tp_shard_weights(T.KIND_GATE_UP, cuda(Wgu), tp)
            del Wgu
            self.p_down = T.tp_shard_weights(T.KIND_ROW, cuda(t["Wd"]), tp)
            self.h = torch.empty(m, spec["I"], dtype=torch.bfloat16, device=device)
            self.Y = torch.empty(m, spec["H"], dtype=torch.bfloat16, device=device)
            self.ws = T.workspace(T.FN_MLP, m, spec["H"], spec["I"], tp, device=device)
            self.act, self.kind_up, self.n_up = T.ACT_SILU_MUL, T.KIND_GATE_UP, 2 * spec["I"]
        elif name in ("gqa_proj", "layer70b"):
            wl = WL.gqa_proj(m=m) if name == "gqa_proj" else WL.layer70b(m=m)
            t = wl.tensors
            self.heads = T.Heads(spec["hq"], spec["hkv"], spec["d"])
            self.X = cuda(t["X"])
            self.A = cuda(t["A"])
            Wqkv = torch.cat([t["Wq"], t["Wk"], t["Wv"]], dim=1)
            self.p_qkv = T.tp_shard_weights(T.KIND_QKV, cuda(Wqkv), tp, heads=self.heads)
            del Wqkv
            self.p_o = T.tp_shard_weights(T.KIND_ROW, cuda(t["Wo"]), tp)
            qf, qc, kf, kc = T.tp_head_map(spec["hq"], spec["hkv"], tp)
            self.n_qkv = (spec["hq"] + 2 * spec["hkv"]) * spec["d"]
            self.qkv = torch.empty(m, tp * (qc[0] + 2 * kc[0]) * spec["d"], dtype=torch.bfloat16, device=device)
            self.Y = torch.empty(m, spec["H"], dtype=torch.bfloat16, device=device)
            self.ws = T.workspace(T.FN_MLP if name == "layer70b" else T.FN_ATTN, m, spec["H"],
                                  spec.get("I", spec["hq"] * spec["d"]), tp, device=device)
            if name == "layer70b":
                Wgu = torch.cat([t["Wg"], t["Wu"]], dim=1)
                self.p_up = T.tp_shard_weights(T.KIND_GATE_UP, cuda(Wgu), tp)
                del Wgu
                self.p_down = T.tp_shard_weights(T.KIND_ROW, cuda(t["Wd"]), tp)
                self.h = torch.empty(m, spec["I"], dtype=torch.bfloat16, device=device)
                self.Y2 = torch.empty(m, spec["H"], dtype=torch.bfloat16, device=device)
        if name == "gqa_attention":
            qf, qc, kf, kc = T.tp_head_map(spec["hq"], spec["hkv"], tp)
            wl = WL.gqa_attention(tp * (qc[0] + 2 * kc[0]) * spec["d"], nseq=spec["nseq"], S=spec["S"])
            self.heads = T.Heads(spec["hq"], spec["hkv"], spec["d"])
            self.X = cuda(wl.tensors["qkv"])
            self.Y = torch.empty(m, spec["hq"] * spec["d"], dtype=torch.bfloat16, device=device)
            self.ws = torch.zeros(16, dtype=torch.uint8, device=device)   # the attention takes no workspace
        if name == "lm_head_greedy":
            wl = WL.lm_head(m_max=max(m, 1))
            t = wl.tensors
            self.X = cuda(t["X"][:m])
            self.p_w = T.tp_shard_weights(T.KIND_COLUMN, cuda(t["W"]), tp)
            self.Y = torch.empty(m, dtype=torch.int32, device=device)   # greedy token ids
            self.val = torch.empty(m, dtype=torch.float32, device=device)
            self.ws = T.workspace(T.FN_ARGMAX, m, spec["V"], spec["H"], tp, device=device)
        del wl
        self._bind()
        torch.cuda.synchronize()

    # Each launcher calls the C entry points directly with argument tuples built
    # once (the same calls the binding makes, without its per-call checks), so
    # the host stays ahead of the GPU. `ev` (optional) gets an event recorded
    # after every kernel so the per-kernel device time is known.
    def _bind(self):
        T, s, torch = self.T, self.spec, self.torch
        st = torch.cuda.current_stream().cuda_stream
        wsb = self.ws.numel()
        name = s["name"]
        calls = []
        self.fused = False
        self.kernels_per_step = None
        if name == "gqa_attention":
            import ctypes
            self._hc = self.heads.c()
            calls.append((T.lib.sharded_gqa_attention,
                          (self.X.data_ptr(), s["nseq"], s["S"], ctypes.byref(self._hc), s["tp"], 1,
                           self.Y.data_ptr(), st)))
            self.calls = calls
            return
        if name == "lm_head_greedy":
            calls.append((T.lib.vocab_parallel_argmax,
                          (self.X.data_ptr(), s["m"], s["H"], self.p_w.data_ptr(), s["V"], s["tp"],
                           self.Y.data_ptr(), self.val.data_ptr(), self.ws.data_ptr(), wsb, st)))
            self.calls = calls
            self.kernels_per_step = 2   # the GEMM with the argmax epilogue and the reduce over shards
            return
        if name in ("gelu_mlp", "gated_decode"):
            # the MLP entry point runs the whole block as one kernel when the shape
            # allows it (every cluster of its row phase resident); a forced probe
            # call tells which path the step takes
            a = (self.X.data_ptr(), s["m"], s["H"], s["I"], s["tp"], self.act, self.p_up.data_ptr(),
                 self.p_down.data_ptr(), self.h.data_ptr(), self.Y.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb,
                 st)
            prev = T.tps_set_plan_override(FUSED_MLP_OVERRIDE)
            rc = T.lib.sharded_mlp_forward(*a)
            T.tps_set_plan_override(prev)
            self.torch.cuda.synchronize()
            if rc == 0:
                self.fused = True
                calls.append((T.lib.sharded_mlp_forward, a))
        if self.fused:
            pass
        elif name in ("gelu_mlp", "gated_decode"):
            calls.append((T.lib.column_parallel_forward,
                          (self.X.data_ptr(), s["m"], s["H"], self.p_up.data_ptr(), self.kind_up, self.n_up, s["tp"],
                           None, None, self.act, self.h.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st)))
            calls.append((T.lib.row_parallel_forward,
                          (self.h.data_ptr(), s["m"], s["I"], self.p_down.data_ptr(), s["H"], s["tp"], None,
                           T.REDUCE_FUSED, None, self.Y.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st)))
        else:
            self._heads_c = self.heads.c()
            import ctypes
            calls.append((T.lib.column_parallel_forward,
                          (self.X.data_ptr(), s["m"], s["H"], self.p_qkv.data_ptr(), T.KIND_QKV, self.n_qkv, s["tp"],
                           ctypes.byref(self._heads_c), None, T.ACT_NONE, self.qkv.data_ptr(), T.DTYPE_BF16,
                           self.ws.data_ptr(), wsb, st)))
            calls.append((T.lib.row_parallel_forward,
                          (self.A.data_ptr(), s["m"], s["hq"] * s["d"], self.p_o.data_ptr(), s["H"], s["tp"], None,
                           T.REDUCE_FUSED, None, self.Y.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st)))
            if name == "layer70b":
                calls.append((T.lib.column_parallel_forward,
                              (self.X.data_ptr(), s["m"], s["H"], self.p_up.data_ptr(), T.KIND_GATE_UP, 2 * s["I"],
                               s["tp"], None, None, T.ACT_SILU_MUL, self.h.data_ptr(), T.DTYPE_BF16,
                               self.ws.data_ptr(), wsb, st)))
                calls.append((T.lib.row_parallel_forward,
                              (self.h.data_ptr(), s["m"], s["I"], self.p_down.data_ptr(), s["H"], s["tp"], None,
                               T.REDUCE_FUSED, None, self.Y2.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st)))
        self.calls = calls

    def variant_calls(self):
        """The block's variants on the same buffers: row layers with the reduction
        fused into the GEMM, with fp32 partials and the standalone reduce kernel, or
        with the partials exchanged in bf16; for the MLPs also the one-launch kernel."""
        T, s, torch = self.T, self.spec, self.torch
        st = torch.cuda.current_stream().cuda_stream
        wsb = self.ws.numel()
        name = s["name"]
        self.variant_overrides = {}
        if name == "gqa_attention":
            # the kernel with one 128-query block per work item (plan-override bit 27)
            self.variant_overrides["one_query_block_per_item"] = 1 << 27
            return {"one_query_block_per_item": list(self.calls)}
        if name in ("layer70b", "lm_head_greedy"):
            return {}
        if name in ("gelu_mlp", "gated_decode"):
            col = (T.lib.column_parallel_forward,
                   (self.X.data_ptr(), s["m"], s["H"], self.p_up.data_ptr(), self.kind_up, self.n_up, s["tp"], None,
                    None, self.act, self.h.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st))
            rin, k_in, p_row = self.h, s["I"], self.p_down
        else:
            import ctypes
            self._heads_c = self.heads.c()
            col = (T.lib.column_parallel_forward,
                   (self.X.data_ptr(), s["m"], s["H"], self.p_qkv.data_ptr(), T.KIND_QKV, self.n_qkv, s["tp"],
                    ctypes.byref(self._heads_c), None, T.ACT_NONE, self.qkv.data_ptr(), T.DTYPE_BF16,
                    self.ws.data_ptr(), wsb, st))
            rin, k_in, p_row = self.A, s["hq"] * s["d"], self.p_o
        self.partials = torch.empty(s["tp"], s["m"], s["H"], dtype=torch.float32, device=self.X.device)

        def row(mode, parts):
            return (T.lib.row_parallel_forward,
                    (rin.data_ptr(), s["m"], k_in, p_row.data_ptr(), s["H"], s["tp"], None, mode, parts,
                     self.Y.data_ptr(), T.DTYPE_BF16, self.ws.data_ptr(), wsb, st))
        # the bf16 exchange (each shard's partial rounded to bf16 and summed in shard order,
        # the numerics of an all-reduce of bf16 activations), fused inside the row GEMM
        out = {"two_launches_fused_reduce": [col, row(T.REDUCE_FUSED, None)],
               "two_launches_standalone_reduce": [col, row(T.REDUCE_PARTIALS, self.partials.data_ptr())],
               "two_launches_bf16_exchange": [col, row(T.REDUCE_BF16, None)]}
        if self.fused:
            out = {"one_launch": list(self.calls), **out}
        return out

    def launch(self, ev=None):
        n = len(self.calls)
        for j, (fn, a) in enumerate(self.calls):
            rc = fn(*a)
            if rc != 0:
                raise RuntimeError(f"{fn.__name__}: {self.T.status_string(rc)}")
            if ev is not None and j + 1 < n:
                ev[j + 1].record()
        return self.kernels_per_step or n

    # ---- end to end through the public entry points, from pinned host memory.
    # A stream of batches is served the way a user pipelines it: batch i's inputs
    # are copied up on one stream, computed on a second, and its result copied
    # down on a third, so later batches' uploads and earlier batches' downloads
    # overlap batch i's compute (E2E_BUFS device buffers per input and output,
    # so a copy's latency does not stall the compute stream). Every batch
    # pays its own copies. The packed weights rotate over enough copies to exceed
    # the L2 twice, so no batch reads weights left warm by the previous one.
    def e2e_setup(self, l2_bytes=L2_BYTES):
        torch, s = self.torch, self.spec
        name = s["name"]
        self.hX = torch.empty(self.X.shape, dtype=self.X.dtype, pin_memory=True)
        self.hX.copy_(self.X.cpu())
        nb = E2E_BUFS
        self.dX = [self.X] + [torch.empty_like(self.X) for _ in range(nb - 1)]
        ins = [(self.hX, self.dX)]
        if name in ("gqa_proj", "layer70b"):
            self.hA = torch.empty(self.A.shape, dtype=self.A.dtype, pin_memory=True)
            self.hA.copy_(self.A.cpu())
            self.dA = [self.A] + [torch.empty_like(self.A) for _ in range(nb - 1)]
            ins.append((self.hA, self.dA))
        outs = [self.Y] + ([self.Y2] if name == "layer70b" else [])
        self.dY = [outs] + [[torch.empty_like(o) for o in outs] for _ in range(nb - 1)]
        self.hY = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs] for _ in range(nb)]
        self.e2e_ins = ins
        if name in ("gelu_mlp", "gated_decode"):
            wts = [self.p_up, self.p_down]
        elif name == "lm_head_greedy":
            wts = [self.p_w]
        elif name == "gqa_attention":
            wts = []
        else:
            wts = [self.p_qkv, self.p_o] + ([self.p_up, self.p_down] if name == "layer70b" else [])
        wbytes = sum(w.numel() * w.element_size() for w in wts)
        ncopies = 1 if (wbytes == 0 or wbytes >= 2 * l2_bytes) else -(-2 * l2_bytes // wbytes)
        self.wsets = [wts] + [[w.clone() for w in wts] for _ in range(ncopies - 1)]
        self.e2e_streams = [torch.cuda.Stream(device=self.X.device) for _ in range(3)]
        h2d = sum(h.numel() * h.element_size() for h, _ in ins)
        d2h = sum(o.numel() * o.element_size() for o in outs)
        return h2d, d2h, ncopies

    def _e2e_bind(self):
        """Prebuilt calls of the pipelined run: per buffer b the host<->device copies,
        per (b, weight copy) the public entry point calls on the compute stream."""
        import ctypes
        T, s = self.T, self.spec
        name = s["name"]
        up, comp, down = (st.cuda_stream for st in self.e2e_streams)
        self.e2e_handles = (up, comp, down)
        nb = E2E_BUFS
        self.copies_in = [[(d[b].data_ptr(), h.data_ptr(), h.numel() * h.element_size()) for h, d in self.e2e_ins]
                          for b in range(nb)]
        self.copies_out = [[(ho.data_ptr(), o.data_ptr(), o.numel() * o.element_size())
                            for o, ho in zip(self.dY[b], self.hY[b])] for b in range(nb)]
        wsb = self.ws.numel()
        self._heads_e2e = self.heads.c() if hasattr(self, "heads") else None
        calls = []
        for b in range(nb):
            per_w = []
            for w in self.wsets:
                if name == "gqa_attention":
                    per_w.append([(T.lib.sharded_gqa_attention,
                                   (self.dX[b].data_ptr(), s["nseq"], s["S"], ctypes.byref(self._heads_e2e), s["tp"],
                                    1, self.dY[b][0].data_ptr(), comp))])
                elif name == "lm_head_greedy":
                    per_w.append([(T.lib.vocab_parallel_argmax,
                                   (self.dX[b].data_ptr(), s["m"], s["H"], w[0].data_ptr(), s["V"], s["tp"],
                                    self.dY[b][0].data_ptr(), None, self.ws.data_ptr(), wsb, comp))])
                elif name in ("gelu_mlp", "gated_decode"):
                    per_w.append([(T.lib.sharded_mlp_forward,
                                   (self.dX[b].data_ptr(), s["m"], s["H"], s["I"], s["tp"], self.act, w[0].data_ptr(),
                                    w[1].data_ptr(), self.h.data_ptr(), self.dY[b][0].data_ptr(), T.DTYPE_BF16,
                                    self.ws.data_ptr(), wsb, comp))])
                else:
                    c = [(T.lib.sharded_attn_proj_forward,
                          (self.dX[b].data_ptr(), self.dA[b].data_ptr(), s["m"], s["H"], ctypes.byref(self._heads_e2e),
                           s["tp"], w[0].data_ptr(), w[1].data_ptr(), self.qkv.data_ptr(), self.dY[b][0].data_ptr(),
                           T.DTYPE_BF16, self.ws.data_ptr(), wsb, comp))]
                    if name == "layer70b":
                        c.append((T.lib.sharded_mlp_forward,
                                  (self.dX[b].data_ptr(), s["m"], s["H"], s["I"], s["tp"], T.ACT_SILU_MUL,
                                   w[2].data_ptr(), w[3].data_ptr(), self.h.data_ptr(), self.dY[b][1].data_ptr(),
                                   T.DTYPE_BF16, self.ws.data_ptr(), wsb, comp)))
                    per_w.append(c)
            calls.append(per_w)
        self.e2e_calls = calls
        cu = _driver()
        self.e2e_events = []
        for _ in range(3 * nb):
            e = ctypes.c_void_p()
            _ck(cu.cuEventCreate(ctypes.byref(e), 2), "cuEventCreate")   # no timing
            self.e2e_events.append(e)

    def copy_times(self):
        """Mean device time (us) of one step's upload and of its download alone."""
        torch = self.torch
        cu = _driver()
        up, _, down = self.e2e_handles
        res = {}
        for name, st, sthandle, items, fn in (
                ("h2d", self.e2e_streams[0], up, self.copies_in[0], cu.cuMemcpyHtoDAsync_v2),
                ("d2h", self.e2e_streams[2], down, self.copies_out[0], cu.cuMemcpyDtoHAsync_v2)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            err = 0
            e0.record(st)
            for _ in range(20):
                for a, b, n in items:
                    err |= fn(a, b, n, sthandle)
            e1.record(st)
            e1.synchronize()
            _ck(err, name)
            res[name] = round(e0.elapsed_time(e1) * 1e3 / 20, 2)
        return res

    def _e2e_enqueue(self, nsteps):
        """Enqueues `nsteps` pipelined batches on the three streams."""
        cu = _driver()
        up, comp, down = self.e2e_handles
        nb = E2E_BUFS
        in_done, comp_done, out_done = (self.e2e_events[0:nb], self.e2e_events[nb:2 * nb],
                                        self.e2e_events[2 * nb:3 * nb])
        nw = len(self.wsets)
        err = 0
        for i in range(nsteps):
            b = i % nb
            if i >= nb:
                err |= cu.cuStreamWaitEvent(up, comp_done[b], 0)      # batch i-nb no longer reads buffer b's inputs
            for d, h, n in self.copies_in[b]:
                err |= cu.cuMemcpyHtoDAsync_v2(d, h, n, up)
            err |= cu.cuEventRecord(in_done[b], up)
            err |= cu.cuStreamWaitEvent(comp, in_done[b], 0)
            if i >= nb:
                err |= cu.cuStreamWaitEvent(comp, out_done[b], 0)     # batch i-nb's result has left buffer b
            for fn, a in self.e2e_calls[b][i % nw]:
                rc = fn(*a)
                if rc != 0:
                    raise RuntimeError(f"{fn.__name__}: {self.T.status_string(rc)}")
            err |= cu.cuEventRecord(comp_done[b], comp)
            err |= cu.cuStreamWaitEvent(down, comp_done[b], 0)
            for h, d, n in self.copies_out[b]:
                err |= cu.cuMemcpyDtoHAsync_v2(h, d, n, down)
            err |= cu.cuEventRecord(out_done[b], down)
        _ck(err, "pipelined copies and event edges")

    def e2e_run(self, nsteps):
        """(device ms, host enqueue ms) of `nsteps` pipelined batches issued call by
        call, from the first upload to the last download."""
        torch = self.torch
        if not hasattr(self, "e2e_calls"):
            self._e2e_bind()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        s_up, s_comp, s_down = self.e2e_streams
        for st in self.e2e_streams:
            st.wait_stream(cur)
        t0.record(s_up)
        h0 = time.perf_counter()
        self._e2e_enqueue(nsteps)
        host_ms = (time.perf_counter() - h0) * 1e3
        for st in (s_up, s_comp):
            s_down.wait_stream(st)
        t1.record(s_down)
        t1.synchronize()
        cur.wait_stream(s_down)
        return t0.elapsed_time(t1), host_ms

    def e2e_graph(self, nsteps, per_graph=64):
        """Device ms of `nsteps` pipelined batches replayed from a CUDA graph that
        holds `per_graph` of them (the public entry-point calls, copies and event
        edges captured once), or None if the capture fails."""
        torch = self.torch
        if not hasattr(self, "e2e_calls"):
            self._e2e_bind()
        per_graph = max(per_graph, len(self.wsets), E2E_BUFS)
        cap = torch.cuda.Stream(device=self.X.device)
        g = torch.cuda.CUDAGraph()
        try:
            cap.wait_stream(torch.cuda.current_stream())
            # thread-local capture: CUDA calls of other threads (the NCCL watchdog
            # under torchrun) neither break the capture nor are refused by it
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                for st in self.e2e_streams:
                    st.wait_stream(cap)
                self._e2e_enqueue(per_graph)
                for st in self.e2e_streams:
                    cap.wait_stream(st)
        except Exception as exc:  # noqa: BLE001 -- report, measure without the graph
            torch.cuda.synchronize()
            self.graph_error = f"{type(exc).__name__}: {exc}"[:200]
            return None
        reps = max(1, nsteps // per_graph)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        t0.record(cur)
        for _ in range(reps):
            g.replay()
        t1.record(cur)
        t1.synchronize()
        del g
        return t0.elapsed_time(t1), reps * per_graph


_DRIVER = None


def _driver():
    """The CUDA driver library (stream-ordered copies and event edges for the
    pipelined end-to-end run)."""
    global _DRIVER
    if _DRIVER is None:
        import ctypes
        cu = ctypes.CDLL("libcuda.so.1")
        P, S, U = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint
        cu.cuMemcpyHtoDAsync_v2.argtypes = [ctypes.c_uint64, P, S, P]
        cu.cuMemcpyDtoHAsync_v2.argtypes = [P, ctypes.c_uint64, S, P]
        cu.cuEventCreate.argtypes = [ctypes.POINTER(P), U]
        cu.cuEventRecord.argtypes = [P, P]
        cu.cuStreamWaitEvent.argtypes = [P, P, U]
        _DRIVER = cu
    return _DRIVER


def _ck(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA driver error {rc}")


# ============================================================ clocks
CLOCK_FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="tps_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(CLOCK_FIELDS)}", "-i", str(self.idx),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < len(CLOCK_FIELDS):
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ============================================================ measurement
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def traffic_for(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("kernel_source_hash") != kernel_source_hash(workload):
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over every rank of the default process group
    (identity without one); the bench times each rank on its device and reports
    the slowest."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_step: float, steps: int, world: int, max_ms: float, scale: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_step * steps / (max_ms * 1e-3) / scale


def run_ours(args, spec, rank, world, local_rank):
    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if getattr(args, "plan_override", 0):
        import tensor_sharded_linear_columnparallel_b200 as T
        T.tps_set_plan_override(args.plan_override)
    step = GpuStep(spec, device)
    flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush_sink = torch.empty((), dtype=torch.float32, device=device)

    class _Flush:
        @staticmethod
        def zero_():
            flush_buf.zero_()
            flush_sink.copy_(flush_buf.sum())

    flush = _Flush()
    if step.fused:
        # one launch per step: the whole block is the kernel the roofline describes
        label = ("fused MLP: fc1+GELU, fc2+reduce (one launch)" if spec["name"] == "gelu_mlp"
                 else "fused MLP: gate/up+SiLU*up, down+reduce (one launch)")
        spec = dict(spec, kernels=[(label, sum(u for _, u in spec["kernels"]))])
    nk = len(spec["kernels"])
    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local_rank])

    # warm-up
    for _ in range(args.warmup):
        step.launch()
        flush.zero_()
    torch.cuda.synchronize()

    # Timed region: events only at the step boundaries, so consecutive kernels of
    # a step overlap launch and prologue (programmatic dependent launch).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    time.sleep(0.2)
    barrier()
    torch.cuda.synchronize()
    # one flush ahead of the first step: the device works on it while the host enqueues
    # that step, so no step's events include host launch latency
    flush.zero_()
    launches = 0
    for i in range(args.steps):
        e = evs[i]
        e[0].record()
        launches += step.launch()
        e[1].record()
        flush.zero_()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    total_ms = max_over_ranks(total_ms, device)

    # Per-kernel split for the roofline: the same steps again, with an event
    # recorded after every kernel (which serialises the kernels of a step).
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    flush.zero_()
    for i in range(args.steps):
        e = kevs[i]
        e[0].record()
        step.launch(e)
        e[nk].record()
        flush.zero_()
    torch.cuda.synchronize()
    per_kernel = [0.0] * nk
    for e in kevs:
        for j in range(nk):
            per_kernel[j] += e[j].elapsed_time(e[j + 1])

    # end to end through the public entry points, pinned host buffers, pipelined:
    # call by call, and replayed from a CUDA graph of the same calls
    h2d, d2h, ncopies = step.e2e_setup()
    step.e2e_run(max(4, args.warmup))
    torch.cuda.synchronize()
    e_steps = max(64, min(args.steps, 256))
    barrier()
    loop_ms, host_ms = step.e2e_run(e_steps)
    loop_ms = max_over_ranks(loop_ms, device)
    gr = step.e2e_graph(e_steps)
    ok_graph = max_over_ranks(0.0 if gr is not None else 1.0, device) == 0.0
    if ok_graph:
        graph_ms, graph_steps = gr
        graph_ms = max_over_ranks(graph_ms, device)

    units = spec["step_units"]
    scale = 1e12 if spec["unit"] == "TFLOP/s" else 1e9
    value = whole_job_value(units, args.steps, world, total_ms, scale)
    loop_val = whole_job_value(units, e_steps, world, loop_ms, scale)
    # e2e is the faster of the two ways of driving the entry points; both are reported
    e2e_val, e2e_ms, e_n = loop_val, loop_ms, e_steps
    method = "entry points called batch by batch"
    graph_info = {"error": getattr(step, "graph_error", "?")}
    if ok_graph:
        graph_val = whole_job_value(units, graph_steps, world, graph_ms, scale)
        graph_info = {"value": graph_val, "ms_per_step": round(graph_ms / graph_steps, 5), "batches_per_replay": 64}
        if graph_val > loop_val:
            e2e_val, e2e_ms, e_n = graph_val, graph_ms, graph_steps
            method = "CUDA graph of the pipelined entry-point calls (64 batches per replay)"

    peaks, src = measured_peaks()
    dom = max(range(nk), key=lambda j: per_kernel[j])
    dom_ms = per_kernel[dom] / args.steps
    dom_name, dom_units = spec["kernels"][dom]
    achieved = dom_units / (dom_ms * 1e-3) / scale
    extra = {}
    if spec["bound"] == "tensor":
        # The burst peak unless the sampled SM clock fell below the maximum during
        # the timed region (a power-capped, sustained run): then the sustained one.
        sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
        sustained = bool(sm and smax and sm < 0.97 * smax)
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        peak_kind = ("sustained" if sustained else "burst") + f" bf16 dense ({src})"
        runit = "TFLOP/s"
        extra = {"frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
                 "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}
    else:
        peak = peaks["hbm_gbs"]
        peak_kind = f"HBM copy ({src})"
        runit = "GB/s"
    roof = {"bound": spec["bound"], "achieved": round(achieved, 2), "peak": peak, "unit": runit,
            "frac": round(achieved / peak, 4), "traffic": traffic_for(spec["name"], dom_name),
            "kernel": dom_name, "peak_source": peak_kind,
            "kernel_ms": [round(x / args.steps, 5) for x in per_kernel],
            "kernels": [k for k, _ in spec["kernels"]], **extra}
    return {
        "value": value, "ms_per_step": total_ms / args.steps, "e2e": {
            "value": e2e_val, "unit": spec["unit"], "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": e_n, "ms_per_step": round(e2e_ms / e_n, 5), "method": method,
            "graph_replay": graph_info,
            "call_by_call": {"value": loop_val, "ms_per_step": round(loop_ms / e_steps, 5),
                             "host_enqueue_ms_per_step": round(host_ms / e_steps, 5)},
            "pipelining": f"upload / compute / download on three streams, {E2E_BUFS} buffers each",
            "copy_us": step.copy_times(),
            "weight_copies": ncopies},
        "roofline": roof, "clocks": clocks, "gpu_launches": launches,
        "variants": variant_times(step, flush, 0 if (args.no_variants or spec["name"] == "layer70b") else
                                  getattr(args, "variant_reps", 100)),
    }


def variant_times(step, flush, reps):
    """Mean ms per step of each variant of the block (same flush between steps);
    the no-workspace override is restored afterwards."""
    import torch
    T = step.T
    res = {}
    vc = step.variant_calls() if reps else {}
    for name, calls in vc.items():
        ov = getattr(step, "variant_overrides", {}).get(name)
        if ov is not None:
            prev = T.tps_set_plan_override(ov)
        # the two-launch variants run the column and row entry points themselves
        for _ in range(3):
            for fn, a in calls:
                rc = fn(*a)
                if rc != 0:
                    raise RuntimeError(f"{name}: {T.status_string(rc)}")
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            e0.record()
            for fn, a in calls:
                fn(*a)
            e1.record()
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        res[name] = {"ms_per_step": round(tot / reps, 5), "api_calls": len(calls)}
        if ov is not None:
            T.tps_set_plan_override(prev)
    return res


def cpu_oracle_step(spec, rows):
    """One oracle pass over the first `rows` token rows of the workload (returns units processed)."""
    import oracle as O
    import workloads as WL
    name, tp = spec["name"], spec["tp"]
    if name == "gelu_mlp":
        wl = cpu_oracle_step.cache.get(name) or WL.gelu_mlp(m=spec["m"])
        cpu_oracle_step.cache[name] = wl
        t = wl.tensors
        O.mlp_gelu_sharded(t["X"][:rows], t["W1"], t["W2"], tp)
        return 4.0 * rows * spec["H"] * spec["I"]
    if name == "gated_decode":
        wl = cpu_oracle_step.cache.get(name) or WL.gated_decode(m_max=max(spec["m"], 1))
        cpu_oracle_step.cache[name] = wl
        t = wl.tensors
        O.mlp_gated_sharded(t["X"][:rows], t["Wg"], t["Wu"], t["Wd"], tp)
        return 3.0 * spec["H"] * spec["I"] * 2 + 2.0 * rows * spec["H"] * 2
    if name == "gqa_attention":
        # a causal prefix of the sequence: its outputs are exactly those of the full sequence
        wl = cpu_oracle_step.cache.get(name)
        if wl is None:
            qh, kh = O.head_map(spec["hq"], spec["hkv"], tp)
            wl = WL.gqa_attention(tp * (len(qh[0]) + 2 * len(kh[0])) * spec["d"], nseq=1, S=spec["S"])
        cpu_oracle_step.cache[name] = wl
        O.gqa_attention_sharded(wl.tensors["qkv"][:rows], spec["hq"], spec["hkv"], spec["d"], tp, 1, rows, True)
        return 4.0 * spec["d"] * spec["hq"] * rows * (rows + 1) / 2
    if name == "lm_head_greedy":
        wl = cpu_oracle_step.cache.get(name) or WL.lm_head(m_max=max(spec["m"], 1))
        cpu_oracle_step.cache[name] = wl
        t = wl.tensors
        O.vocab_parallel_argmax(t["X"][:rows], t["W"], tp)
        return 2.0 * spec["H"] * spec["V"] + rows * spec["H"] * 2.0 + rows * 8.0
    wl = cpu_oracle_step.cache.get(name) or (WL.gqa_proj(m=spec["m"]) if name == "gqa_proj" else
                                             WL.layer70b(m=spec["m"]))
    cpu_oracle_step.cache[name] = wl
    t = wl.tensors
    O.attn_proj_sharded(t["X"][:rows], t["A"][:rows], t["Wq"], t["Wk"], t["Wv"], t["Wo"], spec["hq"], spec["hkv"],
                        spec["d"], tp)
    f = 2.0 * rows * spec["H"] * (spec["hq"] + 2 * spec["hkv"]) * spec["d"] + 2.0 * rows * spec["hq"] * spec["d"] * spec["H"]
    if name == "layer70b":
        O.mlp_gated_sharded(t["X"][:rows], t["Wg"], t["Wu"], t["Wd"], tp)
        f += 6.0 * rows * spec["H"] * spec["I"]
    return f


cpu_oracle_step.cache = {}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_rows_for(spec, seconds: float):
    """Token rows per oracle step so that one step takes about `seconds`."""
    probe = min(spec["m"], 16)
    cpu_oracle_step(spec, probe)  # load tensors / warm BLAS
    t0 = time.perf_counter()
    cpu_oracle_step(spec, probe)
    dt = max(time.perf_counter() - t0, 1e-4)
    if spec["name"] in ("gated_decode", "lm_head_greedy"):   # weight-stream bound: every row, all weights
        return spec["m"]
    rows = int(probe * (seconds / dt) ** (0.5 if spec["name"] == "gqa_attention" else 1.0))
    return max(1, min(spec["m"], rows))


def cpu_baseline(spec, budget_s: float = 12.0):
    rows = oracle_rows_for(spec, budget_s / 4)
    units, t0, n = 0.0, time.perf_counter(), 0
    while True:
        units += cpu_oracle_step(spec, rows)
        n += 1
        el = time.perf_counter() - t0
        if el > budget_s or n >= 2000:
            break
    scale = 1e12 if spec["unit"] == "TFLOP/s" else 1e9
    return {"value": units / el / scale, "unit": spec["unit"], "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle passes over the first {rows} of {spec['m']} token rows "
                      f"(all weights), numpy fp64, {el:.1f} s wall"}


def run_reference(args, spec):
    budget = 90.0
    per_step = budget / max(1, args.steps + args.warmup)
    rows = oracle_rows_for(spec, per_step)
    for _ in range(args.warmup):
        cpu_oracle_step(spec, rows)
    t0 = time.perf_counter()
    units = 0.0
    for _ in range(args.steps):
        units += cpu_oracle_step(spec, rows)
    el = time.perf_counter() - t0
    scale = 1e12 if spec["unit"] == "TFLOP/s" else 1e9
    v = units / el / scale
    sample = (f"each step: oracle pass over the first {rows} of {spec['m']} token rows (all weights), "
              f"numpy fp64")
    return {
        "metric": METRIC, "value": v, "unit": spec["unit"], "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(spec), "impl": "reference",
        "cpu_baseline": {"value": v, "unit": spec["unit"], "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": spec["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def config_block(spec):
    return {"workload": spec["label"], "tp_shards": spec["tp"], "tokens": spec["m"],
            "l2": "flushed between timed steps (512 MiB write, then read back)",
            "parallelism": "tp shards emulated on one GPU; ranks are independent replicas"}


def make_parser():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="layer70b",
                    choices=["gelu_mlp", "gated_decode", "gqa_proj", "layer70b", "lm_head_greedy",
                             "gqa_attention"])
    ap.add_argument("--tp", type=int, default=None)
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip the timing of the block's other variants")
    ap.add_argument("--plan-override", type=int, default=0,
                    help="tps_set_plan_override value for every call (0 = the planner's own choice)")
    ap.add_argument("--no-suite", action="store_true",
                    help="time the chosen workload only (by default a 1-GPU run of the 70B layer also times every "
                         "other workload and reports each under `configs`)")
    return ap


def main():
    args = make_parser().parse_args()
    if args.warmup < 3:
        args.warmup = 3
    spec = workload_spec(args.workload, args.tp, args.m)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, spec)), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_ours(args, spec, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": res["value"], "unit": spec["unit"], "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, shapes and distributions of the workload)",
        "config": config_block(spec), "e2e": res["e2e"], "roofline": res["roofline"], "clocks": res["clocks"],
        "gpu_launches": world * res["gpu_launches"], "variants": res["variants"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(spec)
    if world == 1 and not args.no_suite and args.workload == "layer70b" and args.m is None and args.tp is None:
        line["configs"] = run_suite(args, local_rank)
    print(json.dumps(line), flush=True)
    return 0


# The other workloads of the block, each timed the same way as the headline (its
# own warm-up, K timed steps with the L2 flushed between them, per-kernel split,
# pipelined end to end run, clocks) and reported under `configs`: the decode
# half of the metric (weight-stream GB/s), the smaller prefill blocks, the
# attention on local heads and the greedy lm_head.
SUITE = [
    ("gated_decode_m64", "gated_decode", 8, 64),
    ("gated_decode_m1", "gated_decode", 8, 1),
    ("gelu_mlp_tp8", "gelu_mlp", 8, 512),
    ("gqa_proj_tp8", "gqa_proj", 8, 2048),
    ("gqa_proj_tp16", "gqa_proj", 16, 2048),
    ("gqa_attention_tp8", "gqa_attention", 8, 2048),
    ("lm_head_greedy_m64", "lm_head_greedy", 8, 64),
]


def run_suite(args, local_rank):
    import torch
    out = {}
    sub = argparse.Namespace(**vars(args))
    sub.variant_reps = 30
    for key, name, tp, m in SUITE:
        spec = workload_spec(name, tp, m)
        res = run_ours(sub, spec, 0, 1, local_rank)
        entry = {"metric": METRIC, "value": res["value"], "unit": spec["unit"], "ms_per_step": res["ms_per_step"],
                 "steps": args.steps, "warmup": args.warmup, "config": config_block(spec),
                 "roofline": res["roofline"], "e2e": res["e2e"], "clocks": res["clocks"],
                 "gpu_launches": res["gpu_launches"], "variants": res["variants"]}
        if not args.no_cpu_baseline:
            entry["cpu_baseline"] = cpu_baseline(spec, budget_s=4.0)
        out[key] = entry
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
