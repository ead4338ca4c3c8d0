"""Host logic of bench.py's multi-process path, on CPU with the gloo backend:
every rank times its own replica and the reported time is the max over ranks;
the whole-job value counts the units of every rank. Also: the reference arm
does its work on rank 0 only."""

import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [3.0, 7.5, 5.0, 1.0][rank]
        m = bench.max_over_ranks(per_rank_ms)
        v = bench.whole_job_value(10.0, 4, world, m, 1.0)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks_and_whole_job_value_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + world * 7 + os.getpid() % 400
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    want = max([3.0, 7.5, 5.0, 1.0][:world])
    for _, m, v in res:
        assert m == want
        assert abs(v - world * 10.0 * 4 / (want * 1e-3)) < 1e-6


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.whole_job_value(8.59e9, 10, 1, 1.0, 1e12) == pytest.approx(85.9)


def test_reference_arm_nonzero_rank_does_no_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_workload_specs_units_and_sources():
    """Every bench workload names its metric unit, its roofline bound, the files its
    kernels are built from, and credits exactly the algorithmic work of the step."""
    import bench
    for name in bench.KERNEL_SOURCES:
        s = bench.workload_spec(name, None, None)
        assert s["unit"] in ("TFLOP/s", "GB/s") and s["bound"] in ("tensor", "hbm")
        assert s["step_units"] > 0 and s["kernels"]
        for f in bench.KERNEL_SOURCES[name]:
            assert os.path.exists(os.path.join(ROOT, "tensor_sharded_linear_columnparallel_b200", "csrc", f)), f
        assert len(bench.kernel_source_hash(name)) == 16
    # causal attention credits 4*d FLOP per visible (query, key) pair
    for S in (1, 5, 128, 2048):
        s = bench.workload_spec("gqa_attention", None, S)
        pairs = sum(q + 1 for q in range(S))
        assert s["step_units"] == 4.0 * s["d"] * s["hq"] * pairs
    # greedy lm_head: the weight once, X once, 8 bytes (token id, logit) per row
    s = bench.workload_spec("lm_head_greedy", None, 64)
    assert s["step_units"] == 2.0 * 4096 * 128256 + 64 * 4096 * 2 + 64 * 8


def test_headline_is_the_largest_config_and_the_suite_covers_the_rest():
    """With no flags the bench times the 70B-layer linears (the largest workload that
    fits one GPU) as the headline, and its suite times every other workload: the
    decode half of the metric (GB/s) and the smaller blocks, each with its own line."""
    import bench
    args = bench.make_parser().parse_args([])
    assert args.workload == "layer70b" and args.gpus == 1 and not args.no_suite
    names = {name for _, name, _, _ in bench.SUITE}
    assert names == set(bench.KERNEL_SOURCES) - {"layer70b"}
    assert len({key for key, _, _, _ in bench.SUITE}) == len(bench.SUITE)
    decode = [m for _, name, _, m in bench.SUITE if name == "gated_decode"]
    assert 64 in decode and bench.workload_spec("gated_decode", 8, 64)["unit"] == "GB/s"
