"""bench.py's JSON line, on the CPU: every workload's reference arm (the fp64
oracle timed on the host) prints exactly one line with the contract's keys;
the DRAM-traffic lookup only answers for the shape it was captured on."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
             "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("workload", ["attention", "attention-2k", "decode", "ring", "fp8", "blocksparse", "sweep", "varlen"])
def test_reference_arm_prints_one_contract_line(workload):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          workload, "--steps", "1", "--warmup", "0", "--cpu-budget-s", "0.3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert BASE_KEYS <= set(j), BASE_KEYS - set(j)
    assert j["impl"] == "reference" and j["n_gpus"] == 1 and j["steps"] == 1
    assert j["value"] > 0 and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert isinstance(j["cpu_baseline"]["blas"], str)
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    assert isinstance(j["config"]["workload"], str) and j["config"]["workload"]


def test_traffic_lookup_is_keyed_by_shape():
    import bench
    j = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for kernel, entries in j.items():
        if kernel.startswith("_"):
            continue
        shapes = [e["shape"] for e in entries]
        assert len(shapes) == len(set(shapes)), kernel
        for e in entries:
            assert isinstance(e["shape"], str) and e["dram_bytes_per_launch"] > 0
            if e["source_hash"] == bench.kernel_source_hash(kernel):
                assert bench.traffic_for(kernel, e["shape"]) == e["dram_bytes_per_launch"]
            assert bench.traffic_for(kernel, e["shape"] + " other") is None


def _max_rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(dist, torch.device("cpu"), 1.5 + 10.0 * rank)
        again = bench.max_over_ranks(dist, torch.device("cpu"), 7.25 - rank)
        q.put((rank, got, again))
    finally:
        dist.destroy_process_group()


def test_time_is_the_slowest_ranks_on_cpu_ranks():
    """The multi-GPU bench reports each timed quantity as its maximum over the
    ranks: gloo ranks stand in for the GPUs here."""
    import socket
    import torch.multiprocessing as mp
    import bench
    assert bench.max_over_ranks(None, None, 3.5) == 3.5
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_max_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    assert res == [(0, 11.5, 7.25), (1, 11.5, 7.25)]


def test_kernel_sources_keep_the_kernels_apart():
    """A kernel's DRAM counters are keyed by its own device sources only: the
    dK/dV and dQ kernels do not include the forward's or the preparation's
    header, and the forward does not include the backward's."""
    import bench
    bwd = bench.kernel_sources("fa_bwd_dkdv_kernel")
    assert bwd == bench.kernel_sources("fa_bwd_dq_kernel")
    assert {"fa_bwd_kernel.cuh", "fa_bwd_args.cuh", "fa_tile.cuh", "fa_common.cuh", "sm100_ptx.cuh"} <= set(bwd)
    assert "fa_fwd_kernel.cuh" not in bwd and "fa_bwd_pre_kernel.cuh" not in bwd
    fwd = bench.kernel_sources("fa_fwd_sm100_kernel")
    assert "fa_fwd_kernel.cuh" in fwd and not any(f.startswith("fa_bwd") for f in fwd)
    assert "fa_decode_kernel.cuh" in bench.kernel_sources("fa_decode_kernel")
