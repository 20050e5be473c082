#!/usr/bin/env python
"""Throughput of the exact-attention hot path on B200 (attention TFLOP/s).

One step = the whole hot path over one batch of synthetic input: the causal
bf16 forward pass (O, LSE) and the backward pass (dQ, dK, dV). The default
workload is long-context GQA attention, B=1 Hq=32 Hkv=8 N=16384 d=128
(`--workload attention`); `--workload attention-2k` runs B=4 Hq=Hkv=16 N=2048
d=128. Q, K, V, dO are i.i.d. N(0,1) rounded to bf16, seed 0 (rank r: seed r).
Flops: forward 4*B*Hq*N^2*d halved for causal, backward 2.5x the forward
(five GEMMs instead of two).

The step is timed through the public calls (fa_fwd, fa_bwd); a second pass
times the kernels one by one for the roofline of the dominant one.

Prints ONE JSON line (rank 0). `--impl reference` times the fp64 CPU oracle
instead, on a bounded sample of the same workload. Multi-GPU (torchrun):
every rank runs its own independent batch (weak scaling, no data-path
collective); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# the two padded-batch fwd+bwd workloads; the first is the default line
ATTN_WORKLOADS = {
    "attention": {"workload": "bf16 causal attention fwd+bwd, long-context GQA, B=1 Hq=32 Hkv=8 N=16384 d=128",
                  "B": 1, "Hq": 32, "Hkv": 8, "N": 16384, "d": 128, "causal": True},
    "attention-2k": {"workload": "bf16 causal attention fwd+bwd, B=4 Hq=Hkv=16 N=2048 d=128",
                     "B": 4, "Hq": 16, "Hkv": 16, "N": 2048, "d": 128, "causal": True},
}
WORKLOAD = dict(ATTN_WORKLOADS["attention"])
# above this sequence length the CPU oracle samples query rows of a head
# instead of whole heads (a head's fp64 score matrix alone is N^2 * 8 bytes)
ORACLE_ROWS_FROM_N = 8192
ORACLE_SAMPLE_ROWS = 256
METRIC = "attention TFLOP/s (bf16/fp8, causal, N=2K–16K) and % of B200 tensor peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def fwd_flops(B, Hq, N, d, causal):
    return 4.0 * B * Hq * N * N * d / (2.0 if causal else 1.0)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-bwd", action="store_true", help="time the forward pass only")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--shape", default=None,
                    help="B,Hq,Hkv,N,d,causal: another workload (profiling captures; not the headline line)")
    ap.add_argument("--workload", default="attention",
                    choices=["attention", "attention-2k", "decode", "ring", "fp8", "blocksparse", "sweep", "varlen"],
                    help="attention: causal fwd+bwd, B=1 Hq=32 Hkv=8 N=16384 d=128 (default); attention-2k: causal "
                         "fwd+bwd, B=4 Hq=Hkv=16 N=2048 d=128; decode: Nq new query rows against a KV cache (fa_fwd_kvcache), GB/s of cache read; "
                         "ring: context-parallel ring attention forward over the ranks (one GPU: 4 ranks emulated); "
                         "fp8: Hadamard-rotated e4m3 quantisation + fp8 forward (B=2 H=16 N=8192 d=128 causal); "
                         "sweep: causal fwd+bwd at N = 2K..32K with B*N = 32K tokens (H=16 d=128), plus the tiny "
                         "B=1 H=2 N=256 d=64 case; varlen: 24 packed causal sequences of U[128,4096] tokens, "
                         "fwd+bwd (H=16 d=128)")
    ap.add_argument("--ring-shape", default="1,32,8,16384,128",
                    help="B,Hq,Hkv,N,d of the ring workload (causal; N split over the ring)")
    ap.add_argument("--ring-ranks", type=int, default=4, help="ranks emulated on one GPU (--gpus 1)")
    ap.add_argument("--decode-shape", default="16,1,32,8,16384,128",
                    help="B,Nq,Hq,Hkv,Ncache,d of the decode workload")
    args = ap.parse_args()
    if args.workload in ATTN_WORKLOADS:
        WORKLOAD.clear()
        WORKLOAD.update(ATTN_WORKLOADS[args.workload])
    if args.shape:
        B, Hq, Hkv, N, d, c = (int(x) for x in args.shape.split(","))
        WORKLOAD.update({"B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "causal": bool(c),
                         "workload": f"bf16 {'causal' if c else 'non-causal'} attention fwd+bwd, "
                                     f"B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}"})
    return args


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"bf16_tflops": j["bf16_tflops"], "bf16_tflops_sustained": j["bf16_tflops_sustained"],
                "hbm_gbs": j["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# the device source file that defines each profiled kernel
KERNEL_HEADER = {"fa_fwd_sm100_kernel": "fa_fwd_kernel.cuh", "fa_bwd_dkdv_kernel": "fa_bwd_kernel.cuh",
                 "fa_bwd_dq_kernel": "fa_bwd_kernel.cuh", "fa_decode_kernel": "fa_decode_kernel.cuh"}


def kernel_sources(kernel):
    """The device sources of a profiled kernel: its header and every header it
    includes, followed transitively (sorted names under csrc/)."""
    import re
    csrc = os.path.join(ROOT, "io_aware_exact_27_b200", "csrc")
    todo, seen = [KERNEL_HEADER[kernel]], []
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.append(f)
        todo += re.findall(r'^#include "([^"]+)"', open(os.path.join(csrc, f)).read(), flags=re.M)
    return sorted(seen)


def kernel_source_hash(kernel):
    """Hash of a kernel's device code (kernel_sources). The host launcher is
    not part of it: a change of a kernel's launch configuration there must be
    re-captured by hand."""
    csrc = os.path.join(ROOT, "io_aware_exact_27_b200", "csrc")
    seen = kernel_sources(kernel)
    h = hashlib.sha256()
    for f in sorted(seen):
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel, shape):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when the kernel's device sources changed since those counters were taken
    or the capture ran another shape than `shape`."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_HEADER:
        return None
    j = json.load(open(p))
    entries = j.get(kernel) or []
    if isinstance(entries, dict):
        entries = [entries]
    h = kernel_source_hash(kernel)
    for e in entries:
        if e.get("source_hash") == h and e.get("shape") == shape:
            return e.get("dram_bytes_per_launch")
    return None


def step_shape(B, Hq, Hkv, N, d, causal):
    return f"B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} causal={int(bool(causal))}"


def decode_shape_key(B, Nq, Hq, Hkv, Nc, d):
    return f"B={B} Nq={Nq} Hq={Hq} Hkv={Hkv} Ncache={Nc} d={d}"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        mhz.sort()
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


def oracle_threads():
    """Threads of the BLAS pool numpy runs the oracle's products on (the
    cores the oracle actually uses; its elementwise steps run on one), and
    that BLAS's name and version."""
    try:
        import numpy  # noqa: F401  (loads the BLAS the pool info reports)
        import threadpoolctl
        pools = [p for p in threadpoolctl.threadpool_info() if p.get("user_api") == "blas"]
        if pools:
            p = max(pools, key=lambda x: x.get("num_threads") or 0)
            return int(p["num_threads"]), f"{p.get('internal_api')} {p.get('version')}"
    except Exception:
        pass
    return os.cpu_count(), "unknown"


def max_over_ranks(pg, dev, value):
    """The largest of `value` over the ranks of the default process group
    (every rank calls this at the same point, with its own value): the
    time of a multi-GPU run is its slowest rank's. pg is torch.distributed,
    or None for a single process (value returned as is)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


E2E_OVERLAP = ("inputs in, compute, results out on three streams with two device buffers per tensor; "
               "every step copies all of its inputs in and all of its results out")


def e2e_pipelined(torch, dev, stream, pin_in, ins0, outs0, launch, steps, pg=None):
    """End-to-end time of `steps` steps through the public API: step i copies
    its inputs from the pinned host tensors `pin_in` into device buffers,
    runs launch(ins, outs, b) on `stream`, and copies `outs` back into pinned
    host buffers. Inputs in, compute and results out run on three streams
    with two device buffers per tensor (b = i % 2), so that a step's compute
    overlaps the next step's inputs and the previous step's results, as a
    training loop that prefetches its next batch would. Returns the
    milliseconds (max over ranks) and the bytes copied each way per step."""
    ins = [list(ins0), [torch.empty_like(t) for t in ins0]]
    outs = [list(outs0), [torch.empty_like(t) for t in outs0]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs0] for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in, ev_done, ev_read = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    e0.record(s_in)
    for i in range(steps):
        b = i & 1
        if i >= 2:
            s_in.wait_event(ev_done[b])  # step i-2's compute is done with buffer b's inputs
        with torch.cuda.stream(s_in):
            for dst, src in zip(ins[b], pin_in):
                dst.copy_(src, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_read[b])  # step i-2's results in buffer b are back on the host
        launch(ins[b], outs[b], b)
        ev_done[b].record(stream)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            for dst, src in zip(host_out[b], outs[b]):
                dst.copy_(src, non_blocking=True)
        ev_read[b].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e_ms = max_over_ranks(pg, dev, e0.elapsed_time(e1))
    return e_ms, sum(t.numel() * t.element_size() for t in pin_in), sum(t.numel() * t.element_size() for t in host_out[0])


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------- reference arm (CPU oracle)

def oracle_sample(budget_s, with_bwd, w=None):
    """Times the fp64 oracle on a bounded sample of the workload (default:
    the bench's) until `budget_s` is spent: whole (batch, head) problems, or
    for N >= ORACLE_ROWS_FROM_N the seeded 256 query rows of one (batch,
    head) at a time (forward, and the rows' backward: their dQ and their
    share of dK, dV). Returns (TFLOP/s, units done, seconds, cores, what a
    unit is); flops are the algorithmic ones of the rows computed (causal:
    row i sees i + 1 keys)."""
    import numpy as np
    import oracle
    import synth
    w = w or WORKLOAD
    q, k, v, do = synth.qkv_bf16(0, w["B"], w["N"], w["Hq"], w["Hkv"], w["d"], with_dout=True)
    scale = 1.0 / math.sqrt(w["d"])
    mult = 3.5 if with_bwd else 1.0
    N, d = w["N"], w["d"]
    by_rows = N >= ORACLE_ROWS_FROM_N
    rows_all = synth.sample_rows(2, N, w["Hq"], R=ORACLE_SAMPLE_ROWS) if by_rows else None
    done, flops, t0 = 0, 0.0, time.perf_counter()
    total = w["B"] * w["Hq"]
    while done < total:
        b, h = divmod(done, w["Hq"])
        g = oracle.kv_head_of(h, w["Hq"], w["Hkv"])
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        slk = (slice(b, b + 1), slice(None), slice(g, g + 1))
        if by_rows:
            r = rows_all[h:h + 1]
            oracle.attn_fwd_rows(q[sl], k[slk], v[slk], w["causal"], scale, r)
            if with_bwd:
                oracle.attn_bwd_rows(q[sl], k[slk], v[slk], do[sl], w["causal"], scale, r)
            seen = (r[0] + 1).sum() if w["causal"] else r.shape[1] * N
            flops += 4.0 * d * float(seen) * mult
        else:
            oracle.attn_fwd(q[sl], k[slk], v[slk], w["causal"], scale)
            if with_bwd:
                oracle.attn_bwd(q[sl], k[slk], v[slk], do[sl], w["causal"], scale)
            flops += fwd_flops(1, 1, N, d, w["causal"]) * mult
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    cores = oracle_threads()[0]
    unit = (f"{ORACLE_SAMPLE_ROWS} seeded query rows of one (batch, head)" if by_rows
            else "one whole (batch, head) problem")
    return flops / el / 1e12, done, el, cores, unit


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    with_bwd = not args.no_bwd
    # each step: a bounded sample sized so the whole run ends within minutes
    per_step_budget = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        tf, heads, el, cores, unit = oracle_sample(per_step_budget, with_bwd)
        if i >= args.warmup:
            vals.append((tf, heads, el))
    tf = sum(v[0] for v in vals) / len(vals)
    ms = sum(v[2] for v in vals) / len(vals) * 1e3
    heads = vals[-1][1]
    total = WORKLOAD["B"] * WORKLOAD["Hq"]
    sample = (f"{heads} units per step (unit: {unit}; {total} (batch, head) problems in the workload), "
              f"fp64 numpy, {'fwd+bwd' if with_bwd else 'fwd'}")
    line = {"metric": METRIC, "value": tf, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": dict(WORKLOAD, parallelism=f"replicas{args.gpus}", l2="n/a (CPU)"),
            "cpu_baseline": {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "blas": oracle_threads()[1], "sample": sample},
            "e2e": {"value": tf, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    world, rank, local = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    import synth

    w = WORKLOAD
    B, Hq, Hkv, N, d, causal = w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], w["causal"]
    scale = 1.0 / math.sqrt(d)
    with_bwd = not args.no_bwd
    if with_bwd:
        try:
            probe_ws = fa.fa_bwd_workspace_size(B * N, B, Hq, d)
            fa.fa_bwd(0, 0, 0, 0, 0, 0, 0, 0, 0, 0, probe_ws, B, Hq, Hkv, N, d, 1, scale)
        except fa.FAError as e:
            if e.status == fa.FA_ERR_UNSUPPORTED:
                with_bwd = False  # backward not in this build of the library
    q_h, k_h, v_h, do_h = synth.qkv_bf16(rank, B, N, Hq, Hkv, d, with_dout=True)
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa.fa_bwd_workspace_size(B * N, B, Hq, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    def step():
        fa.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, int(causal), scale, sptr)
        if with_bwd:
            fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, N, d, int(causal), scale, sptr)

    launches_per_step = 1 + (3 if with_bwd else 0)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error during warm-up")

    # timed region: K steps through the public calls (fa_fwd, then fa_bwd,
    # which runs its dQ kernel beside the dK/dV kernel), L2 flushed before
    # each step (outside the step's events)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    st = fa.fa_get_status(sptr)
    if st != fa.FA_OK:
        raise SystemExit(f"device status error: {fa.fa_status_string(st)}")
    tot_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    # per-kernel times for the roofline: a second pass with the backward as its
    # three parts one after another (exactly fa_bwd's work), events between them
    nev = 5 if with_bwd else 2
    nseg = max(3, args.steps // 4)
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(nseg)]
    for i in range(nseg):
        flush.zero_()
        e = ev2[i]
        e[0].record(stream)
        fa.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, int(causal), scale, sptr)
        e[1].record(stream)
        if with_bwd:
            for j, part in enumerate((fa.FA_BWD_PREPARE, fa.FA_BWD_DKDV, fa.FA_BWD_DQ)):
                fa.fa_bwd_part(part, q, k, v, o, lse, do, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, N, d,
                               int(causal), scale, sptr)
                e[2 + j].record(stream)
    torch.cuda.synchronize(dev)
    seg = [[e[j].elapsed_time(e[j + 1]) for e in ev2] for j in range(nev - 1)]
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    ms_per_step = tot_ms / args.steps
    f_fwd = fwd_flops(B, Hq, N, d, causal)
    f_step = f_fwd * (3.5 if with_bwd else 1.0)
    value = f_step * world * args.steps / (tot_ms * 1e-3) / 1e12

    # roofline of the dominant kernel (largest share of the step). Flops per
    # launch are the tensor-core flops the kernel executes: forward 2 GEMMs
    # (= the algorithmic forward count), dK/dV 4 GEMMs, dQ 3 GEMMs (S and dP
    # recomputed); the D/LSE preparation is HBM-bound (bytes moved).
    pk = peaks()
    avg = [sum(x) / len(x) for x in seg]
    tok = B * N
    kernels = [{"kernel": "fa_fwd_sm100_kernel", "ms": avg[0], "bound": "tensor", "flops": f_fwd}]
    if with_bwd:
        pre_bytes = 2 * tok * Hq * d * 2 + tok * Hq * 4 + 2 * Hq * (tok + 128) * 4
        kernels += [{"kernel": "fa_bwd_pre_kernel", "ms": avg[1], "bound": "hbm", "bytes": pre_bytes},
                    {"kernel": "fa_bwd_dkdv_kernel", "ms": avg[2], "bound": "tensor", "flops": 2.0 * f_fwd},
                    {"kernel": "fa_bwd_dq_kernel", "ms": avg[3], "bound": "tensor", "flops": 1.5 * f_fwd}]
    for kk in kernels:
        if kk["bound"] == "tensor":
            kk["achieved_tflops"] = kk["flops"] / (kk["ms"] * 1e-3) / 1e12
            kk["frac"] = kk["achieved_tflops"] / pk["bf16_tflops"]
        else:
            kk["achieved_gbs"] = kk["bytes"] / (kk["ms"] * 1e-3) / 1e9
            kk["frac"] = kk["achieved_gbs"] / pk["hbm_gbs"]
    dom = max(kernels, key=lambda x: x["ms"])
    # the forward kernel's own roofline beside the dominant kernel's
    fk = kernels[0]
    forward = {"kernel": fk["kernel"], "bound": "tensor", "ms": fk["ms"], "achieved": fk["achieved_tflops"],
               "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": fk["frac"],
               "traffic": traffic_for(fk["kernel"], step_shape(B, Hq, Hkv, N, d, causal)),
               "peak_source": f"{pk['source']} bf16 burst (cuBLAS)"}
    if dom["bound"] == "tensor":
        roofline = {"bound": "tensor", "kernel": dom["kernel"], "achieved": dom["achieved_tflops"],
                    "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": dom["frac"],
                    "traffic": traffic_for(dom["kernel"], step_shape(B, Hq, Hkv, N, d, causal)),
                    "peak_source": f"{pk['source']} bf16 burst (cuBLAS)", "kernels": kernels}
    else:
        roofline = {"bound": "hbm", "kernel": dom["kernel"], "achieved": dom["achieved_gbs"],
                    "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": dom["frac"],
                    "traffic": traffic_for(dom["kernel"], step_shape(B, Hq, Hkv, N, d, causal)), "peak_source": f"{pk['source']} HBM copy",
                    "kernels": kernels}

    # end to end through the public API with host buffers (pinned), copies timed
    e2e = None
    if args.e2e_steps > 0:
        n_in = 4 if with_bwd else 3
        n_out = 5 if with_bwd else 2
        pin = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)][:n_in]
        ws_pair = [ws, torch.empty_like(ws)]

        def e2e_step(ins, outs, b):
            fa.fa_fwd(ins[0], ins[1], ins[2], outs[0], outs[1], B, Hq, Hkv, N, d, int(causal), scale, sptr)
            if with_bwd:
                fa.fa_bwd(ins[0], ins[1], ins[2], outs[0], outs[1], ins[3], outs[2], outs[3], outs[4], ws_pair[b],
                          ws_bytes, B, Hq, Hkv, N, d, int(causal), scale, sptr)

        e_ms, h2d, d2h = e2e_pipelined(torch, dev, stream, pin, [q, k, v, do][:n_in], [o, lse, dq, dk, dv][:n_out],
                                       e2e_step, args.e2e_steps, pg)
        if fa.fa_get_status(sptr) != fa.FA_OK:
            raise SystemExit("device status error in the end-to-end pass")
        e2e = {"value": f_step * world * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "overlap": E2E_OVERLAP}

    cpu = None
    if rank == 0 and world == 1:
        tf, heads, el, cores, unit = oracle_sample(args.cpu_budget_s, with_bwd)
        cpu = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{heads} units (unit: {unit}) of the workload's {B * Hq} (batch, head) problems, "
                         f"fp64 numpy, {'fwd+bwd' if with_bwd else 'fwd'}, {el:.1f} s"}

    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = dict(WORKLOAD)
    cfg["workload"] = WORKLOAD["workload"] if with_bwd else WORKLOAD["workload"].replace("fwd+bwd", "fwd")
    cfg.update({"parallelism": f"dp{world}" if world > 1 else "single", "l2": "flushed before every step",
                "global_batch": B * world})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": roofline, "forward_roofline": forward, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps if with_bwd else args.steps,
            "pct_of_peak": value / world / pk["bf16_tflops"]}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- decode workload

DEC_METRIC = "decode against a KV cache: GB/s of cache read (HBM-bound)"


def decode_shape(args):
    B, Nq, Hq, Hkv, Nc, d = (int(x) for x in args.decode_shape.split(","))
    cfg = {"workload": f"bf16 causal decode, B={B} Nq={Nq} Hq={Hq} Hkv={Hkv} Ncache={Nc} (full caches) d={d}",
           "B": B, "Nq": Nq, "Hq": Hq, "Hkv": Hkv, "Ncache": Nc, "d": d, "causal": True}
    # algorithmic bytes of one step: the K and V cache rows read once, the
    # query rows read and the output rows written (bf16), LSE written (fp32)
    byts = 2 * B * Nc * Hkv * d * 2 + 2 * B * Nq * Hq * d * 2 + B * Hq * Nq * 4
    return B, Nq, Hq, Hkv, Nc, d, cfg, byts


def decode_oracle_sample(args, budget_s):
    """Times the oracle on whole sequences of the decode workload until
    `budget_s` is spent; returns (GB/s of cache, sequences, seconds, cores)."""
    import numpy as np
    import oracle
    B, Nq, Hq, Hkv, Nc, d, cfg, byts = decode_shape(args)
    rng = np.random.default_rng(0)
    done, el, t_start = 0, 0.0, time.perf_counter()
    while done < B:
        q = rng.standard_normal((1, Nq, Hq, d), dtype=np.float32)
        k = rng.standard_normal((1, Nc, Hkv, d), dtype=np.float32)
        v = rng.standard_normal((1, Nc, Hkv, d), dtype=np.float32)
        t1 = time.perf_counter()
        oracle.attn_fwd_kvcache(q, k, v, np.array([Nc]), True, 1.0 / math.sqrt(d))
        el += time.perf_counter() - t1  # the oracle's time only, not the input draw
        done += 1
        if time.perf_counter() - t_start >= budget_s:
            break
    return byts / B * done / el / 1e9, done, el, oracle_threads()[0]


def run_decode_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    B, Nq, Hq, Hkv, Nc, d, cfg, byts = decode_shape(args)
    per_step_budget = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        r = decode_oracle_sample(args, per_step_budget)
        if i >= args.warmup:
            vals.append(r)
    gbs = sum(v[0] for v in vals) / len(vals)
    ms = sum(v[2] for v in vals) / len(vals) * 1e3
    sample = f"{vals[-1][1]} of {B} sequences per step, fp64 numpy (input draw not timed)"
    line = {"metric": DEC_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": dict(cfg, parallelism=f"replicas{args.gpus}", l2="n/a (CPU)"),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1], "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args):
    import torch
    world, rank, local = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    import synth
    B, Nq, Hq, Hkv, Nc, d, cfg, byts = decode_shape(args)
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator(device=dev)
    g.manual_seed(rank)
    # the cache is resident state of the decoder (drawn on the device); the
    # step's inputs are the new query rows and the cache lengths
    kc = torch.randn((B, Nc, Hkv, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((B, Nc, Hkv, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    import numpy as np
    q_h = synth.to_bf16(synth.normal_f32(np.random.default_rng(rank), (B, Nq, Hq, d)))
    lens_h = torch.full((B,), Nc, dtype=torch.int32)
    q, lens = q_h.to(dev), lens_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    splits = fa.fa_fwd_kvcache_num_splits(B, Hkv, Nc, d)
    ws_bytes = fa.fa_fwd_kvcache_workspace_size(B, Nq, Hq, d, splits)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    def step():
        fa.fa_fwd_kvcache(q, kc, vc, lens, o, lse, ws, ws_bytes, B, Nq, Hq, Hkv, Nc, d, 1, scale, splits, sptr)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error during warm-up")
    # The cache (B*Ncache*Hkv*d*4 bytes) is far larger than L2: steps run back
    # to back without a flush; events bracket every step.
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
    st = fa.fa_get_status(sptr)
    if st != fa.FA_OK:
        raise SystemExit(f"device status error: {fa.fa_status_string(st)}")
    tot_ms = ev[0].elapsed_time(ev[-1])
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    ms_per_step = tot_ms / args.steps
    value = byts * world * args.steps / (tot_ms * 1e-3) / 1e9
    pk = peaks()
    per_kernel = byts / (ms_per_step * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "fa_decode_kernel" + (" + fa_decode_merge_kernel" if splits > 1 else ""),
                "achieved": per_kernel, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": per_kernel / pk["hbm_gbs"],
                "traffic": traffic_for("fa_decode_kernel", decode_shape_key(B, Nq, Hq, Hkv, Nc, d)), "peak_source": f"{pk['source']} HBM copy",
                "bytes_per_launch": byts, "num_splits": splits}
    e2e = None
    if args.e2e_steps > 0:
        q_pin, lens_pin = q_h.pin_memory(), lens_h.pin_memory()
        o_pin = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lse_pin = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            q.copy_(q_pin, non_blocking=True)
            lens.copy_(lens_pin, non_blocking=True)
            step()
            o_pin.copy_(o, non_blocking=True)
            lse_pin.copy_(lse, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(pg, dev, e_ms)
        e2e = {"value": byts * world * args.e2e_steps / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": q_pin.numel() * 2 + lens_pin.numel() * 4,
               "d2h_bytes_per_step": o_pin.numel() * 2 + lse_pin.numel() * 4,
               "note": "the KV cache is resident decoder state; the step's inputs are q and the cache lengths"}
    cpu = None
    if rank == 0 and world == 1:
        gbs, seqs, el, cores = decode_oracle_sample(args, args.cpu_budget_s)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{seqs} of {B} sequences of the workload, fp64 numpy, {el:.1f} s"}
    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg.update({"parallelism": f"dp{world}" if world > 1 else "single",
                "l2": "inputs larger than L2 (cache %.2f GB), no flush" % (2 * B * Nc * Hkv * d * 2 / 1e9),
                "global_batch": B * world})
    line = {"metric": DEC_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": args.steps * (2 if splits > 1 else 1)}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- ring workload

RING_METRIC = "context-parallel ring attention forward TFLOP/s (bf16, causal)"


def run_ring(args):
    import torch
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_ring_reference(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    from io_aware_exact_27_b200 import ring as rg
    import synth
    B, Hq, Hkv, N, d = (int(x) for x in args.ring_shape.split(","))
    R = world if world > 1 else args.ring_ranks
    n = N // R
    if n * R != N:
        raise SystemExit("N must split evenly over the ring")
    scale = 1.0 / math.sqrt(d)
    # this process's ranks: its own one (NCCL ring) or all R (emulated)
    mine = [rank] if world > 1 else list(range(R))
    q_h, k_h, v_h = synth.qkv_bf16(0, B, N, Hq, Hkv, d)
    sh = lambda t, r: t[:, r * n:(r + 1) * n].contiguous()  # noqa: E731
    qs = {r: sh(q_h, r).to(dev) for r in range(R)}
    ks = {r: sh(k_h, r).to(dev) for r in range(R)}
    vs = {r: sh(v_h, r).to(dev) for r in range(R)}
    stream = torch.cuda.current_stream(dev)
    rec = []  # (start, end, flops) of every forward-kernel launch of a timed step
    recm = []  # (start, end) of every merge step (a launch for ranks with more than one block)
    timing = {"on": False}

    def rank_fns(r):
        g = rg._gpu_rank(qs[r], r, R, True, scale)

        def blk(qq, kk, vv, c):
            if timing["on"]:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            out = g.block(qq, kk, vv, c)
            if timing["on"]:
                e1.record(stream)
                rec.append((e0, e1, fwd_flops(B, Hq, n, d, c)))
            return out

        def merge(o_t, lse_t, first, last):
            if timing["on"]:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            out = g.merge(o_t, lse_t, first, last)
            if timing["on"]:
                e1.record(stream)
                recm.append((e0, e1))
            return out
        return blk, merge

    def step():
        res = []
        for r in mine:
            if world > 1:
                blocks = rg.ring_exchange(ks[r], vs[r])
            else:
                blocks = (((r - t) % R, ks[(r - t) % R], vs[(r - t) % R]) for t in range(R))
            blk, merge = rank_fns(r)
            res.append(rg.ring_forward(qs[r], blocks, r, R, True, blk, merge))
        return res

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status() != fa.FA_OK:
        raise SystemExit("device status error during warm-up")
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    e_beg, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    timing["on"] = True
    with ClockSampler(local) as clk:
        e_beg.record(stream)
        for _ in range(args.steps):
            step()
        e_end.record(stream)
        torch.cuda.synchronize(dev)
    timing["on"] = False
    tot_ms = e_beg.elapsed_time(e_end)
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    f_job = fwd_flops(B, Hq, N, d, True)  # the whole sequence's causal attention
    value = f_job * args.steps / (tot_ms * 1e-3) / 1e12
    k_ms = sum(a.elapsed_time(b) for a, b, _ in rec)
    k_fl = sum(f for _, _, f in rec)
    m_ms = sum(a.elapsed_time(b) for a, b in recm)
    pk = peaks()
    achieved = k_fl / (k_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "fa_fwd_sm100_kernel", "achieved": achieved, "peak": pk["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                "peak_source": f"{pk['source']} bf16 burst (cuBLAS)",
                "launches": len(rec), "kernel_ms_per_step": k_ms / args.steps,
                "merge_ms_per_step": m_ms / args.steps,
                "note": "per-launch flops: a full n x n block 4*B*Hq*n^2*d, the causal diagonal block half of it"}
    clocks = clk.summary()
    # the ring backward on the same shards (dO drawn after Q, K, V), timed on its own
    bwd = None
    if not args.no_bwd:
        do_h = synth.qkv_bf16(0, B, N, Hq, Hkv, d, with_dout=True)[3]
        dos = {r: sh(do_h, r).to(dev) for r in range(R)}
        fw = step()
        outs = dict(zip(mine, fw))

        def bstep():
            if world > 1:
                return [rg.ring_attention_bwd(qs[rank], ks[rank], vs[rank], outs[rank][0], outs[rank][1],
                                              dos[rank], causal=True, scale=scale)]
            return rg.ring_attention_bwd_local([qs[r] for r in range(R)], [ks[r] for r in range(R)],
                                               [vs[r] for r in range(R)], [outs[r][0] for r in range(R)],
                                               [outs[r][1] for r in range(R)], [dos[r] for r in range(R)],
                                               causal=True, scale=scale)
        for _ in range(max(1, args.warmup)):
            bstep()
        torch.cuda.synchronize(dev)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            bstep()
        b1.record(stream)
        torch.cuda.synchronize(dev)
        b_ms = b0.elapsed_time(b1)
        b_ms = max_over_ranks(pg, dev, b_ms)
        bwd = {"ms_per_step": b_ms / args.steps,
               "tflops": 2.5 * f_job * args.steps / (b_ms * 1e-3) / 1e12,
               "note": "ring backward timed separately: flops 2.5x the forward (five GEMMs)"}
        if fa.fa_get_status() != fa.FA_OK:
            raise SystemExit("device status error in the ring backward")
    # end to end: this process's shards copied in from pinned host memory,
    # its O and LSE copied out, every step
    e2e = None
    if args.e2e_steps > 0:
        pin = {r: [sh(t, r).pin_memory() for t in (q_h, k_h, v_h)] for r in mine}
        outs_h = {r: (torch.empty((B, n, Hq, d), dtype=torch.bfloat16).pin_memory(),
                      torch.empty((B, Hq, n), dtype=torch.float32).pin_memory()) for r in mine}
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for r in mine:
                qs[r].copy_(pin[r][0], non_blocking=True)
                ks[r].copy_(pin[r][1], non_blocking=True)
                vs[r].copy_(pin[r][2], non_blocking=True)
            res = step()
            for r, (o_r, l_r) in zip(mine, res):
                outs_h[r][0].copy_(o_r, non_blocking=True)
                outs_h[r][1].copy_(l_r, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(pg, dev, e_ms)
        h2d = sum(x.numel() * x.element_size() for r in mine for x in pin[r])
        d2h = sum(x.numel() * x.element_size() for r in mine for x in outs_h[r])
        e2e = {"value": f_job * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and world == 1:
        tf, rows, el, cores = ring_oracle_sample(args, args.cpu_budget_s)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{rows} query rows of head 0, fp64 numpy, {el:.1f} s"}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = {"workload": f"bf16 causal ring attention forward, B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}, "
                       f"{R} ranks of {n} tokens" + (" (emulated on one GPU)" if world == 1 else ""),
           "B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "ring_ranks": R,
           "parallelism": f"cp{world}" if world > 1 else f"cp{R} emulated", "l2": "no flush (whole-job timing)"}
    line = {"metric": RING_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "backward": bwd,
            "gpu_launches": len(rec) + len(recm)}
    print(json.dumps(line), flush=True)
    return 0


def ring_oracle_sample(args, budget_s):
    """The oracle on sampled query rows of the ring workload (full sequence)."""
    import numpy as np
    import oracle
    import synth
    B, Hq, Hkv, N, d = (int(x) for x in args.ring_shape.split(","))
    q, k, v = synth.qkv_bf16(0, 1, N, Hq, Hkv, d)
    rng = np.random.default_rng(2)
    done, el = 0, 0.0
    flops = 0.0
    while el < budget_s and done < N:
        rows = np.sort(rng.choice(N, size=64, replace=False))
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(q[:, :, :1], k[:, :, :1], v[:, :, :1], True, 1 / math.sqrt(d), rows[None, :])
        el += time.perf_counter() - t0
        flops += float(sum(4.0 * (r + 1) * d for r in rows))
        done += 64
    return flops / el / 1e12, done, el, oracle_threads()[0]


def run_ring_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    per = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    vals = [ring_oracle_sample(args, per) for _ in range(args.warmup + args.steps)][args.warmup:]
    tf = sum(v[0] for v in vals) / len(vals)
    B, Hq, Hkv, N, d = (int(x) for x in args.ring_shape.split(","))
    line = {"metric": RING_METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(v[2] for v in vals) / len(vals) * 1e3,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"bf16 causal ring attention forward, B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}",
                       "parallelism": f"replicas{args.gpus}", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1],
                             "sample": f"{vals[-1][1]} query rows of head 0 per step, fp64 numpy"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- fp8 workload

FP8_METRIC = "fp8 attention forward TFLOP/s (e4m3, Hadamard-rotated Q/K, causal)"
FP8_SHAPE = (2, 16, 8192, 128)  # B, H, N, d


def fp8_inputs(seed=0):
    """Q, K, V as fp32 with 0.1% of entries x20 (outlier channels), drawn in
    the order Q, K, V, and their bf16 roundings (what the quantiser reads)."""
    import numpy as np
    import synth
    B, H, N, d = FP8_SHAPE
    rng = np.random.default_rng(seed)
    f32 = []
    for _ in range(3):
        x = synth.normal_f32(rng, (B, N, H, d))
        x = np.where(rng.random(size=x.shape) < 1e-3, x * np.float32(20.0), x).astype(np.float32)
        f32.append(x)
    return f32, [synth.to_bf16(x) for x in f32]


def fp8_sample_rows(N, count=64, seed=2):
    import numpy as np
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=count - 2, replace=False).tolist()) | {0, N - 1}
    return np.array(sorted(rows))


def run_fp8(args):
    import numpy as np
    import torch
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_fp8_reference(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    import oracle
    B, H, N, d = FP8_SHAPE
    f32, bf = fp8_inputs(rank)
    q, k, v = (t.to(dev) for t in bf)
    scale = 1.0 / math.sqrt(d)
    nblk = (N + 127) // 128
    codes = [torch.empty((B, N, H, d), dtype=torch.float8_e4m3fn, device=dev) for _ in range(3)]
    scl = [torch.empty((B, H, nblk), dtype=torch.float32, device=dev) for _ in range(3)]
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def quantize(rotate_qk=True):
        for i, (x, rot) in enumerate(((q, rotate_qk), (k, rotate_qk), (v, False))):
            fa.fa_fp8_quantize(x, codes[i], scl[i], B, N, H, d, int(rot), sptr)

    def forward():
        fa.fa_fwd_fp8(codes[0], codes[1], codes[2], scl[0], scl[1], scl[2], o, lse, B, H, H, N, d, 1, scale, sptr)

    # the training step's backward, timed apart: dequantise Q, K (rotation
    # undone) and V for the 16-bit products, then fa_bwd_fp8 (scores on the
    # codes) with the fp8 forward's O and LSE
    import synth
    do = synth.qkv_bf16(rank + 200, B, N, H, H, d, with_dout=True)[3].to(dev)
    deq = [torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    grads = [torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    ws_bytes = fa.fa_bwd_workspace_size(B * N, B, H, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def backward():
        for i, rot in enumerate((True, True, False)):
            fa.fa_fp8_dequantize(codes[i], scl[i], deq[i], B, N, H, d, int(rot), sptr)
        fa.fa_bwd_fp8(codes[0], codes[1], scl[0], scl[1], deq[0], deq[1], deq[2], o, lse, do, grads[0], grads[1],
                      grads[2], ws, ws_bytes, B, H, H, N, d, 1, scale, sptr)

    # error against fp64 attention on the unquantised fp32 values (sampled rows)
    rows = fp8_sample_rows(N)
    rows_h = np.tile(rows[None, :], (H, 1))
    O_ref, _ = oracle.attn_fwd_rows(f32[0][:1], f32[1][:1], f32[2][:1], True, scale, rows_h)
    errs = {}
    for rot in (False, True):
        quantize(rot)
        forward()
        torch.cuda.synchronize(dev)
        got = o[:1].cpu().double().numpy()[:, rows].transpose(0, 2, 1, 3)  # [1,H,R,d]
        errs["rotated" if rot else "plain"] = oracle.rel_rms(got, O_ref)

    for _ in range(args.warmup):
        quantize()
        forward()
        backward()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            quantize()
            ev[i][1].record(stream)
            forward()
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
    st = fa.fa_get_status(sptr)
    if st != fa.FA_OK:
        raise SystemExit(f"device status error: {fa.fa_status_string(st)}")
    q_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    f_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    tot_ms = (q_ms + f_ms) * args.steps
    bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for b0, b1 in bev:
        flush.zero_()
        b0.record(stream)
        backward()
        b1.record(stream)
    torch.cuda.synchronize(dev)
    b_ms = sum(b0.elapsed_time(b1) for b0, b1 in bev) / args.steps
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error in the backward")
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    flops = fwd_flops(B, H, N, d, True)
    value = flops * world * args.steps / (tot_ms * 1e-3) / 1e12
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    ach = flops / (f_ms * 1e-3) / 1e12
    q_bytes = 3 * B * N * H * d * (2 + 1) + 3 * B * H * nblk * 4
    roofline = {"bound": "tensor", "kernel": "fa_fwd_sm100_kernel (fp8)", "achieved": ach, "peak": fp8_peak,
                "unit": "TFLOP/s", "frac": ach / fp8_peak,
                "traffic": traffic_for("fa_fwd_sm100_kernel", "fp8 " + step_shape(B, H, H, N, d, True)),
                "peak_source": f"{pk['source']} bf16 burst x 2 (nominal e4m3/bf16 ratio)",
                "note": "S = Q K^T runs at the e4m3 rate, O += P V at the 16-bit rate (P and V as f16): "
                        "at most 4/3 of the bf16 peak for this kernel",
                "quantize_ms": q_ms, "forward_ms": f_ms,
                "quantize_gbs": q_bytes / (q_ms * 1e-3) / 1e9, "quantize_frac_hbm": q_bytes / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    e2e = None
    if args.e2e_steps > 0:
        pin = [t.pin_memory() for t in bf]
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        l_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for x, hsrc in zip((q, k, v), pin):
                x.copy_(hsrc, non_blocking=True)
            quantize()
            forward()
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(pg, dev, e_ms)
        e2e = {"value": flops * world * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * 2 for x in pin),
               "d2h_bytes_per_step": o_h.numel() * 2 + l_h.numel() * 4}
    cpu = None
    if rank == 0 and world == 1:
        tf, nr, el, cores = fp8_oracle_sample(args.cpu_budget_s)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{nr} (head, query row) pairs of the workload, fp64 numpy, {el:.1f} s"}
    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = {"workload": f"fp8-e4m3 causal forward from bf16 inputs with 0.1% outliers x20, B={B} Hq=Hkv={H} N={N} "
                       f"d={d}: Q, K rotated by H_d/sqrt(d), per-(head,128-row block) scales",
           "B": B, "Hq": H, "Hkv": H, "N": N, "d": d, "causal": True,
           "parallelism": f"dp{world}" if world > 1 else "single", "l2": "flushed before every step",
           "error_vs_fp64_unquantised": errs, "error_sample": f"{len(rows)} query rows x {H} heads of batch 0"}
    line = {"metric": FP8_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": 4 * args.steps,
            "backward": {"ms": b_ms, "tflops": 2.5 * flops / (b_ms * 1e-3) / 1e12,
                         "note": "fa_fp8_dequantize x3 (Q, K unrotated) + fa_bwd_fp8 (scores on the e4m3 codes, "
                                 "the other products 16-bit) with the fp8 forward's O and LSE, timed apart, per GPU; "
                                 "flops 2.5x the forward's"}}
    print(json.dumps(line), flush=True)
    return 0


def fp8_oracle_sample(budget_s):
    """The oracle's rotation + quantisation + attention on sampled query rows
    of one head until `budget_s` is spent: (TFLOP/s, rows, seconds, cores)."""
    import numpy as np
    import oracle
    B, H, N, d = FP8_SHAPE
    f32, _ = fp8_inputs(0)
    q, k, v = (x[:1, :, :1] for x in f32)
    done, el, flops = 0, 0.0, 0.0
    rng = np.random.default_rng(3)
    while el < budget_s and done < N:
        rows = np.sort(rng.choice(N, size=64, replace=False))
        t0 = time.perf_counter()
        cq, sq = oracle.quantize_blockscaled(oracle.rotate_f32(q))
        ck, sk = oracle.quantize_blockscaled(oracle.rotate_f32(k))
        cv, sv = oracle.quantize_blockscaled(v)
        oracle.attn_fwd_rows(oracle.dequantize_blockscaled(cq, sq), oracle.dequantize_blockscaled(ck, sk),
                             oracle.dequantize_blockscaled(cv, sv), True, 1 / math.sqrt(d), rows[None, :])
        el += time.perf_counter() - t0
        flops += float(sum(4.0 * (r + 1) * d for r in rows))
        done += 64
    return flops / el / 1e12, done, el, oracle_threads()[0]


def run_fp8_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    per = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    vals = [fp8_oracle_sample(per) for _ in range(args.warmup + args.steps)][args.warmup:]
    tf = sum(v[0] for v in vals) / len(vals)
    B, H, N, d = FP8_SHAPE
    line = {"metric": FP8_METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(v[2] for v in vals) / len(vals) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"fp8-e4m3 causal forward, B={B} Hq=Hkv={H} N={N} d={d}, rotated Q/K",
                       "parallelism": f"replicas{args.gpus}", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1],
                             "sample": f"{vals[-1][1]} query rows of one head per step, fp64 numpy"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- block-sparse workload

BS_METRIC = "block-sparse attention forward TFLOP/s over the visible query-key pairs (bf16, causal)"
BS_SHAPE = (1, 32, 8, 16384, 128)  # B, Hq, Hkv, N, d
BS_WINDOW = 8  # key blocks of the sliding window (the query's own block and the 7 before it)


def bs_mask(Hq, nb):
    """Sliding window of BS_WINDOW blocks plus block 0 (a global first block), every head."""
    import numpy as np
    m = np.zeros((Hq, nb, nb), dtype=np.uint8)
    for i in range(nb):
        m[:, i, max(0, i - BS_WINDOW + 1):i + 1] = 1
        m[:, i, 0] = 1
    return m


def bs_pairs(mask, N, causal=True):
    """Visible (query, key) pairs of one head under the block mask (and causal)."""
    import numpy as np
    nb = mask.shape[1]
    pairs = 0
    for i in range(nb):
        for j in range(nb):
            if not mask[0, i, j]:
                continue
            qi = np.arange(i * 128, min(N, (i + 1) * 128))
            kj = np.arange(j * 128, min(N, (j + 1) * 128))
            pairs += int((kj[None, :] <= qi[:, None]).sum()) if causal else qi.size * kj.size
    return pairs


def run_blocksparse(args):
    import numpy as np
    import torch
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_bs_reference(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    import synth
    B, Hq, Hkv, N, d = BS_SHAPE
    nb = (N + 127) // 128
    mask_h = bs_mask(Hq, nb)
    pairs = bs_pairs(mask_h, N)
    flops = 4.0 * d * pairs * Hq * B
    q_h, k_h, v_h = synth.qkv_bf16(rank, B, N, Hq, Hkv, d)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    mask = torch.from_numpy(mask_h).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        fa.fa_fwd_blocksparse(q, k, v, mask, o, lse, B, Hq, Hkv, N, d, 1, scale, sptr)

    def dense():
        fa.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, 1, scale, sptr)

    # the training step's backward over the same mask, timed apart (and the
    # dense causal backward beside it); flops 2.5x the forward's (five GEMMs)
    do = synth.qkv_bf16(rank + 100, B, N, Hq, Hkv, d, with_dout=True)[3].to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa.fa_bwd_blocksparse_workspace_size(B, Hq, Hkv, N, d)  # >= the dense backward's
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    o_bs = torch.empty_like(q)
    lse_bs = torch.empty_like(lse)
    o_dn = torch.empty_like(q)
    lse_dn = torch.empty_like(lse)
    fa.fa_fwd_blocksparse(q, k, v, mask, o_bs, lse_bs, B, Hq, Hkv, N, d, 1, scale, sptr)
    fa.fa_fwd(q, k, v, o_dn, lse_dn, B, Hq, Hkv, N, d, 1, scale, sptr)

    def bwd_step():
        fa.fa_bwd_blocksparse(q, k, v, mask, o_bs, lse_bs, do, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, N, d, 1, scale,
                              sptr)

    def bwd_dense():
        fa.fa_bwd(q, k, v, o_dn, lse_dn, do, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, N, d, 1, scale, sptr)

    def timed(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs)

    for _ in range(args.warmup):
        step()
        dense()
        bwd_step()
        bwd_dense()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error during warm-up")
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        tot_ms = timed(step, args.steps)
    dense_ms = timed(dense, args.steps) / args.steps
    b_ms = timed(bwd_step, args.steps) / args.steps
    bd_ms = timed(bwd_dense, args.steps) / args.steps
    bwd = {"ms": b_ms, "tflops": 2.5 * flops / (b_ms * 1e-3) / 1e12, "dense_causal_ms": bd_ms,
           "speedup_vs_dense_causal": bd_ms / b_ms,
           "note": "fa_bwd_blocksparse (pre + dK/dV + dQ) on the same mask, per GPU; flops 2.5x the forward's"}
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    ms = tot_ms / args.steps
    value = flops * world / (ms * 1e-3) / 1e12
    pk = peaks()
    roofline = {"bound": "tensor", "kernel": "fa_fwd_sm100_kernel (block-sparse)", "achieved": value / world,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": value / world / pk["bf16_tflops"],
                "traffic": None, "peak_source": f"{pk['source']} bf16 burst (cuBLAS)",
                "note": "flops of the visible (query, key) pairs, 4*d each",
                "dense_causal_ms": dense_ms, "speedup_vs_dense_causal": dense_ms / ms,
                "pair_density_vs_causal": pairs / (N * (N + 1) / 2)}
    e2e = None
    if args.e2e_steps > 0:
        pin = [t.pin_memory() for t in (q_h, k_h, v_h)]
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        l_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for x, hsrc in zip((q, k, v), pin):
                x.copy_(hsrc, non_blocking=True)
            step()
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e2e = {"value": flops * world * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * 2 for x in pin),
               "d2h_bytes_per_step": o_h.numel() * 2 + l_h.numel() * 4}
    cpu = None
    if rank == 0 and world == 1:
        tf, nr, el, cores = bs_oracle_sample(args.cpu_budget_s)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{nr} query rows of head 0, fp64 numpy, {el:.1f} s"}
    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = {"workload": f"bf16 causal block-sparse forward, B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}: every query "
                       f"block sees its own and the {BS_WINDOW - 1} previous key blocks plus block 0",
           "B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "parallelism": f"dp{world}" if world > 1 else "single",
           "l2": "flushed before every step"}
    line = {"metric": BS_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": args.steps, "backward": bwd}
    print(json.dumps(line), flush=True)
    return 0


def bs_oracle_sample(budget_s):
    """The oracle's block-masked attention on sampled query rows of head 0."""
    import numpy as np
    import oracle
    import synth
    B, Hq, Hkv, N, d = BS_SHAPE
    q, k, v = synth.qkv_bf16(0, 1, N, 1, 1, d)
    q, k, v = (t.double().numpy() for t in (q, k, v))
    nb = (N + 127) // 128
    m = bs_mask(1, nb)[0]
    rng = np.random.default_rng(5)
    done, el, flops = 0, 0.0, 0.0
    blk = np.arange(N) // 128
    while el < budget_s and done < N:
        rows = rng.choice(N, size=32, replace=False)
        t0 = time.perf_counter()
        for i in rows:
            keys = np.nonzero((m[blk[i]][blk] != 0) & (np.arange(N) <= i))[0]
            s = (q[0, i, 0] @ k[0, keys, 0].T) / math.sqrt(d)
            p = np.exp(s - s.max())
            _ = (p / p.sum()) @ v[0, keys, 0]
            flops += 4.0 * d * keys.size
        el += time.perf_counter() - t0
        done += 32
    return flops / el / 1e12, done, el, oracle_threads()[0]


def run_bs_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    per = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    vals = [bs_oracle_sample(per) for _ in range(args.warmup + args.steps)][args.warmup:]
    tf = sum(v[0] for v in vals) / len(vals)
    B, Hq, Hkv, N, d = BS_SHAPE
    line = {"metric": BS_METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(v[2] for v in vals) / len(vals) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"bf16 causal block-sparse forward, B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}",
                       "parallelism": f"replicas{args.gpus}", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1],
                             "sample": f"{vals[-1][1]} query rows of head 0 per step, fp64 numpy"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- sweep over N

SWEEP_TOKENS = 32768
SWEEP_NS = (2048, 4096, 8192, 16384, 32768)
SWEEP_H, SWEEP_D = 16, 128
TINY = (1, 2, 2, 256, 64, False)  # B, Hq, Hkv, N, d, causal


def sweep_workload(N):
    return {"B": SWEEP_TOKENS // N, "Hq": SWEEP_H, "Hkv": SWEEP_H, "N": N, "d": SWEEP_D, "causal": True}


def run_sweep(args):
    """Causal fwd+bwd at every N of SWEEP_NS (B = 32K / N tokens, H=16,
    d=128), each timed on its own (L2 flushed before every step), and the tiny
    non-causal case (launch-bound: microseconds and GB/s). One step of the
    line = one fwd+bwd at every N; the value is the flops of that step over
    its time."""
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        if rank != 0:
            return 0
        budget = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
        vals = [oracle_sample(budget, True, sweep_workload(SWEEP_NS[0])) for _ in range(args.warmup + args.steps)]
        vals = vals[args.warmup:]
        tf = sum(v[0] for v in vals) / len(vals)
        sample = f"{vals[0][1]} (batch, head) problems of the N=2048 point per step, fp64 numpy, fwd+bwd"
        print(json.dumps({"metric": METRIC + " (sweep)", "value": tf, "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "impl": "reference",
                          "config": {"workload": f"causal attention fwd+bwd sweep, N in {list(SWEEP_NS)}, "
                                                 f"B*N = {SWEEP_TOKENS}, Hq=Hkv={SWEEP_H}, d={SWEEP_D}"},
                          "cpu_baseline": {"value": tf, "unit": UNIT, "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1],
                                           "sample": sample},
                          "e2e": {"value": tf, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return 0
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    import synth
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    pk = peaks()

    def time_point(B, Hq, Hkv, N, d, causal):
        q, k, v, do = (t.to(dev) for t in synth.qkv_bf16(rank, B, N, Hq, Hkv, d, with_dout=True))
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        wsb = fa.fa_bwd_workspace_size(B * N, B, Hq, d)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        scale = 1.0 / math.sqrt(d)
        fwd = lambda: fa.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, int(causal), scale, sptr)
        bwd = lambda: fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, wsb, B, Hq, Hkv, N, d, int(causal), scale, sptr)
        for _ in range(args.warmup):
            fwd()
            bwd()
        ms = []
        for with_bwd in (False, True):
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record(stream)
                fwd()
                if with_bwd:
                    bwd()
                ev[i][1].record(stream)
            torch.cuda.synchronize(dev)
            ms.append(sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps)
        if fa.fa_get_status(sptr) != fa.FA_OK:
            raise SystemExit(f"device status error at N={N}")
        return ms[0], ms[1]

    steps = max(3, min(args.steps, 20))
    args.steps = steps
    points, tot_flops, tot_ms = [], 0.0, 0.0
    if pg:
        pg.barrier()
    with ClockSampler(local) as clk:
        for N in SWEEP_NS:
            w = sweep_workload(N)
            f = fwd_flops(w["B"], w["Hq"], N, w["d"], True)
            ms_f, ms_s = time_point(w["B"], w["Hq"], w["Hkv"], N, w["d"], True)
            points.append({"N": N, "B": w["B"], "fwd_ms": ms_f, "step_ms": ms_s,
                           "fwd_tflops": f / (ms_f * 1e-3) / 1e12,
                           "bwd_tflops": 2.5 * f / ((ms_s - ms_f) * 1e-3) / 1e12,
                           "step_tflops": 3.5 * f / (ms_s * 1e-3) / 1e12,
                           "fwd_frac": f / (ms_f * 1e-3) / 1e12 / pk["bf16_tflops"]})
            tot_flops += 3.5 * f
            tot_ms += ms_s
            torch.cuda.empty_cache()
        B, Hq, Hkv, N, d, causal = TINY
        ms_f, ms_s = time_point(B, Hq, Hkv, N, d, causal)
    tiny_bytes = (2 * B * N * Hq * d + 2 * B * N * Hkv * d) * 2 + B * Hq * N * 4  # Q, K, V read; O, LSE written
    tiny = {"B": B, "Hq": Hq, "N": N, "d": d, "causal": causal, "fwd_us": ms_f * 1e3, "step_us": ms_s * 1e3,
            "fwd_gbs": tiny_bytes / (ms_f * 1e-3) / 1e9}
    tot_ms = max_over_ranks(pg, dev, tot_ms)
    value = tot_flops * world / (tot_ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1:
        tf, heads, el, cores, _ = oracle_sample(args.cpu_budget_s, True, sweep_workload(SWEEP_NS[0]))
        cpu = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{heads} (batch, head) problems of the N=2048 point, fp64 numpy, fwd+bwd, {el:.1f} s"}
    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    p16 = next(p for p in points if p["N"] == 16384)
    roofline = {"bound": "tensor", "kernel": "fa_fwd_sm100_kernel (N=16384 point)", "achieved": p16["fwd_tflops"],
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": p16["fwd_frac"], "traffic": None,
                "peak_source": f"{pk['source']} bf16 burst (cuBLAS)"}
    cfg = {"workload": f"bf16 causal attention fwd+bwd sweep, N in {list(SWEEP_NS)} at B*N = {SWEEP_TOKENS} "
                       f"tokens, Hq=Hkv={SWEEP_H}, d={SWEEP_D}; plus B=1 H=2 N=256 d=64 non-causal",
           "parallelism": f"dp{world}" if world > 1 else "single", "l2": "flushed before every step"}
    line = {"metric": METRIC + " (sweep)", "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": tot_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": None, "clocks": clocks,
            "gpu_launches": 4 * steps * (len(SWEEP_NS) + 1) + steps * (len(SWEEP_NS) + 1),
            "points": points, "tiny": tiny}
    print(json.dumps(line), flush=True)
    return 0



# ----------------------------------------------------------------- varlen (packed sequences)

VARLEN_H, VARLEN_D = 16, 128


def varlen_flops(lengths, H, d):
    return sum(4.0 * H * int(n) * int(n) * d / 2.0 for n in lengths)  # causal forward


def varlen_oracle_sample(budget_s, lengths, cu):
    """The fp64 oracle on whole (sequence, head) problems of the packed batch,
    fwd+bwd, until `budget_s` is spent; returns (TFLOP/s, problems, seconds, cores)."""
    import oracle
    import synth
    q, k, v, do, _ = synth.qkv_varlen_bf16(0, lengths, VARLEN_H, VARLEN_H, VARLEN_D, with_dout=True)
    scale = 1.0 / math.sqrt(VARLEN_D)
    done, flops, t0 = 0, 0.0, time.perf_counter()
    while done < len(lengths) * VARLEN_H:
        i, h = divmod(done, VARLEN_H)
        a, b = int(cu[i]), int(cu[i + 1])
        sl = (None, slice(a, b), slice(h, h + 1))
        oracle.attn_fwd(q[sl], k[sl], v[sl], True, scale)
        oracle.attn_bwd(q[sl], k[sl], v[sl], do[sl], True, scale)
        flops += 3.5 * varlen_flops([b - a], 1, VARLEN_D)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return flops / el / 1e12, done, el, oracle_threads()[0]


def run_varlen(args):
    """Packed causal fwd+bwd over 24 sequences of U[128, 4096] tokens (seeded:
    T = 52,929), Hq = Hkv = 16, d = 128, through fa_fwd_varlen / fa_bwd_varlen;
    L2 flushed before every step; the forward timed alone in a second pass."""
    import synth
    world, rank, local = dist_setup(args)
    lengths = synth.varlen_lengths(rank)
    cu_h = synth.cu_seqlens_of(lengths)
    T, mx = int(cu_h[-1]), int(lengths.max())
    f = varlen_flops(lengths, VARLEN_H, VARLEN_D)
    wl = (f"bf16 causal varlen attention fwd+bwd, {len(lengths)} sequences of U[128,4096] tokens "
          f"(T={T}), Hq=Hkv={VARLEN_H}, d={VARLEN_D}")
    if args.impl == "reference":
        if rank != 0:
            return 0
        budget = max(0.5, min(args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
        vals = [varlen_oracle_sample(budget, lengths, cu_h) for _ in range(args.warmup + args.steps)][args.warmup:]
        tf = sum(v[0] for v in vals) / len(vals)
        print(json.dumps({"metric": METRIC + " (varlen)", "value": tf, "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "impl": "reference", "config": {"workload": wl},
                          "cpu_baseline": {"value": tf, "unit": UNIT, "cores": vals[-1][3], "kind": "oracle", "blas": oracle_threads()[1],
                                           "sample": f"{vals[0][1]} (sequence, head) problems per step, fp64 "
                                                     f"numpy, fwd+bwd"},
                          "e2e": {"value": tf, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return 0
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist
    import io_aware_exact_27_b200 as fa
    H, d = VARLEN_H, VARLEN_D
    q_h, k_h, v_h, do_h, _ = synth.qkv_varlen_bf16(rank, lengths, H, H, d, with_dout=True)
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    cu = torch.from_numpy(cu_h).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nseq = len(lengths)
    wsb = fa.fa_bwd_workspace_size(T, nseq, H, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    scale = 1.0 / math.sqrt(d)
    fwd = lambda: fa.fa_fwd_varlen(q, k, v, o, lse, cu, nseq, mx, T, H, H, d, 1, scale, sptr)
    bwd = lambda: fa.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, ws, wsb, cu, nseq, mx, T, H, H, d, 1, scale,
                                   sptr)
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error during warm-up")
    if pg:
        pg.barrier()
    ms = []
    with ClockSampler(local) as clk:
        for with_bwd in (True, False):
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record(stream)
                fwd()
                if with_bwd:
                    bwd()
                ev[i][1].record(stream)
            torch.cuda.synchronize(dev)
            ms.append(sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps)
    if fa.fa_get_status(sptr) != fa.FA_OK:
        raise SystemExit("device status error")
    ms_s, ms_f = ms
    ms_s, ms_f = max_over_ranks(pg, dev, ms_s), max_over_ranks(pg, dev, ms_f)
    value = 3.5 * f * world / (ms_s * 1e-3) / 1e12
    pk = peaks()
    fwd_tf = f / (ms_f * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "fa_fwd_sm100_kernel (varlen)", "achieved": fwd_tf,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": fwd_tf / pk["bf16_tflops"], "traffic": None,
                "peak_source": f"{pk['source']} bf16 burst (cuBLAS)",
                "backward_tflops": 2.5 * f / ((ms_s - ms_f) * 1e-3) / 1e12}
    e2e = None
    if args.e2e_steps > 0:
        pin = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)]
        ws_pair = [ws, torch.empty_like(ws)]

        def e2e_step(ins, outs, b):
            fa.fa_fwd_varlen(ins[0], ins[1], ins[2], outs[0], outs[1], cu, nseq, mx, T, H, H, d, 1, scale, sptr)
            fa.fa_bwd_varlen(ins[0], ins[1], ins[2], outs[0], outs[1], ins[3], outs[2], outs[3], outs[4], ws_pair[b],
                             wsb, cu, nseq, mx, T, H, H, d, 1, scale, sptr)

        e_ms, h2d, d2h = e2e_pipelined(torch, dev, stream, pin, [q, k, v, do], [o, lse, dq, dk, dv], e2e_step,
                                       args.e2e_steps, pg)
        if fa.fa_get_status(sptr) != fa.FA_OK:
            raise SystemExit("device status error in the end-to-end pass")
        e2e = {"value": 3.5 * f * world * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "overlap": E2E_OVERLAP}
    cpu = None
    if rank == 0 and world == 1:
        tf, n, el, cores = varlen_oracle_sample(args.cpu_budget_s, lengths, cu_h)
        cpu = {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "blas": oracle_threads()[1],
               "sample": f"{n} of {nseq * H} (sequence, head) problems, fp64 numpy, fwd+bwd, {el:.1f} s"}
    clocks = clk.summary()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    cfg = {"workload": wl, "T": T, "nseq": nseq, "Hq": H, "Hkv": H, "d": d, "causal": True,
           "parallelism": f"dp{world}" if world > 1 else "single", "l2": "flushed before every step"}
    line = {"metric": METRIC + " (varlen)", "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_s, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": 5 * args.steps,
            "forward_ms": ms_f}
    print(json.dumps(line), flush=True)
    return 0



def main():
    args = parse()
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload == "varlen":
        return run_varlen(args)
    if args.workload == "blocksparse":
        return run_blocksparse(args)
    if args.workload == "fp8":
        return run_fp8(args)
    if args.workload == "ring":
        return run_ring(args)
    if args.workload == "decode":
        return run_decode_reference(args) if args.impl == "reference" else run_decode(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
