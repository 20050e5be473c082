"""Host logic of context-parallel ring attention, on CPU ranks (gloo).

The ring's schedule and its K/V exchange (`ring_exchange`, the same
point-to-point code that runs over NCCL on GPUs) are checked with the fp64
oracle standing in for the per-block kernel and the oracle's LSE merge of key
partitions standing in for the merge kernel: every rank must end with exact
attention of its query rows over the whole sequence.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from io_aware_exact_27_b200.ring import ring_block_mode, ring_exchange, ring_forward, ring_schedule


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_covers_each_pair_once(world, causal):
    for r in range(world):
        sched = ring_schedule(r, world, causal)
        assert [t for t, _, _ in sched] == list(range(world))
        assert sorted(src for _, src, _ in sched) == list(range(world))  # every shard once
        assert sched[0] == (0, r, "causal" if causal else "full")  # own shard first
        for _, src, mode in sched:
            want = "full" if (not causal or src < r) else ("causal" if src == r else "skip")
            assert mode == want == ring_block_mode(r, src, causal)
        # causal: rank r computes exactly the r + 1 shards at or before its own
        if causal:
            assert sum(m != "skip" for _, _, m in sched) == r + 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, causal, B, N, Hq, Hkv, d, errs):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = synth.qkv_bf16(3, B, N, Hq, Hkv, d)
        n = N // world
        sl = slice(rank * n, (rank + 1) * n)
        q_r, k_r, v_r = (t[:, sl].float().contiguous() for t in (q, k, v))
        scale = 1.0 / math.sqrt(d)
        parts_o, parts_l = [], []

        def block(qq, kk, vv, c):
            return oracle.attn_fwd(qq, kk, vv, c, scale)

        def merge(o_t, lse_t, first, last):
            parts_o.append(o_t)
            parts_l.append(np.transpose(lse_t, (0, 2, 1)))  # [B,H,n] -> [B,n,H], the layout of O's rows
            if not last:
                return None
            o, l = oracle.merge_partials(parts_o, parts_l)
            return o, np.transpose(l, (0, 2, 1))

        O, L = ring_forward(q_r, ring_exchange(k_r, v_r), rank, world, causal, block, merge)
        O_ref, L_ref = oracle.attn_fwd(q, k, v, causal, scale)
        e_o = float(np.max(np.abs(O - O_ref[:, sl])))
        e_l = float(np.max(np.abs(L - L_ref[:, :, sl])))
        if e_o > 1e-12 or e_l > 1e-12:
            errs.put(f"rank {rank}: |dO| {e_o:.3g} |dLSE| {e_l:.3g}")
        else:
            errs.put(None)
    except Exception as e:  # reported to the parent
        errs.put(f"rank {rank}: {type(e).__name__}: {e}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (2, False), (3, True)])
def test_ring_on_cpu_ranks(world, causal):
    ctx = mp.get_context("spawn")
    errs = ctx.Queue()
    port = _free_port()
    B, N, Hq, Hkv, d = 2, 24 * world, 4, 2, 8
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, B, N, Hq, Hkv, d, errs))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [errs.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(r is None for r in results), results


def _rank_bwd_main(rank, world, port, causal, B, N, Hq, Hkv, d, errs):
    from io_aware_exact_27_b200.ring import _p2p_exchange, ring_backward
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(4)
        q, k, v, do = (rng.standard_normal((B, N, H, d)) for H in (Hq, Hkv, Hkv, Hq))
        scale = 1.0 / math.sqrt(d)
        O, L = oracle.attn_fwd(q, k, v, causal, scale)
        n = N // world
        sl = slice(rank * n, (rank + 1) * n)
        q_r, do_r, o_r, l_r = q[:, sl], do[:, sl], O[:, sl], L[:, :, sl]
        dq = np.zeros_like(q_r)

        def block_grad(kk, vv, c):
            a, bb, cc = oracle.attn_bwd_block(q_r, kk.numpy(), vv.numpy(), do_r, o_r, l_r, c, scale)
            dq[...] += a
            return torch.from_numpy(bb), torch.from_numpy(cc)

        def add(acc, part, first):
            if first:
                acc.copy_(part)
            else:
                acc.add_(part)

        k_r = torch.from_numpy(np.ascontiguousarray(k[:, sl]))
        v_r = torch.from_numpy(np.ascontiguousarray(v[:, sl]))
        dk, dv = ring_backward(k_r, v_r, rank, world, causal, block_grad, lambda x: torch.zeros_like(x), add,
                               _p2p_exchange())
        dq_ref, dk_ref, dv_ref = oracle.attn_bwd(q, k, v, do, causal, scale)
        e = max(float(np.abs(dq - dq_ref[:, sl]).max()), float(np.abs(dk.numpy() - dk_ref[:, sl]).max()),
                float(np.abs(dv.numpy() - dv_ref[:, sl]).max()))
        errs.put(None if e <= 1e-12 else f"rank {rank}: max |d grad| {e:.3g}")
    except Exception as e:  # reported to the parent
        errs.put(f"rank {rank}: {type(e).__name__}: {e}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (2, False), (3, True)])
def test_ring_backward_on_cpu_ranks(world, causal):
    ctx = mp.get_context("spawn")
    errs = ctx.Queue()
    port = _free_port()
    B, N, Hq, Hkv, d = 2, 16 * world, 4, 2, 8
    procs = [ctx.Process(target=_rank_bwd_main, args=(r, world, port, causal, B, N, Hq, Hkv, d, errs))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [errs.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(r is None for r in results), results
