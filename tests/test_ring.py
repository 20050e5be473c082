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

        k_keep, v_keep = k_r.clone(), v_r.clone()
        O, L = ring_forward(q_r, ring_exchange(k_r, v_r), rank, world, causal, block, merge)
        O_ref, L_ref = oracle.attn_fwd(q, k, v, causal, scale)
        e_o = float(np.max(np.abs(O - O_ref[:, sl])))
        e_l = float(np.max(np.abs(L - L_ref[:, :, sl])))
        intact = torch.equal(k_r, k_keep) and torch.equal(v_r, v_keep)  # sent, never received into
        if e_o > 1e-12 or e_l > 1e-12 or not intact:
            errs.put(f"rank {rank}: |dO| {e_o:.3g} |dLSE| {e_l:.3g}, inputs intact: {intact}")
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
        k_keep, v_keep = k_r.clone(), v_r.clone()
        dk, dv = ring_backward(k_r, v_r, rank, world, causal, block_grad, lambda x: torch.zeros_like(x), add,
                               _p2p_exchange())
        if not (torch.equal(k_r, k_keep) and torch.equal(v_r, v_keep)):
            raise RuntimeError("the ring overwrote the caller's K/V shard")
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


# ---------------------------------------------------------------- zig-zag layout

from io_aware_exact_27_b200.ring import (chunk_mode, zigzag_backward, zigzag_chunks, zigzag_forward,  # noqa: E402
                                         zigzag_schedule, zigzag_shard, zigzag_unshard)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 6])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_schedule_is_balanced_and_covers_each_pair_once(world, causal):
    seen = {}
    for r in range(world):
        sched = zigzag_schedule(r, world, causal)
        assert [t for t, _, _ in sched] == list(range(world))
        assert sorted(src for _, src, _ in sched) == list(range(world))
        mine = zigzag_chunks(r, world)
        work = 0.0
        for _, src, pairs in sched:
            theirs = zigzag_chunks(src, world)
            for i, j, mode in pairs:
                key = (mine[i], theirs[j])
                assert key not in seen
                seen[key] = mode
                assert mode == chunk_mode(mine[i], theirs[j], causal) != "skip"
                work += 1.0 if mode == "full" else 0.5
        # every rank: 2R full c x c blocks with the causal mask, 4R without
        assert work == (2 * world if causal else 4 * world)
    n = 2 * world
    want = {(a, b) for a in range(n) for b in range(n) if not causal or b <= a}
    assert set(seen) == want


@pytest.mark.parametrize("world", [1, 2, 3])
def test_zigzag_shard_round_trip(world):
    x = torch.arange(2 * 12 * world * 3 * 2, dtype=torch.float32).reshape(2, 12 * world, 3, 2)
    shards = [zigzag_shard(x, r, world) for r in range(world)]
    assert all(s.shape == (2, 2, 6, 3, 2) for s in shards)
    assert torch.equal(zigzag_unshard(shards), x)
    with pytest.raises(ValueError):
        zigzag_shard(x[:, :-1], 0, world)


def _zigzag_chunks_np(x, rank, world, axis):
    n = x.shape[axis] // (2 * world)
    a, b = zigzag_chunks(rank, world)
    take = lambda i: np.take(x, np.arange(i * n, (i + 1) * n), axis=axis)  # noqa: E731
    return take(a), take(b)


def _zz_rank_main(rank, world, port, causal, B, N, Hq, Hkv, d, errs):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)
        q, k, v, do = (rng.standard_normal((B, N, H, d)) for H in (Hq, Hkv, Hkv, Hq))
        scale = 1.0 / math.sqrt(d)
        O, L = oracle.attn_fwd(q, k, v, causal, scale)
        qc = _zigzag_chunks_np(q, rank, world, 1)
        kz = torch.from_numpy(np.stack(_zigzag_chunks_np(k, rank, world, 1)))
        vz = torch.from_numpy(np.stack(_zigzag_chunks_np(v, rank, world, 1)))
        parts = [([], []), ([], [])]

        def block(i, qq, kk, vv, c):
            return oracle.attn_fwd(qq, kk.numpy(), vv.numpy(), c, scale)

        def merge(i, o_t, lse_t, first, last):
            parts[i][0].append(o_t)
            parts[i][1].append(np.transpose(lse_t, (0, 2, 1)))
            if not last:
                return None
            o, l = oracle.merge_partials(*parts[i])
            return o, np.transpose(l, (0, 2, 1))

        res = zigzag_forward(qc, ring_exchange(kz, vz), rank, world, causal, block, merge)
        e = 0.0
        for i, (o_ref, l_ref) in enumerate(zip(_zigzag_chunks_np(O, rank, world, 1),
                                              _zigzag_chunks_np(L, rank, world, 2))):
            e = max(e, float(np.abs(res[i][0] - o_ref).max()), float(np.abs(res[i][1] - l_ref).max()))
        e_fwd = e
        # backward: the same ring with the oracle's block gradients
        from io_aware_exact_27_b200.ring import _p2p_exchange
        doc = _zigzag_chunks_np(do, rank, world, 1)
        oc, lc = _zigzag_chunks_np(O, rank, world, 1), _zigzag_chunks_np(L, rank, world, 2)
        dq = [np.zeros_like(x) for x in qc]

        def block_grad(i, kk, vv, c):
            a, bb, cc = oracle.attn_bwd_block(qc[i], kk.numpy(), vv.numpy(), doc[i], oc[i], lc[i], c, scale)
            dq[i] += a
            return torch.from_numpy(bb), torch.from_numpy(cc)

        def add(acc, part, first):
            if first:
                acc.copy_(part)
            else:
                acc.add_(part)

        dk, dv = zigzag_backward(kz, vz, rank, world, causal, block_grad, lambda x: torch.zeros_like(x), add,
                                 _p2p_exchange())
        dq_ref, dk_ref, dv_ref = oracle.attn_bwd(q, k, v, do, causal, scale)
        for i in range(2):
            e = max(e, float(np.abs(dq[i] - _zigzag_chunks_np(dq_ref, rank, world, 1)[i]).max()),
                    float(np.abs(dk[i].numpy() - _zigzag_chunks_np(dk_ref, rank, world, 1)[i]).max()),
                    float(np.abs(dv[i].numpy() - _zigzag_chunks_np(dv_ref, rank, world, 1)[i]).max()))
        # the ring sends the caller's K/V shards but never receives into them
        intact = np.array_equal(kz.numpy(), np.stack(_zigzag_chunks_np(k, rank, world, 1))) and \
            np.array_equal(vz.numpy(), np.stack(_zigzag_chunks_np(v, rank, world, 1)))
        errs.put(None if e <= 1e-12 and intact else
                 f"rank {rank}: max error {e:.3g} (forward {e_fwd:.3g}), inputs intact: {intact}")
    except Exception as ex:  # reported to the parent
        errs.put(f"rank {rank}: {type(ex).__name__}: {ex}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (2, False), (3, True)])
def test_zigzag_ring_fwd_bwd_on_cpu_ranks(world, causal):
    ctx = mp.get_context("spawn")
    errs = ctx.Queue()
    port = _free_port()
    B, N, Hq, Hkv, d = 2, 12 * world, 4, 2, 8
    procs = [ctx.Process(target=_zz_rank_main, args=(r, world, port, causal, B, N, Hq, Hkv, d, errs))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [errs.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(r is None for r in results), results


def _sub_rank_main(rank, world, port, errs):
    """Ranks 1 and 2 of 3 run the ring on a sub-group (group-local ranks 0 and
    1); rank 0 only takes part in creating the group."""
    from io_aware_exact_27_b200.ring import _p2p_exchange, ring_backward
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sub = dist.new_group([1, 2])
        if rank == 0:
            errs.put(None)
            return
        r, R = dist.get_rank(sub), dist.get_world_size(sub)
        B, N, H, d, causal = 1, 16, 2, 8, True
        rng = np.random.default_rng(9)
        q, k, v, do = (rng.standard_normal((B, N, H, d)) for _ in range(4))
        scale = 1.0 / math.sqrt(d)
        n = N // R
        sl = slice(r * n, (r + 1) * n)
        k_r, v_r = torch.from_numpy(np.ascontiguousarray(k[:, sl])), torch.from_numpy(np.ascontiguousarray(v[:, sl]))
        parts_o, parts_l = [], []

        def block(qq, kk, vv, c):
            return oracle.attn_fwd(qq, kk.numpy(), vv.numpy(), c, scale)

        def merge(o_t, lse_t, first, last):
            parts_o.append(o_t)
            parts_l.append(np.transpose(lse_t, (0, 2, 1)))
            if not last:
                return None
            o, l = oracle.merge_partials(parts_o, parts_l)
            return o, np.transpose(l, (0, 2, 1))

        O, L = ring_forward(q[:, sl], ring_exchange(k_r, v_r, group=sub), r, R, causal, block, merge)
        O_ref, L_ref = oracle.attn_fwd(q, k, v, causal, scale)
        e = max(float(np.abs(O - O_ref[:, sl]).max()), float(np.abs(L - L_ref[:, :, sl]).max()))
        dq = np.zeros_like(q[:, sl])

        def block_grad(kk, vv, c):
            a, bb, cc = oracle.attn_bwd_block(q[:, sl], kk.numpy(), vv.numpy(), do[:, sl], O_ref[:, sl],
                                              L_ref[:, :, sl], c, scale)
            dq[...] += a
            return torch.from_numpy(bb), torch.from_numpy(cc)

        def add(acc, part, first):
            if first:
                acc.copy_(part)
            else:
                acc.add_(part)

        dk, dv = ring_backward(k_r, v_r, r, R, causal, block_grad, lambda x: torch.zeros_like(x), add,
                               _p2p_exchange(sub))
        g = oracle.attn_bwd(q, k, v, do, causal, scale)
        e = max(e, float(np.abs(dq - g[0][:, sl]).max()), float(np.abs(dk.numpy() - g[1][:, sl]).max()),
                float(np.abs(dv.numpy() - g[2][:, sl]).max()))
        errs.put(None if e <= 1e-12 else f"rank {rank} (group rank {r}): max error {e:.3g}")
    except Exception as ex:  # reported to the parent
        errs.put(f"rank {rank}: {type(ex).__name__}: {ex}")
    finally:
        dist.destroy_process_group()


def test_ring_on_a_sub_group():
    ctx = mp.get_context("spawn")
    errs = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sub_rank_main, args=(r, 3, port, errs)) for r in range(3)]
    for p in procs:
        p.start()
    results = [errs.get(timeout=120) for _ in range(3)]
    for p in procs:
        p.join(timeout=60)
    assert all(r is None for r in results), results
