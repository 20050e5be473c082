"""Context-parallel ring attention (forward and backward) over torch.distributed ranks.

The topic page "Flash Attention and Efficient Transformer Mechanisms" (opening
paragraph) says the method extends to multi-GPU settings for very long
sequences; the Dao-AILab repository overview (training sub-package) names
sequence parallelism. Neither gives an algorithm; this module takes the plain
one (a reading): every rank holds one contiguous shard of the sequence, the
key/value shards travel once around the ring, and each rank folds the exact
attention of its query rows over every shard it sees into a running result
through the log-sum-exp merge of disjoint key sets.

Rank r of R holds tokens [r*n, (r+1)*n) of every sequence (n = N/R) of Q, K
and V, laid out [B, n, H, d]. At hop t it holds the K/V shard of rank
src = (r - t) mod R and computes, with the single-GPU forward kernel:
  * src < r, or no causal mask: every key precedes every query: full block;
  * src == r: the shard's own keys: causal within the block;
  * src > r with the causal mask: every key follows every query: skipped.
While a block is computed the shard moves one hop on (NCCL send to r+1,
receive from r-1 into a second buffer). Each block's bf16 (O_t, LSE_t) goes
to its own slot; after the last block `fa_attn_merge` combines the slots in
fp32 (one pass over them).

The backward walks the same ring: each block runs the single-GPU backward
kernels with the full rows' O and LSE, dQ is summed on the rank, and the fp32
dK/dV accumulators of a shard travel with it and come home after the last hop
(see the backward section below).

Only the exchange of K/V shards (and, in the backward, their gradient
accumulators) crosses GPUs; the arithmetic of every step runs in the
library's kernels. The contiguous sharding gives causal ranks unequal work
(rank r computes r + 1 blocks); the zig-zag layout at the end of this module
(rank r holds sequence chunks r and 2R-1-r) gives every rank the same work.
The exchange only ever sends the caller's K/V tensors: shards are received
into two spare buffers used in turn.
"""

from __future__ import annotations

import math


def ring_block_mode(rank: int, src: int, causal: bool) -> str:
    """How rank `rank`'s query shard attends the key shard of rank `src`."""
    if not causal or src < rank:
        return "full"
    if src == rank:
        return "causal"
    return "skip"


def ring_schedule(rank: int, world: int, causal: bool):
    """[(hop, source rank of the K/V shard held at that hop, mode)] for one rank."""
    return [(t, (rank - t) % world, ring_block_mode(rank, (rank - t) % world, causal)) for t in range(world)]


def ring_forward(q, kv_blocks, rank: int, world: int, causal: bool, block_attention, merge):
    """Transport-agnostic core of the ring.

    kv_blocks yields (src, k, v) in hop order; block_attention(q, k, v,
    causal) returns (O_t, LSE_t) of one block; merge(o_t, lse_t, first, last)
    folds it into the running result and returns that result after the last
    block. Blocks in "skip" mode are not computed; the caller's merge sees
    first=True on the first computed block and last=True on the last one.
    """
    sched = ring_schedule(rank, world, causal)
    todo = [t for t, _, mode in sched if mode != "skip"]
    last_t = todo[-1]
    out = None
    first = True
    for t, (src, k, v) in enumerate(kv_blocks):
        if src != sched[t][1]:
            raise RuntimeError(f"ring order broken: hop {t} holds shard {src}, expected {sched[t][1]}")
        mode = sched[t][2]
        if mode != "skip":
            o_t, lse_t = block_attention(q, k, v, mode == "causal")
            out = merge(o_t, lse_t, first, t == last_t)
            first = False
    return out


def ring_exchange(k, v, group=None):
    """Yields (src, k, v) for hops 0..R-1 of the ring; the next shard's
    transfer (send to rank+1, receive from rank-1, both K and V) runs while
    the caller works on the current one. Works with any torch.distributed
    backend that has point-to-point ops (NCCL on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % R) if group is not None else (r + 1) % R
    prv = dist.get_global_rank(group, (r - 1) % R) if group is not None else (r - 1) % R
    # receive buffers: two, used in turn, so that the caller's k and v are
    # only ever sent, never overwritten
    cur = (k, v)
    spares = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, R - 1))]
    for t in range(R):
        reqs = []
        if t + 1 < R:
            into = spares[t % len(spares)]
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group), dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, into[0], prv, group), dist.P2POp(dist.irecv, into[1], prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        yield (r - t) % R, cur[0], cur[1]
        for req in reqs:
            req.wait()
        if t + 1 < R:
            cur = into


class _GpuRank:
    """The GPU side of one rank's ring: each computed block writes its bf16
    (O_t, LSE_t) into its own slot, and after the last block one merge kernel
    combines the slots (a rank with a single block returns it as is)."""

    def __init__(self, q_shape, nblocks, scale, device):
        import torch
        B, n, H, d = q_shape
        self.shape = (B, n, H, d)
        self.scale = scale
        self.nblocks = nblocks
        self.o_parts = torch.empty((nblocks, B, n, H, d), dtype=torch.bfloat16, device=device)
        self.lse_parts = torch.empty((nblocks, B, H, n), dtype=torch.float32, device=device)
        self.i = 0

    def block(self, q, k, v, causal):
        from . import attention_fwd
        i = self.i
        self.i += 1
        return attention_fwd(q, k, v, causal=causal, scale=self.scale, out=self.o_parts[i], lse=self.lse_parts[i])

    def merge(self, o_t, lse_t, first, last):
        import torch
        from . import fa_attn_merge
        if not last:
            return None
        if self.nblocks == 1:
            return self.o_parts[0], self.lse_parts[0]
        B, n, H, d = self.shape
        o = torch.empty((B, n, H, d), dtype=torch.bfloat16, device=self.o_parts.device)
        lse = torch.empty((B, H, n), dtype=torch.float32, device=self.o_parts.device)
        fa_attn_merge(self.o_parts, self.lse_parts, self.nblocks, o, lse, B, n, H, d)
        return o, lse


def _gpu_rank(q, rank, world, causal, scale):
    nblocks = sum(mode != "skip" for _, _, mode in ring_schedule(rank, world, causal))
    return _GpuRank(tuple(q.shape), nblocks, scale, q.device)


def ring_attention_fwd(q, k, v, causal=True, scale=None, group=None):
    """Sequence-parallel exact attention over the ranks of `group`.

    q [B, n, Hq, d], k, v [B, n, Hkv, d] bf16 on this rank's GPU: this rank's
    shard (tokens rank*n .. rank*n + n - 1) of sequences of length n*R.
    Returns (o [B, n, Hq, d] bf16, lse [B, Hq, n] fp32) for this rank's query
    rows, over all keys of the sequence."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    d = q.shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    g = _gpu_rank(q, r, R, causal, scale)
    return ring_forward(q, ring_exchange(k, v, group), r, R, causal, g.block, g.merge)


def ring_attention_fwd_local(q_shards, k_shards, v_shards, causal=True, scale=None):
    """The ring of R ranks run by one process on one GPU: shard r of each
    list plays rank r, and hop t of rank r reads shard (r - t) mod R straight
    from the lists instead of receiving it. Same blocks, kernels and merge
    order as `ring_attention_fwd`; for checking and timing the per-rank work
    where only one GPU is at hand. Returns per-rank (o, lse)."""
    R = len(q_shards)
    d = q_shards[0].shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    outs = []
    for r in range(R):
        blocks = (((r - t) % R, k_shards[(r - t) % R], v_shards[(r - t) % R]) for t in range(R))
        g = _gpu_rank(q_shards[r], r, R, causal, scale)
        outs.append(ring_forward(q_shards[r], blocks, r, R, causal, g.block, g.merge))
    return outs


# ---------------------------------------------------------------- backward
#
# With the forward's O and LSE of this rank's query rows (over all keys), the
# gradient splits over key shards exactly: for the block (my queries, shard
# src), P = exp(S - LSE), D = rowsum(dO * O), and the block adds
# dQ += scale dS K_src, dK_src += scale dS^T Q, dV_src += P^T dO with
# dS = P * (dO V_src^T - D) -- what the single-GPU backward kernels compute
# when given the full rows' O and LSE. dQ stays on the rank; the fp32 dK/dV
# accumulators of a shard travel with it and come home after the last hop.


def _p2p_exchange(group=None):
    """send(list) to rank+1 and receive into recv(list) from rank-1, as one
    batch of point-to-point ops; returns a handle whose wait() completes it."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % R) if group is not None else (r + 1) % R
    prv = dist.get_global_rank(group, (r - 1) % R) if group is not None else (r - 1) % R

    class _Handle:
        def __init__(self, reqs):
            self.reqs = reqs

        def wait(self):
            for req in self.reqs:
                req.wait()

    def exchange(send, recv):
        ops = [dist.P2POp(dist.isend, t, nxt, group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
        return _Handle(dist.batch_isend_irecv(ops))

    return exchange


def ring_backward(k, v, rank: int, world: int, causal: bool, block_grad, new_acc, add, exchange):
    """Transport-agnostic ring backward for one rank.

    block_grad(k, v, causal) -> (dk_t, dv_t): this rank's queries against one
    key shard (it folds its own dq contribution in); new_acc(x) -> an
    accumulator shaped like x; add(acc, part, first) sets or adds in place;
    exchange(send, recv) -> handle (send to rank+1, receive from rank-1).
    Returns (dk_acc, dv_acc) of this rank's own key shard."""
    sched = ring_schedule(rank, world, causal)
    cur = [k, v]
    acc = [new_acc(k), new_acc(v)]
    # K/V receive buffers used in turn (the caller's k, v are never overwritten)
    spares = [[x.new_empty(x.shape) for x in cur] for _ in range(min(2, world - 1))]
    if world > 1:
        acc_spare = [new_acc(k), new_acc(v)]
    for t, src, mode in sched:
        spare = spares[t % len(spares)] if t + 1 < world else None
        kv_move = exchange(cur, spare) if t + 1 < world else None  # overlaps the block
        if mode != "skip":
            dk_t, dv_t = block_grad(cur[0], cur[1], mode == "causal")
            add(acc[0], dk_t, t == 0)  # hop 0 is the own shard: always computed
            add(acc[1], dv_t, t == 0)
        if world > 1:  # the accumulators follow their shard (home after the last hop)
            exchange(acc, acc_spare).wait()
            acc, acc_spare = acc_spare, acc
        if kv_move is not None:
            kv_move.wait()
            cur = spare
    return acc[0], acc[1]


class _GpuRankBwd:
    """The query side of one rank's backward on the GPU: the D / base-2 LSE
    workspace prepared once, one fa_bwd_part call per key block, dQ summed in
    fp32 by fa_grad_accumulate."""

    def __init__(self, q, o, lse, do, Hkv, scale):
        import torch
        from . import fa_bwd_workspace_size
        B, n, Hq, d = q.shape
        self.q, self.o, self.lse, self.do = q, o, lse, do
        self.dims = (B, Hq, Hkv, n, d)
        self.scale = scale
        self.ws_bytes = fa_bwd_workspace_size(B * n, B, Hq, d)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=q.device)
        self.dq_t = torch.empty_like(q)
        self.dk_t = torch.empty((B, n, Hkv, d), dtype=q.dtype, device=q.device)
        self.dv_t = torch.empty_like(self.dk_t)
        self.dq_acc = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        self.prepared = False
        self.first = True

    def block(self, k, v, causal):
        from . import FA_BWD_DKDV, FA_BWD_DQ, FA_BWD_PREPARE, fa_bwd_part, fa_grad_accumulate
        B, Hq, Hkv, n, d = self.dims
        parts = FA_BWD_DKDV | FA_BWD_DQ | (0 if self.prepared else FA_BWD_PREPARE)
        fa_bwd_part(parts, self.q, k, v, self.o, self.lse, self.do, self.dq_t, self.dk_t, self.dv_t, self.ws,
                    self.ws_bytes, B, Hq, Hkv, n, d, causal, self.scale)
        self.prepared = True
        fa_grad_accumulate(self.dq_acc, self.dq_t, None, self.dq_t.numel(), self.first)
        self.first = False
        return self.dk_t, self.dv_t

    def dq(self):
        import torch
        from . import fa_grad_accumulate
        out = torch.empty_like(self.q)
        fa_grad_accumulate(self.dq_acc, None, out, out.numel(), 0)
        return out


def _gpu_acc_ops():
    import torch
    from . import fa_grad_accumulate

    def new_acc(x):
        return torch.empty(x.shape, dtype=torch.float32, device=x.device)

    def add(acc, part, first):
        fa_grad_accumulate(acc, part, None, part.numel(), first)

    def to_bf16(acc):
        out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
        fa_grad_accumulate(acc, None, out, acc.numel(), 0)
        return out

    return new_acc, add, to_bf16


def ring_attention_bwd(q, k, v, o, lse, do, causal=True, scale=None, group=None):
    """Gradients of ring attention over the ranks of `group`: this rank's
    shards q, do, o [B,n,Hq,d], lse [B,Hq,n] (from ring_attention_fwd) and
    k, v [B,n,Hkv,d] -> (dq, dk, dv) bf16 for this rank's shards."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    d = q.shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    g = _GpuRankBwd(q, o, lse, do, k.shape[2], scale)
    new_acc, add, to_bf16 = _gpu_acc_ops()
    dk, dv = ring_backward(k, v, r, R, causal, g.block, new_acc, add, _p2p_exchange(group))
    return g.dq(), to_bf16(dk), to_bf16(dv)


def ring_attention_bwd_local(q_shards, k_shards, v_shards, o_shards, lse_shards, do_shards, causal=True,
                             scale=None):
    """The ring backward of R ranks run by one process on one GPU, hop by hop
    (at hop t every rank r works on shard (r - t) mod R, whose accumulators
    receive their partials in the same hop order as on the ring). For
    checking where only one GPU is at hand. Returns per-rank (dq, dk, dv)."""
    R = len(q_shards)
    d = q_shards[0].shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    new_acc, add, to_bf16 = _gpu_acc_ops()
    gs = [_GpuRankBwd(q_shards[r], o_shards[r], lse_shards[r], do_shards[r], k_shards[r].shape[2], scale)
          for r in range(R)]
    acc_k = [new_acc(x) for x in k_shards]
    acc_v = [new_acc(x) for x in v_shards]
    for t in range(R):
        for r in range(R):
            src = (r - t) % R
            mode = ring_block_mode(r, src, causal)
            if mode == "skip":
                continue
            dk_t, dv_t = gs[r].block(k_shards[src], v_shards[src], mode == "causal")
            add(acc_k[src], dk_t, t == 0)
            add(acc_v[src], dv_t, t == 0)
    return [(gs[r].dq(), to_bf16(acc_k[r]), to_bf16(acc_v[r])) for r in range(R)]


# ---------------------------------------------------------------- zig-zag layout
#
# With the causal mask the contiguous shards give rank r r + 1 blocks of work
# (rank R-1 does R times what rank 0 does). The zig-zag layout cuts the
# sequence into 2R chunks of c = N / (2R) tokens and gives rank r chunks r and
# 2R-1-r: every rank then holds one early and one late chunk, and for the
# causal mask every hop after the first is exactly two full c x c blocks on
# every rank (hop 0: two causal diagonal blocks and one full block), 2R
# full-block equivalents per rank. Shards are chunk-major, [2, B, c, H, d]
# (chunk 0 = the early one), so that each chunk is a contiguous [B, c, H, d]
# input of the single-GPU kernels, which take equal query and key lengths:
# every block of the ring is one c x c call.


def zigzag_chunks(rank: int, world: int):
    """Global indices (of the 2R chunks of the sequence) of the two chunks rank holds."""
    return rank, 2 * world - 1 - rank


def chunk_mode(q_chunk: int, k_chunk: int, causal: bool) -> str:
    """How query chunk q_chunk attends key chunk k_chunk (global chunk indices)."""
    if not causal or k_chunk < q_chunk:
        return "full"
    if k_chunk == q_chunk:
        return "causal"
    return "skip"


def zigzag_schedule(rank: int, world: int, causal: bool):
    """[(hop, source rank of the K/V shard, [(i, j, mode), ...])] for one rank:
    local query chunk i (0 early, 1 late) against chunk j of the held shard,
    skipped pairs left out, in the order they are computed."""
    mine = zigzag_chunks(rank, world)
    out = []
    for t in range(world):
        src = (rank - t) % world
        theirs = zigzag_chunks(src, world)
        pairs = [(i, j, chunk_mode(mine[i], theirs[j], causal)) for i in range(2) for j in range(2)]
        out.append((t, src, [p for p in pairs if p[2] != "skip"]))
    return out


def zigzag_shard(x, rank: int, world: int):
    """[B, N, H, d] -> this rank's chunk-major zig-zag shard [2, B, N/(2R), H, d]."""
    import torch
    B, N, H, d = x.shape
    if N % (2 * world):
        raise ValueError(f"N = {N} is not a multiple of 2 x {world} ranks")
    c = N // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.stack([x[:, a * c:(a + 1) * c], x[:, b * c:(b + 1) * c]]).contiguous()


def zigzag_unshard(shards):
    """Per-rank chunk-major shards [2, B, c, H, d] -> the whole sequence [B, 2Rc, H, d]."""
    import torch
    R = len(shards)
    chunks = [None] * (2 * R)
    for r, s in enumerate(shards):
        a, b = zigzag_chunks(r, R)
        chunks[a], chunks[b] = s[0], s[1]
    return torch.cat(chunks, dim=1)


def zigzag_unshard_lse(shards):
    """Per-rank [2, B, H, c] LSE shards -> [B, H, 2Rc]."""
    import torch
    R = len(shards)
    chunks = [None] * (2 * R)
    for r, s in enumerate(shards):
        a, b = zigzag_chunks(r, R)
        chunks[a], chunks[b] = s[0], s[1]
    return torch.cat(chunks, dim=-1)


def zigzag_forward(q_chunks, kv_blocks, rank: int, world: int, causal: bool, block_attention, merge):
    """Transport-agnostic core of the zig-zag ring.

    q_chunks = (early, late) query chunks of this rank; kv_blocks yields
    (src, k, v) in hop order with k, v indexable by chunk (0, 1);
    block_attention(i, q, k, v, causal) -> (O, LSE) of one c x c block of
    query chunk i;
    merge(i, o, lse, first, last) folds a block into query chunk i's result
    and returns that result after the chunk's last block. Returns
    [result of chunk 0, result of chunk 1]."""
    sched = zigzag_schedule(rank, world, causal)
    last = {}
    for t, _, pairs in sched:
        for p, (i, _, _) in enumerate(pairs):
            last[i] = (t, p)
    seen, out = set(), [None, None]
    for t, (src, k, v) in enumerate(kv_blocks):
        if src != sched[t][1]:
            raise RuntimeError(f"ring order broken: hop {t} holds shard {src}, expected {sched[t][1]}")
        for p, (i, j, mode) in enumerate(sched[t][2]):
            o_t, lse_t = block_attention(i, q_chunks[i], k[j], v[j], mode == "causal")
            res = merge(i, o_t, lse_t, i not in seen, last[i] == (t, p))
            seen.add(i)
            if res is not None:
                out[i] = res
    return out


def zigzag_backward(k, v, rank: int, world: int, causal: bool, block_grad, new_acc, add, exchange):
    """Transport-agnostic zig-zag ring backward for one rank.

    k, v: this rank's chunk-major shards; block_grad(i, kk, vv, causal) ->
    (dk_t, dv_t) of query chunk i against one key chunk (it folds its own dq
    contribution in); new_acc(x) -> an accumulator shaped like x (chunk-major,
    it travels with its shard); add(acc, part, first) sets or adds in place;
    exchange(send, recv) -> handle. Returns (dk_acc, dv_acc) of this rank's
    own shard."""
    sched = zigzag_schedule(rank, world, causal)
    cur = [k, v]
    acc = [new_acc(k), new_acc(v)]
    # K/V receive buffers used in turn (the caller's k, v are never overwritten)
    spares = [[x.new_empty(x.shape) for x in cur] for _ in range(min(2, world - 1))]
    if world > 1:
        acc_spare = [new_acc(k), new_acc(v)]
    for t, src, pairs in sched:
        spare = spares[t % len(spares)] if t + 1 < world else None
        kv_move = exchange(cur, spare) if t + 1 < world else None  # overlaps the blocks
        started = set()
        for i, j, mode in pairs:
            dk_t, dv_t = block_grad(i, cur[0][j], cur[1][j], mode == "causal")
            first = t == 0 and j not in started  # hop 0 is the own shard: both chunks get a block
            add(acc[0][j], dk_t, first)
            add(acc[1][j], dv_t, first)
            started.add(j)
        if world > 1:  # the accumulators follow their shard (home after the last hop)
            exchange(acc, acc_spare).wait()
            acc, acc_spare = acc_spare, acc
        if kv_move is not None:
            kv_move.wait()
            cur = spare
    return acc[0], acc[1]


class _GpuZigzag:
    """The GPU side of one rank's zig-zag ring forward: each block of query
    chunk i writes its bf16 (O, LSE) into the next of chunk i's slots, and
    after the chunk's last block one merge kernel combines its slots."""

    def __init__(self, q, rank, world, causal, scale):
        import torch
        _, B, c, H, d = q.shape
        self.dims = (B, c, H, d)
        self.scale = scale
        counts = [0, 0]
        for _, _, pairs in zigzag_schedule(rank, world, causal):
            for i, _, _ in pairs:
                counts[i] += 1
        self.counts = counts
        self.o_parts = [torch.empty((n, B, c, H, d), dtype=torch.bfloat16, device=q.device) for n in counts]
        self.lse_parts = [torch.empty((n, B, H, c), dtype=torch.float32, device=q.device) for n in counts]
        self.o = torch.empty((2, B, c, H, d), dtype=torch.bfloat16, device=q.device)
        self.lse = torch.empty((2, B, H, c), dtype=torch.float32, device=q.device)
        self.used = [0, 0]

    def block(self, i, q, k, v, causal):
        from . import attention_fwd
        n = self.used[i]
        self.used[i] += 1
        return attention_fwd(q, k, v, causal=causal, scale=self.scale, out=self.o_parts[i][n],
                             lse=self.lse_parts[i][n])

    def merge(self, i, o_t, lse_t, first, last):
        from . import fa_attn_merge
        if not last:
            return None
        B, c, H, d = self.dims
        if self.counts[i] == 1:
            self.o[i].copy_(self.o_parts[i][0])
            self.lse[i].copy_(self.lse_parts[i][0])
        else:
            fa_attn_merge(self.o_parts[i], self.lse_parts[i], self.counts[i], self.o[i], self.lse[i], B, c, H, d)
        return True


def _zigzag_fwd_rank(q, kv_blocks, rank, world, causal, scale):
    g = _GpuZigzag(q, rank, world, causal, scale)
    zigzag_forward((q[0], q[1]), kv_blocks, rank, world, causal, g.block, g.merge)
    return g.o, g.lse


def ring_attention_fwd_zigzag(q, k, v, causal=True, scale=None, group=None):
    """Zig-zag sequence-parallel exact attention over the ranks of `group`.

    q [2, B, c, Hq, d], k, v [2, B, c, Hkv, d] bf16 on this rank's GPU: this
    rank's chunks (zigzag_shard) of sequences of length 2Rc. Returns
    (o [2, B, c, Hq, d] bf16, lse [2, B, Hq, c] fp32) for this rank's query
    rows over all keys of the sequence."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    return _zigzag_fwd_rank(q, ring_exchange(k, v, group), r, R, causal, scale)


def ring_attention_fwd_zigzag_local(q_shards, k_shards, v_shards, causal=True, scale=None):
    """The zig-zag ring of R ranks run by one process on one GPU (shard r of
    each list plays rank r, hop t reads shard (r - t) mod R from the lists).
    Same blocks, kernels and merge order as ring_attention_fwd_zigzag.
    Returns per-rank (o, lse)."""
    R = len(q_shards)
    scale = 1.0 / math.sqrt(q_shards[0].shape[-1]) if scale is None else scale
    outs = []
    for r in range(R):
        blocks = (((r - t) % R, k_shards[(r - t) % R], v_shards[(r - t) % R]) for t in range(R))
        outs.append(_zigzag_fwd_rank(q_shards[r], blocks, r, R, causal, scale))
    return outs


def _zigzag_bwd_rank(q, k, v, o, lse, do, rank, world, causal, scale, exchange):
    import torch
    new_acc, add, to_bf16 = _gpu_acc_ops()
    gs = [_GpuRankBwd(q[i], o[i], lse[i], do[i], k.shape[3], scale) for i in range(2)]

    def block_grad(i, kk, vv, c):
        return gs[i].block(kk, vv, c)

    dk, dv = zigzag_backward(k, v, rank, world, causal, block_grad, new_acc, add, exchange)
    return torch.stack([gs[0].dq(), gs[1].dq()]), to_bf16(dk), to_bf16(dv)


def ring_attention_bwd_zigzag(q, k, v, o, lse, do, causal=True, scale=None, group=None):
    """Gradients of zig-zag ring attention over the ranks of `group`: this
    rank's chunk-major shards q, do, o [2,B,c,Hq,d], lse [2,B,Hq,c] (from
    ring_attention_fwd_zigzag) and k, v [2,B,c,Hkv,d] -> (dq, dk, dv) bf16,
    chunk-major, for this rank's shards."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    return _zigzag_bwd_rank(q, k, v, o, lse, do, r, R, causal, scale, _p2p_exchange(group))


def ring_attention_bwd_zigzag_local(q_shards, k_shards, v_shards, o_shards, lse_shards, do_shards, causal=True,
                                    scale=None):
    """The zig-zag ring backward of R ranks run by one process on one GPU,
    hop by hop (at hop t every rank r works on shard (r - t) mod R, whose
    accumulators receive their partials in the same order as on the ring).
    Returns per-rank (dq, dk, dv), chunk-major."""
    import torch
    R = len(q_shards)
    scale = 1.0 / math.sqrt(q_shards[0].shape[-1]) if scale is None else scale
    new_acc, add, to_bf16 = _gpu_acc_ops()
    gs = [[_GpuRankBwd(q_shards[r][i], o_shards[r][i], lse_shards[r][i], do_shards[r][i], k_shards[r].shape[3],
                       scale) for i in range(2)] for r in range(R)]
    acc_k = [new_acc(x) for x in k_shards]
    acc_v = [new_acc(x) for x in v_shards]
    for t in range(R):
        for r in range(R):
            src = (r - t) % R
            started = set()
            for i, j, mode in zigzag_schedule(r, R, causal)[t][2]:
                dk_t, dv_t = gs[r][i].block(k_shards[src][j], v_shards[src][j], mode == "causal")
                first = t == 0 and j not in started
                add(acc_k[src][j], dk_t, first)
                add(acc_v[src][j], dv_t, first)
                started.add(j)
    return [(torch.stack([gs[r][0].dq(), gs[r][1].dq()]), to_bf16(acc_k[r]), to_bf16(acc_v[r])) for r in range(R)]
