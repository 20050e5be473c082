"""Plain fp64 definition of exact scaled dot-product attention (oracle).

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Everything is computed in float64 with numpy; the score matrix of each head is
materialised in full (the very thing the GPU path must never do), so the result
is the textbook definition and nothing else.

Definition followed (the catalogue record "Dao and colleagues: IO-aware exact
attention with FlashAttention", field ``summary``: exact attention; the topic
page "Flash Attention and Efficient Transformer Mechanisms", opening paragraph:
"without approximation"). For one (batch, query head) pair with key/value head
g(hq):

    S_ij   = scale * sum_c Q[i,c] K[j,c]          (masked entries are -inf)
    LSE_i  = m_i + ln sum_j exp(S_ij - m_i),      m_i = max_j S_ij
    P_ij   = exp(S_ij - LSE_i)
    O_i    = sum_j P_ij V[j]

Causal mask: key j is hidden from query i when j > i (query and key sequences
have one common length, counted from the start of each sequence).
GQA mapping (reading; the pages do not mention GQA): query head hq reads
key/value head hq // (Hq / Hkv), i.e. contiguous groups.
LSE is the natural log of the *scaled* scores (reading).

Backward (the record's ``summary``: recomputation instead of storing P); the
gradient is ordinary calculus applied to the definition above:

    dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
    dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q

with dK, dV summed over the query heads that share a key/value head.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    """Return ``x`` as a float64 numpy array (torch tensors are upcast exactly)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """Key/value head read by query head ``hq`` (contiguous GQA groups, a reading)."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def attention_head(q, k, v, causal: bool, scale: float, rows=None):
    """Attention of one head: q [Nq,d], k [Nk,d], v [Nk,dv] (Nq == Nk when causal).

    ``rows`` (optional) restricts the computation to those query rows (their
    causal limit is still their own index). Returns (O [R,dv], LSE [R], P [R,Nk]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    qi = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    S = scale * (q[qi] @ k.T)
    if causal:
        hidden = np.arange(k.shape[0])[None, :] > qi[:, None]
        S = np.where(hidden, -np.inf, S)
    m = S.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(S - m).sum(axis=1))
    P = np.exp(S - lse[:, None])
    return P @ v, lse, P


def attn_fwd(q, k, v, causal: bool, scale: float):
    """Padded-batch forward. q [B,N,Hq,d]; k, v [B,N,Hkv,d] (BSHD).

    Returns O [B,N,Hq,d] and LSE [B,Hq,N], both float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    O = np.empty((B, N, Hq, v.shape[3]))
    L = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            O[b, :, h], L[b, h], _ = attention_head(q[b, :, h], k[b, :, g], v[b, :, g], causal, scale)
    return O, L


def attn_fwd_rows(q, k, v, causal: bool, scale: float, rows):
    """Forward on a sample of query rows per head (long-context checks).

    ``rows`` is an int array [Hq, R]: the query rows checked for each head (the
    same rows for every batch entry). Returns O [B,Hq,R,d], LSE [B,Hq,R].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[1]
    O = np.empty((B, Hq, R, v.shape[3]))
    L = np.empty((B, Hq, R))
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            O[b, h], L[b, h], _ = attention_head(q[b, :, h], k[b, :, g], v[b, :, g], causal, scale, rows[h])
    return O, L


def attn_fwd_varlen(q, k, v, cu_seqlens, causal: bool, scale: float):
    """Packed (varlen) forward. q [T,Hq,d]; k, v [T,Hkv,d]; cu_seqlens [nseq+1].

    Sequence s occupies tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 and attends
    only within itself. Returns O [T,Hq,d], LSE [Hq,T].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    O = np.zeros((T, Hq, v.shape[2]))
    L = np.zeros((Hq, T))
    for s in range(len(cu) - 1):
        a, e = cu[s], cu[s + 1]
        if e == a:
            continue
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            O[a:e, h], L[h, a:e], _ = attention_head(q[a:e, h], k[a:e, g], v[a:e, g], causal, scale)
    return O, L


def _bwd_head(q, k, v, do, causal, scale):
    """Analytic gradient of one head, recomputing P from the definition."""
    O, _, P = attention_head(q, k, v, causal, scale)
    dV = P.T @ do
    dP = do @ v.T
    D = (do * O).sum(axis=1, keepdims=True)
    dS = P * (dP - D)
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return dQ, dK, dV


def attn_bwd(q, k, v, dout, causal: bool, scale: float):
    """Padded-batch backward: gradients of sum(O * dout) w.r.t. q, k, v (float64)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            a, bb, c = _bwd_head(q[b, :, h], k[b, :, g], v[b, :, g], do[b, :, h], causal, scale)
            dq[b, :, h] = a
            dk[b, :, g] += bb
            dv[b, :, g] += c
    return dq, dk, dv


def attn_bwd_rows(q, k, v, dout, causal: bool, scale: float, rows):
    """Backward on a sample of query rows per head (long-context checks).

    The same gradient as ``attn_bwd`` (the catalogue record's ``summary``:
    recomputation of P from Q, K, V), restricted to the query rows ``rows``
    [Hq, R] of each head (the same rows for every batch entry): for those
    rows P, dP = dO V^T, D = rowsum(dO * O) and dS = P * (dP - D), then

        dQ[rows] = scale dS K      (exact: a query row's gradient needs only its own row)
        dK      += scale dS^T Q[rows],   dV += P^T dO[rows]   (the rows' share)

    Returns dq [B,Hq,R,d] and the rows' contributions dk, dv [B,N,Hkv,d]
    (float64; summed over the query heads of a kv head). Over a partition of
    the rows the contributions sum to the full dK, dV (pinned)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[1]
    dq = np.empty((B, Hq, R, d))
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            r = rows[h]
            O, _, P = attention_head(q[b, :, h], k[b, :, g], v[b, :, g], causal, scale, r)
            dP = do[b, r, h] @ v[b, :, g].T
            D = (do[b, r, h] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, h] = scale * (dS @ k[b, :, g])
            dk[b, :, g] += scale * (dS.T @ q[b, r, h])
            dv[b, :, g] += P.T @ do[b, r, h]
    return dq, dk, dv


def attn_bwd_varlen(q, k, v, dout, cu_seqlens, causal: bool, scale: float):
    """Packed (varlen) backward: q, dout [T,Hq,d]; k, v [T,Hkv,d]."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    Hq, Hkv = q.shape[1], k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for s in range(len(cu) - 1):
        a, e = cu[s], cu[s + 1]
        if e == a:
            continue
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            x, y, z = _bwd_head(q[a:e, h], k[a:e, g], v[a:e, g], do[a:e, h], causal, scale)
            dq[a:e, h] = x
            dk[a:e, g] += y
            dv[a:e, g] += z
    return dq, dk, dv


def merge_partials(outs, lses):
    """Combine attention over disjoint key sets from each part's (O_r, LSE_r).

    LSE = ln sum_r exp(LSE_r) and O = sum_r exp(LSE_r - LSE) O_r: the exact
    result over the union of the key sets, because each O_r is normalised by
    exp(LSE_r). Shapes: outs [R, ..., d], lses [R, ...].
    """
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    m = lses.max(axis=0)
    lse = m + np.log(np.exp(lses - m).sum(axis=0))
    w = np.exp(lses - lse)
    return (w[..., None] * outs).sum(axis=0), lse


def dequantize_blockscaled(codes, scales, block: int = 128):
    """Values an e4m3 input stands for: codes * scale of its (b, h, row-block).

    codes [B,N,H,d] (the decoded e4m3 values), scales [B,H,ceil(N/block)].
    Follows the FP8 forward-pass contribution of the FlashAttention-3 summary;
    the per-(head, 128-row block) scale granularity is a reading.
    """
    c = _f64(codes)
    s = _f64(scales)
    B, N, H, d = c.shape
    blk = np.arange(N) // block
    per_row = s[:, :, blk]  # [B,H,N]
    return c * per_row.transpose(0, 2, 1)[..., None]


def attn_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, causal: bool, scale: float):
    """Attention of a few new query rows against a key/value cache (decode).

    q [B,Nq,Hq,d]; k_cache, v_cache [B,Ncache,Hkv,d]; cache_seqlens [B]: batch
    b holds L_b valid cache rows (keys 0 .. L_b-1). The queries are the newest
    Nq positions of the sequence: query i sits at position L_b - Nq + i, so
    with causal=True it sees keys 0 .. L_b - Nq + i (readings: the KV-cache API
    of the Dao-AILab repository overview is named there without semantics;
    bottom-right alignment is the decode convention where the newest query
    sees the whole cache). A row that sees no key has O = 0, LSE = -inf.
    Returns O [B,Nq,Hq,d], LSE [B,Hq,Nq] (float64).
    """
    q, k, v = _f64(q), _f64(k_cache), _f64(v_cache)
    L = np.asarray(cache_seqlens, dtype=np.int64)
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    O = np.zeros((B, Nq, Hq, v.shape[3]))
    LSE = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        Lb = int(L[b])
        if Lb <= 0:
            continue
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            S = scale * (q[b, :, h] @ k[b, :Lb, g].T)  # [Nq, Lb]
            if causal:
                pos = Lb - Nq + np.arange(Nq)
                S = np.where(np.arange(Lb)[None, :] > pos[:, None], -np.inf, S)
            for i in range(Nq):
                row = S[i]
                if not np.any(np.isfinite(row)):
                    continue
                m = row.max()
                lse = m + np.log(np.exp(row - m).sum())
                O[b, i, h] = np.exp(row - lse) @ v[b, :Lb, g]
                LSE[b, h, i] = lse
    return O, LSE


def attn_bwd_block(q, k, v, dout, o, lse, causal: bool, scale: float):
    """Gradient contributions of one key block when the query rows' softmax
    statistics come from attention over a larger key set (context-parallel
    ring attention, reading of the topic page's multi-GPU variants).

    q, dout, o [B,N,Hq,d] and lse [B,Hq,N]: the query rows with the O and LSE
    of their full attention; k, v [B,Nk,Hkv,d]: one key block (causal: the
    block on the diagonal, key j hidden from query i when j > i). With
    P = exp(S - LSE) on this block, D = rowsum(dout * o):
        dV = P^T dout,  dS = P * (dout V^T - D),  dQ = scale dS K,  dK = scale dS^T q
    (dK, dV summed over the query heads of a kv head). Summed over disjoint key
    blocks these give the gradient of the full attention (pinned).
    Returns (dq, dk, dv) float64."""
    q, k, v, do, o, L = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(o), _f64(lse)
    B, N, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            S = scale * (q[b, :, h] @ k[b, :, g].T)
            if causal:
                S = np.where(np.arange(Nk)[None, :] > np.arange(N)[:, None], -np.inf, S)
            P = np.exp(S - L[b, h][:, None])
            D = (do[b, :, h] * o[b, :, h]).sum(axis=1, keepdims=True)
            dP = do[b, :, h] @ v[b, :, g].T
            dS = P * (dP - D)
            dq[b, :, h] = scale * (dS @ k[b, :, g])
            dk[b, :, g] += scale * (dS.T @ q[b, :, h])
            dv[b, :, g] += P.T @ do[b, :, h]
    return dq, dk, dv


def attn_fwd_blocksparse(q, k, v, block_mask, causal: bool, scale: float, block: int = 128):
    """Attention with a block-sparse mask (the topic page's block-sparse
    variant; its layout is a reading): key j is hidden from query i when
    block_mask[h, i // block, j // block] == 0 (and, with causal, when j > i).
    q [B,N,Hq,d]; k, v [B,N,Hkv,d]; block_mask [Hq, ceil(N/block),
    ceil(N/block)], shared by the batch. A row that sees no key has O = 0 and
    LSE = -inf. Returns O [B,N,Hq,d], LSE [B,Hq,N] (float64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    M = np.asarray(block_mask) != 0
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    blk = np.arange(N) // block
    O = np.zeros((B, N, Hq, v.shape[3]))
    L = np.full((B, Hq, N), -np.inf)
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        visible = M[h][blk[:, None], blk[None, :]]
        if causal:
            visible &= np.arange(N)[None, :] <= np.arange(N)[:, None]
        for b in range(B):
            S = np.where(visible, scale * (q[b, :, h] @ k[b, :, g].T), -np.inf)
            rows = visible.any(axis=1)
            if not rows.any():
                continue
            Sr = S[rows]
            m = Sr.max(axis=1, keepdims=True)
            lse = m[:, 0] + np.log(np.exp(Sr - m).sum(axis=1))
            O[b, rows, h] = np.exp(Sr - lse[:, None]) @ v[b, :, g]
            L[b, h, rows] = lse
    return O, L


def attn_bwd_blocksparse(q, k, v, dout, block_mask, causal: bool, scale: float, block: int = 128):
    """Gradients of sum(O * dout) for attn_fwd_blocksparse (the same mask
    reading): the analytic gradient of the definition with hidden entries'
    P = 0; a row that sees no key contributes nothing. Returns dq, dk, dv
    (float64; dk, dv summed over the query heads of a kv head)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    M = np.asarray(block_mask) != 0
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    blk = np.arange(N) // block
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        visible = M[h][blk[:, None], blk[None, :]]
        if causal:
            visible &= np.arange(N)[None, :] <= np.arange(N)[:, None]
        rows = visible.any(axis=1)
        for b in range(B):
            S = np.where(visible, scale * (q[b, :, h] @ k[b, :, g].T), -np.inf)
            P = np.zeros_like(S)
            Sr = S[rows]
            m = Sr.max(axis=1, keepdims=True)
            E = np.exp(Sr - m)
            P[rows] = E / E.sum(axis=1, keepdims=True)
            O = P @ v[b, :, g]
            dv[b, :, g] += P.T @ do[b, :, h]
            dP = do[b, :, h] @ v[b, :, g].T
            D = (do[b, :, h] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, :, h] = scale * (dS @ k[b, :, g])
            dk[b, :, g] += scale * (dS.T @ q[b, :, h])
    return dq, dk, dv
