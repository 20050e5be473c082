"""The tiled online-softmax algorithm, in fp64, as an executable specification.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Steps, in the order the pages give them in words (Dao-AILab repository
overview: "online softmax with rescaling, tiled attention with shared-memory
staging"; topic page "Flash Attention and Efficient Transformer Mechanisms":
blocks of Q, K, V are read into on-chip memory and partial attention outputs
are computed): for each block of query rows, walk the key/value blocks, keep a
running row maximum m and running row sum l, rescale the partial output when
the maximum grows, and normalise once at the end.

One refinement is a reading of this library (any choice gives the same exact
result): the maximum is only moved when it grows by more than ``tau`` in base-2
exponent units ("lazy rescaling"); otherwise the stale maximum is kept, so the
unnormalised weights stay below 2**tau.

The tests pin this function to the plain definition in ``attention.py``.
"""

from __future__ import annotations

import numpy as np

LOG2E = 1.4426950408889634


def attn_head_tiled(q, k, v, causal: bool, scale: float, block_m: int = 16, block_n: int = 16,
                    tau: float = 8.0):
    """Tiled attention of one head. q [N,d], k [N,d], v [N,dv]. Returns (O, LSE)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[0]
    Nk = k.shape[0]
    c = scale * LOG2E  # scores are handled in base 2: exp(scale*x) = 2**(c*x)
    O = np.zeros((N, v.shape[1]))
    LSE = np.zeros(N)
    for i0 in range(0, N, block_m):
        rows = np.arange(i0, min(i0 + block_m, N))
        m = np.full(len(rows), -np.inf)  # running max of the raw scores q.k
        l = np.zeros(len(rows))           # running sum of 2**(c*(x - m))
        acc = np.zeros((len(rows), v.shape[1]))
        for j0 in range(0, Nk, block_n):
            cols = np.arange(j0, min(j0 + block_n, Nk))
            if causal and cols[0] > rows[-1]:
                break  # every key of this block lies after every query row
            x = q[rows] @ k[cols].T  # raw scores of the block
            if causal:
                x = np.where(cols[None, :] > rows[:, None], -np.inf, x)
            m_blk = x.max(axis=1)
            grow = np.where(np.isfinite(m_blk), (m_blk - m) * c, -np.inf)
            move = grow > tau
            m_new = np.where(move, m_blk, m)
            alpha = np.where(move, np.exp2((m - m_new) * c), 1.0)
            p = np.exp2((x - m_new[:, None]) * c)
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v[cols]
            m = m_new
        O[rows] = acc / l[:, None]
        LSE[rows] = scale * m + np.log(l)
    return O, LSE
