"""fp8 inputs with incoherent processing: a Hadamard rotation along d, then
block-scaled e4m3 quantisation (oracle).

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Source: "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
Low-precision" (summary, contribution 3: FP8 with lower error than per-tensor
quantisation; the technique is not named there). Reading: multiply the rows
of Q and K by an orthogonal Hadamard matrix H_d before quantising them.
Because H_d H_d^T = I, (Q H_d)(K H_d)^T = Q K^T: the scores, and so the
attention, are unchanged; an outlier channel is spread over all d channels,
so a 128-row block's amax, and with it the rounding step of every other
entry, shrinks. V is not rotated.

Definitions followed here:
  * H_d (d a power of two) by Sylvester's construction, H_1 = [1],
    H_2n = [[H_n, H_n], [H_n, -H_n]]; the orthogonal rotation is H_d / sqrt(d).
  * The fast Walsh-Hadamard transform computes x H_d with d/2 butterflies per
    stage: for stage width h = 1, 2, 4, ..., d/2 and every pair (j, j+h) with
    bit h of j clear, (x_j, x_{j+h}) -> (x_j + x_{j+h}, x_j - x_{j+h}). Done
    here in float32, stage by stage, then multiplied by float32(1/sqrt(d)).
  * Block-scaled e4m3: per (batch, head, 128-row block) scale
    s = amax / 448 in float32 (1 for an all-zero block), codes = RNE e4m3 of
    the float32 quotient x / s (torch's float32 -> float8_e4m3fn conversion).
"""

from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0


def hadamard(d: int) -> np.ndarray:
    """Sylvester's Hadamard matrix H_d (entries +-1, float64); d a power of two."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def fwht_f32(x) -> np.ndarray:
    """x H_d along the last axis by the butterfly stages, in float32."""
    y = np.array(x, dtype=np.float32, copy=True)
    d = y.shape[-1]
    h = 1
    while h < d:
        z = y.reshape(*y.shape[:-1], d // (2 * h), 2, h)
        a = z[..., 0, :].copy()
        b = z[..., 1, :].copy()
        z[..., 0, :] = a + b
        z[..., 1, :] = a - b
        h *= 2
    return y


def rotate_f32(x) -> np.ndarray:
    """The orthogonal rotation x H_d / sqrt(d) as the float32 butterflies
    followed by one float32 multiply by float32(1/sqrt(d))."""
    d = np.shape(x)[-1]
    return fwht_f32(x) * np.float32(1.0 / np.sqrt(d))


def quantize_blockscaled(x, block: int = 128):
    """x [B,N,H,d] float32 -> (codes float32 [B,N,H,d] holding the e4m3 values,
    scales float32 [B,H,ceil(N/block)])."""
    x = np.asarray(x, dtype=np.float32)
    B, N, H, d = x.shape
    nblk = (N + block - 1) // block
    scales = np.empty((B, H, nblk), dtype=np.float32)
    codes = np.empty_like(x)
    for j in range(nblk):
        rows = slice(j * block, min(N, (j + 1) * block))
        xb = x[:, rows]  # [B, r, H, d]
        amax = np.abs(xb).max(axis=(1, 3)).astype(np.float32)  # [B, H]
        s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        scales[:, :, j] = s
        q = (xb / s[:, None, :, None]).astype(np.float32)
        codes[:, rows] = torch.from_numpy(np.ascontiguousarray(q)).to(torch.float8_e4m3fn).float().numpy()
    return codes, scales


def dequantize_f32(codes, scales, unrotate: bool = False, block: int = 128) -> np.ndarray:
    """float32 counterpart of attention.dequantize_blockscaled, step by step:
    the values the fp8 forward attends over, restated in the original space
    (the input of the fp8 backward, which differentiates attention on them:
    the straight-through reading of "an fp8 backward").
    codes float32 [B,N,H,d] holding e4m3 values, scales float32 [B,H,nblk].
    Steps, each one float32 operation: y = code * s of the row's block; with
    `unrotate`, the inverse of the rotation, which is the rotation itself
    (H_d / sqrt(d) is symmetric and orthogonal): the same butterflies as
    rotate_f32, then the multiply by float32(1/sqrt(d)). Returns float32."""
    codes = np.asarray(codes, dtype=np.float32)
    scales = np.asarray(scales, dtype=np.float32)
    B, N, H, d = codes.shape
    blk = np.arange(N) // block
    s = scales[:, :, blk]  # [B, H, N]
    y = (codes * np.transpose(s, (0, 2, 1))[..., None]).astype(np.float32)
    return rotate_f32(y) if unrotate else y
