"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module only draws random numbers and rounds them to the storage formats
the kernels read (bf16, e4m3 with per-block scales); it holds none of the
attention arithmetic. Recipes (the workloads the pages describe in words; no
public dataset is involved):

* Q, K, V, dO: i.i.d. N(0, 1) float32 from ``numpy.random.default_rng(seed)``,
  drawn in the fixed order Q, K, V, dO, then rounded to bf16 (round to nearest
  even, by torch's float32 -> bfloat16 conversion).
* varlen lengths: ``default_rng(seed + 1).integers(lo, hi + 1, nseq)``.
* sampled query rows of long-context checks: ``default_rng(seed + 2)``, R
  distinct rows per head, always including rows 0 and N-1.
* fp8: N(0, 1) float32 with each entry independently (probability 0.001)
  multiplied by 20 (outliers), then per (batch, head, 128-row block) scale
  s = amax / 448 (1 when the block is all zero) and codes = e4m3(x / s) with
  round-to-nearest-even (torch's float32 -> float8_e4m3fn conversion).
"""

from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0


def normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """float32 numpy -> CPU bf16 tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def qkv_bf16(seed: int, B: int, N: int, Hq: int, Hkv: int, d: int, with_dout: bool = False):
    """Padded BSHD inputs [B,N,H,d] as CPU bf16 tensors: (q, k, v[, dout])."""
    rng = np.random.default_rng(seed)
    q = to_bf16(normal_f32(rng, (B, N, Hq, d)))
    k = to_bf16(normal_f32(rng, (B, N, Hkv, d)))
    v = to_bf16(normal_f32(rng, (B, N, Hkv, d)))
    if not with_dout:
        return q, k, v
    do = to_bf16(normal_f32(rng, (B, N, Hq, d)))
    return q, k, v, do


def varlen_lengths(seed: int, nseq: int = 24, lo: int = 128, hi: int = 4096) -> np.ndarray:
    return np.random.default_rng(seed + 1).integers(lo, hi + 1, nseq).astype(np.int64)


def cu_seqlens_of(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def qkv_varlen_bf16(seed: int, lengths, Hq: int, Hkv: int, d: int, with_dout: bool = False):
    """Packed inputs [T,H,d] as CPU bf16 tensors plus cu_seqlens (int32 numpy)."""
    cu = cu_seqlens_of(lengths)
    T = int(cu[-1])
    rng = np.random.default_rng(seed)
    q = to_bf16(normal_f32(rng, (T, Hq, d)))
    k = to_bf16(normal_f32(rng, (T, Hkv, d)))
    v = to_bf16(normal_f32(rng, (T, Hkv, d)))
    out = [q, k, v]
    if with_dout:
        out.append(to_bf16(normal_f32(rng, (T, Hq, d))))
    return (*out, cu)


def sample_rows(seed: int, N: int, Hq: int, R: int = 256) -> np.ndarray:
    """[Hq, R] sorted distinct query rows per head, rows 0 and N-1 always included."""
    rng = np.random.default_rng(seed + 2)
    R = min(R, N)
    out = np.empty((Hq, R), dtype=np.int64)
    for h in range(Hq):
        if N <= 2:
            out[h] = np.arange(N)[:R]
            continue
        mid = rng.choice(np.arange(1, N - 1), size=R - 2, replace=False)
        out[h] = np.sort(np.concatenate([[0, N - 1], mid]))
    return out


def _quantize_blocks(x: np.ndarray, block: int = 128):
    """x [B,N,H,d] float32 -> (codes float8_e4m3fn tensor [B,N,H,d], scales [B,H,nblk] f32)."""
    B, N, H, d = x.shape
    nblk = (N + block - 1) // block
    pad = nblk * block - N
    xp = np.pad(x, ((0, 0), (0, pad), (0, 0), (0, 0)))
    xb = xp.reshape(B, nblk, block, H, d)
    amax = np.abs(xb).max(axis=(2, 4))  # [B,nblk,H]
    s = np.where(amax > 0, amax / E4M3_MAX, 1.0).astype(np.float32)
    s_bh = np.ascontiguousarray(s.transpose(0, 2, 1))  # [B,H,nblk]
    per_row = np.repeat(s, block, axis=1)[:, :N]  # [B,N,H]
    y = (x / per_row[..., None]).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn)
    return codes, torch.from_numpy(s_bh)


def qkv_fp8(seed: int, B: int, N: int, Hq: int, Hkv: int, d: int, outlier_p: float = 1e-3,
            outlier_mul: float = 20.0):
    """fp8 workload: returns dict with float32 originals and block-scaled e4m3 codes."""
    rng = np.random.default_rng(seed)
    out = {}
    for name, H in (("q", Hq), ("k", Hkv), ("v", Hkv)):
        x = normal_f32(rng, (B, N, H, d))
        mask = rng.random(size=x.shape) < outlier_p
        x = np.where(mask, x * np.float32(outlier_mul), x).astype(np.float32)
        codes, scales = _quantize_blocks(x)
        out[name + "_f32"] = x
        out[name + "8"] = codes
        out[name + "_scale"] = scales
    return out
