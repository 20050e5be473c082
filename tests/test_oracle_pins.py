"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each test would fail on a plausible slip in ``oracle/`` (a dropped term, a
wrong sign or index, a transposed operand, a wrong GQA mapping or mask):
closed-form worked examples (tests/golden), invariants of the definition of
exact attention, brute force on tiny inputs, finite differences of the
forward, an independent library routine (torch's fp64 CPU scaled dot-product
attention and autograd), and the tiled online-softmax algorithm.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.attention import attention_head
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "closed_form.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --- closed forms -----------------------------------------------------------

def test_golden_closed_forms():
    cases = json.load(open(GOLD))["cases"]
    for c in cases:
        q, k, v = (np.array(c[n])[None, :, None, :] for n in ("q", "k", "v"))
        O, L = oracle.attn_fwd(q, k, v, c["causal"], c["scale"])
        np.testing.assert_allclose(O[0, :, 0], np.array(c["o"]), rtol=0, atol=1e-13)
        np.testing.assert_allclose(L[0, 0], np.array(c["lse"]), rtol=0, atol=1e-13)
        if "do" in c:
            do = np.array(c["do"])[None, :, None, :]
            dq, dk, dv = oracle.attn_bwd(q, k, v, do, c["causal"], c["scale"])
            np.testing.assert_allclose(dq[0, :, 0], np.array(c["dq"]), atol=1e-13)
            np.testing.assert_allclose(dk[0, :, 0], np.array(c["dk"]), atol=1e-13)
            np.testing.assert_allclose(dv[0, :, 0], np.array(c["dv"]), atol=1e-13)


# --- invariants (C4 - C6f) --------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    q, k, v = _rand((37, 8), 1), _rand((37, 8), 2), _rand((37, 8), 3)
    _, lse, P = attention_head(q, k, v, causal, 0.3)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    if causal:
        assert np.all(np.triu(P, 1) == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_v_all_ones_gives_ones(causal):
    q, k = _rand((2, 50, 3, 16), 4), _rand((2, 50, 3, 16), 5)
    v = np.ones((2, 50, 3, 16))
    O, _ = oracle.attn_fwd(q, k, v, causal, 0.25)
    assert np.max(np.abs(O - 1.0)) <= 1e-14
    dq, dk, dv = oracle.attn_bwd(q, k, v, _rand((2, 50, 3, 16), 6), causal, 0.25)
    assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12


def test_causal_row0_is_v0():
    q, k, v = _rand((1, 40, 2, 8), 7), _rand((1, 40, 2, 8), 8), _rand((1, 40, 2, 8), 9)
    O, L = oracle.attn_fwd(q, k, v, True, 0.7)
    np.testing.assert_allclose(O[:, 0], v[:, 0], atol=1e-14)
    np.testing.assert_allclose(L[0, :, 0], 0.7 * np.einsum("hd,hd->h", q[0, 0], k[0, 0]), atol=1e-13)


def test_single_key():
    q, k, v = _rand((3, 1, 2, 8), 10), _rand((3, 1, 2, 8), 11), _rand((3, 1, 2, 8), 12)
    for causal in (False, True):
        O, L = oracle.attn_fwd(q, k, v, causal, 0.5)
        np.testing.assert_allclose(O, v, atol=1e-14)
        np.testing.assert_allclose(L, 0.5 * np.einsum("bnhd,bnhd->bhn", q, k), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_is_uniform(causal):
    N = 33
    q = np.zeros((1, N, 1, 4))
    k, v = _rand((1, N, 1, 4), 13), _rand((1, N, 1, 4), 14)
    O, L = oracle.attn_fwd(q, k, v, causal, 1.0)
    if causal:
        want = np.cumsum(v[0, :, 0], axis=0) / np.arange(1, N + 1)[:, None]
        lse = np.log(np.arange(1, N + 1))
    else:
        want = np.broadcast_to(v[0, :, 0].mean(axis=0), (N, 4))
        lse = np.full(N, np.log(N))
    np.testing.assert_allclose(O[0, :, 0], want, atol=1e-13)
    np.testing.assert_allclose(L[0, 0], lse, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift(causal):
    q, k, v = _rand((1, 30, 1, 6), 15), _rand((1, 30, 1, 6), 16), _rand((1, 30, 1, 6), 17)
    u = _rand((6,), 18)
    O1, L1 = oracle.attn_fwd(q, k, v, causal, 0.4)
    O2, L2 = oracle.attn_fwd(q, k + u, v, causal, 0.4)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(L2[0, 0], L1[0, 0] + 0.4 * q[0, :, 0] @ u, atol=1e-12)


def test_kv_permutation_noncausal():
    q, k, v = _rand((1, 25, 2, 6), 19), _rand((1, 25, 2, 6), 20), _rand((1, 25, 2, 6), 21)
    perm = np.random.default_rng(22).permutation(25)
    O1, L1 = oracle.attn_fwd(q, k, v, False, 0.4)
    O2, L2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], False, 0.4)
    np.testing.assert_allclose(O2, O1, atol=1e-13)
    np.testing.assert_allclose(L2, L1, atol=1e-13)


def test_bwd_equal_keys_zero_dq():
    q, v, do = _rand((1, 12, 1, 5), 23), _rand((1, 12, 1, 5), 24), _rand((1, 12, 1, 5), 25)
    k = np.broadcast_to(_rand((5,), 26), (1, 12, 1, 5)).copy()
    dq, _, _ = oracle.attn_bwd(q, k, v, do, False, 0.9)
    assert np.max(np.abs(dq)) < 1e-12


# --- brute force and an independent library routine ------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_loops(causal):
    """Pure-Python triple loop on a tiny case (no matmul, no vectorised softmax)."""
    N, d, scale = 5, 3, 0.8
    q, k, v = _rand((N, d), 27), _rand((N, d), 28), _rand((N, d), 29)
    O, L, _ = attention_head(q, k, v, causal, scale)
    import math
    for i in range(N):
        keys = [j for j in range(N) if not (causal and j > i)]
        s = [scale * sum(q[i, c] * k[j, c] for c in range(d)) for j in keys]
        den = sum(math.exp(x) for x in s)
        for c in range(d):
            assert abs(O[i, c] - sum(math.exp(x) * v[j, c] for x, j in zip(s, keys)) / den) < 1e-13
        assert abs(L[i] - math.log(den)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(causal):
    B, N, Hq, Hkv, d, scale = 2, 70, 4, 2, 16, 0.3
    q, k, v = _rand((B, N, Hq, d), 30), _rand((B, N, Hkv, d), 31), _rand((B, N, Hkv, d), 32)
    do = _rand((B, N, Hq, d), 33)
    O, L = oracle.attn_fwd(q, k, v, causal, scale)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, scale)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64).transpose(1, 2).requires_grad_() for x in (q, k, v))
    rep = Hq // Hkv
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(rep, dim=1), tv.repeat_interleave(rep, dim=1), is_causal=causal, scale=scale)
    np.testing.assert_allclose(O, to.detach().transpose(1, 2).numpy(), atol=1e-12)
    to.backward(torch.tensor(do).transpose(1, 2))
    np.testing.assert_allclose(dq, tq.grad.transpose(1, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.transpose(1, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.transpose(1, 2).numpy(), atol=1e-11)
    # LSE pinned by torch's logsumexp of the scaled, masked scores
    s = scale * torch.einsum("bhnd,bhmd->bhnm", tq.detach(), tk.detach().repeat_interleave(rep, dim=1))
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


# --- finite differences (C8) -------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    B, N, H, d, scale = 1, 8, 1, 4, 0.6
    q, k, v = _rand((B, N, H, d), 34), _rand((B, N, H, d), 35), _rand((B, N, H, d), 36)
    W = _rand((B, N, H, d), 37)
    dq, dk, dv = oracle.attn_bwd(q, k, v, W, causal, scale)

    def loss(q_, k_, v_):
        return float(np.sum(oracle.attn_fwd(q_, k_, v_, causal, scale)[0] * W))

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (loss(**{a + "_": b for a, b in args_p.items()}) -
                        loss(**{a + "_": b for a, b in args_m.items()})) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


# --- structure: GQA, varlen, sampled rows, merge (C8b, C8c, C10) ------------

def test_gqa_equals_repeated_mha():
    B, N, Hq, Hkv, d = 1, 20, 6, 2, 8
    q, k, v, do = (_rand((B, N, h, d), s) for h, s in ((Hq, 38), (Hkv, 39), (Hkv, 40), (Hq, 41)))
    O, L = oracle.attn_fwd(q, k, v, True, 0.35)
    kr, vr = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
    O2, L2 = oracle.attn_fwd(q, kr, vr, True, 0.35)
    np.testing.assert_allclose(O, O2, atol=1e-14)
    np.testing.assert_allclose(L, L2, atol=1e-14)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, True, 0.35)
    dq2, dk2, dv2 = oracle.attn_bwd(q, kr, vr, do, True, 0.35)
    np.testing.assert_allclose(dq, dq2, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, N, Hkv, 3, d).sum(axis=3), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, N, Hkv, 3, d).sum(axis=3), atol=1e-13)
    # contiguous groups: query head 1 reads kv head 0, query head 3 reads kv head 1
    assert oracle.kv_head_of(1, 6, 2) == 0 and oracle.kv_head_of(3, 6, 2) == 1


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_separate(causal):
    lengths = [5, 1, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T, H, d = cu[-1], 2, 8
    q, k, v, do = (_rand((T, H, d), s) for s in (42, 43, 44, 45))
    O, L = oracle.attn_fwd_varlen(q, k, v, cu, causal, 0.5)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu, causal, 0.5)
    for s in range(len(lengths)):
        a, e = cu[s], cu[s + 1]
        Os, Ls = oracle.attn_fwd(q[None, a:e], k[None, a:e], v[None, a:e], causal, 0.5)
        np.testing.assert_allclose(O[a:e], Os[0], atol=1e-14)
        np.testing.assert_allclose(L[:, a:e], Ls[0], atol=1e-14)
        g = oracle.attn_bwd(q[None, a:e], k[None, a:e], v[None, a:e], do[None, a:e], causal, 0.5)
        for x, y in zip((dq, dk, dv), g):
            np.testing.assert_allclose(x[a:e], y[0], atol=1e-13)


def test_sampled_rows_match_full():
    q, k, v = _rand((2, 40, 4, 8), 46), _rand((2, 40, 2, 8), 47), _rand((2, 40, 2, 8), 48)
    rows = synth.sample_rows(0, 40, 4, R=10)
    O, L = oracle.attn_fwd(q, k, v, True, 0.3)
    Or, Lr = oracle.attn_fwd_rows(q, k, v, True, 0.3, rows)
    for h in range(4):
        np.testing.assert_allclose(Or[:, h], O[:, rows[h], h], atol=1e-14)
        np.testing.assert_allclose(Lr[:, h], L[:, h, rows[h]], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_backward_against_autograd(causal):
    """attn_bwd_rows: torch fp64 SDPA autograd with dO zeroed outside each
    head's sampled rows gives the sampled rows' dQ and exactly their share of
    dK, dV (a query row's dQ needs only its own dO row)."""
    B, N, Hq, Hkv, d, scale = 2, 40, 4, 2, 8, 0.35
    q, k, v = _rand((B, N, Hq, d), 60), _rand((B, N, Hkv, d), 61), _rand((B, N, Hkv, d), 62)
    do = _rand((B, N, Hq, d), 63)
    rows = synth.sample_rows(1, N, Hq, R=9)
    dq, dk, dv = oracle.attn_bwd_rows(q, k, v, do, causal, scale, rows)
    keep = np.zeros((N, Hq))
    for h in range(Hq):
        keep[rows[h], h] = 1.0
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64).transpose(1, 2).requires_grad_() for x in (q, k, v))
    rep = Hq // Hkv
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(rep, dim=1), tv.repeat_interleave(rep, dim=1), is_causal=causal, scale=scale)
    to.backward(torch.tensor(do * keep[None, :, :, None]).transpose(1, 2))
    gq = tq.grad.transpose(1, 2).numpy()
    for h in range(Hq):
        np.testing.assert_allclose(dq[:, h], gq[:, rows[h], h], atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.transpose(1, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.transpose(1, 2).numpy(), atol=1e-12)


def test_sampled_rows_backward_partition_sums_to_full():
    """Over a partition of every head's rows the contributions add up to the
    full gradient, and the rows' dQ are the full dQ's rows."""
    B, N, Hq, Hkv, d, scale = 1, 24, 2, 1, 8, 0.4
    q, k, v = _rand((B, N, Hq, d), 64), _rand((B, N, Hkv, d), 65), _rand((B, N, Hkv, d), 66)
    do = _rand((B, N, Hq, d), 67)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, True, scale)
    perm = np.random.default_rng(68).permutation(N)
    parts = [np.stack([perm[:10]] * Hq), np.stack([perm[10:]] * Hq)]
    sk, sv = np.zeros_like(dk), np.zeros_like(dv)
    for rows in parts:
        rq, rk, rv = oracle.attn_bwd_rows(q, k, v, do, True, scale, rows)
        for h in range(Hq):
            np.testing.assert_allclose(rq[:, h], dq[:, rows[h], h], atol=1e-13)
        sk += rk
        sv += rv
    np.testing.assert_allclose(sk, dk, atol=1e-12)
    np.testing.assert_allclose(sv, dv, atol=1e-12)


def test_merge_partials_reproduces_full():
    N, d = 29, 8
    q, k, v = _rand((N, d), 49), _rand((N, d), 50), _rand((N, d), 51)
    O, L, _ = attention_head(q, k, v, False, 0.4)
    parts = [(0, 7), (7, 8), (8, 29)]
    outs, lses = [], []
    for a, e in parts:
        o, l, _ = attention_head(q, k[a:e], v[a:e], False, 0.4)
        outs.append(o)
        lses.append(l)
    Om, Lm = oracle.merge_partials(outs, lses)
    np.testing.assert_allclose(Om, O, atol=1e-12)
    np.testing.assert_allclose(Lm, L, atol=1e-12)


# --- the tiled online-softmax algorithm (C7) --------------------------------

@pytest.mark.parametrize("N,d,bm,bn", [(1, 4, 16, 16), (7, 4, 16, 16), (64, 64, 16, 32), (130, 4, 32, 16),
                                        (130, 64, 32, 32)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_tiled_equals_untiled(N, d, bm, bn, causal, tau):
    rng = np.random.default_rng(N * 100 + d)
    q, k, v = (rng.standard_normal((N, d)) * 3 for _ in range(3))
    O, L, _ = attention_head(q, k, v, causal, 1 / np.sqrt(d))
    Ot, Lt = oracle.attn_head_tiled(q, k, v, causal, 1 / np.sqrt(d), bm, bn, tau)
    np.testing.assert_allclose(Ot, O, atol=1e-12)
    np.testing.assert_allclose(Lt, L, atol=1e-12)


# --- fp8 dequantisation -----------------------------------------------------

def test_dequantize_blockscaled_by_hand():
    codes = np.zeros((1, 130, 1, 2))
    codes[0, 0, 0] = [1.0, -2.0]
    codes[0, 129, 0] = [3.0, 0.5]
    scales = np.array([[[0.25, 4.0]]])  # block 0 rows 0..127, block 1 rows 128..129
    x = oracle.dequantize_blockscaled(codes, scales)
    np.testing.assert_array_equal(x[0, 0, 0], [0.25, -0.5])
    np.testing.assert_array_equal(x[0, 129, 0], [12.0, 2.0])


def test_fp8_synth_roundtrip_error_bounded():
    """e4m3 has 3 mantissa bits: |x - s*code| <= s * 2**-4 * 2**e for each element."""
    d = synth.qkv_fp8(0, 1, 256, 2, 2, 64)
    x = d["q_f32"].astype(np.float64)
    xh = oracle.dequantize_blockscaled(d["q8"].float(), d["q_scale"])
    rel = np.abs(x - xh) / np.maximum(np.abs(x), 1e-30)
    small = np.abs(x) < 2 ** -6 * d["q_scale"].numpy().max()
    assert np.all(rel[~small] <= 2 ** -4 + 1e-7)


def test_dequantize_f32_without_rotation_by_hand():
    """Power-of-two scales make every product exact: the float32 steps equal
    the values by hand (and the fp64 definition)."""
    codes = np.zeros((1, 130, 1, 4), dtype=np.float32)
    codes[0, 0, 0] = [1.0, -2.0, 448.0, 0.001953125]
    codes[0, 129, 0] = [3.0, 0.5, -0.75, 0.0]
    scales = np.array([[[0.25, 4.0]]], dtype=np.float32)
    x = oracle.dequantize_f32(codes, scales)
    assert x.dtype == np.float32
    np.testing.assert_array_equal(x[0, 0, 0], [0.25, -0.5, 112.0, 0.00048828125])
    np.testing.assert_array_equal(x[0, 129, 0], [12.0, 2.0, -3.0, 0.0])
    np.testing.assert_array_equal(x, oracle.dequantize_blockscaled(codes, scales))


def test_dequantize_f32_unrotate_inverts_the_rotation():
    """H_d/sqrt(d) is its own inverse (H_d H_d = d I): with unit scales the
    unrotated values are the codes times H_d / sqrt(d) (closed form, fp64),
    and quantise(rotate(x)) -> dequantise(unrotate) returns x within the
    e4m3 step of the rotated block."""
    rng = np.random.default_rng(3)
    d = 64
    codes = torch.from_numpy(rng.standard_normal((1, 5, 2, d)).astype(np.float32)).to(torch.float8_e4m3fn).float()
    x = oracle.dequantize_f32(codes.numpy(), np.ones((1, 2, 1), dtype=np.float32), unrotate=True)
    want = codes.double().numpy() @ (oracle.hadamard(d) / np.sqrt(d))
    np.testing.assert_allclose(x, want, rtol=0, atol=2e-5 * np.abs(want).max())
    xs = rng.standard_normal((1, 200, 2, d)).astype(np.float32)
    c, s = oracle.quantize_blockscaled(oracle.rotate_f32(xs))
    back = oracle.dequantize_f32(c, s, unrotate=True)
    # each rotated entry is off by at most half an e4m3 step (2**-4 relative,
    # amax/448 * 2**-9 absolute below the normal range); the orthogonal
    # unrotation keeps the per-row 2-norm of that error
    err = np.linalg.norm((back - xs).astype(np.float64), axis=-1)
    bound = np.linalg.norm(oracle.rotate_f32(xs).astype(np.float64), axis=-1) * 2 ** -4 + \
        np.sqrt(d) * s.max() * 2 ** -9 + 1e-6
    assert np.all(err <= bound)


# --- decode against a KV cache (bottom-right causal alignment) -------------

def test_kvcache_full_cache_equals_causal_self_attention():
    """With Nq = L = Ncache every row of the cache is a query: the causal
    decode result is ordinary causal attention."""
    B, N, Hq, Hkv, d = 2, 9, 4, 2, 8
    q, k, v = _rand((B, N, Hq, d), 60), _rand((B, N, Hkv, d), 61), _rand((B, N, Hkv, d), 62)
    O, L = oracle.attn_fwd_kvcache(q, k, v, [N, N], True, 0.4)
    O2, L2 = oracle.attn_fwd(q, k, v, True, 0.4)
    np.testing.assert_allclose(O, O2, atol=1e-13)
    np.testing.assert_allclose(L, L2, atol=1e-13)


def test_kvcache_rows_against_brute_force():
    """Per-row brute force with Python loops: lengths shorter than the cache,
    bottom-right causal positions, an empty cache row, GQA mapping."""
    import math
    B, Nq, Hq, Hkv, Nc, d, scale = 3, 3, 4, 2, 10, 5, 0.7
    q, k, v = _rand((B, Nq, Hq, d), 63), _rand((B, Nc, Hkv, d), 64), _rand((B, Nc, Hkv, d), 65)
    lens = [10, 2, 0]
    for causal in (False, True):
        O, L = oracle.attn_fwd_kvcache(q, k, v, lens, causal, scale)
        for b in range(B):
            for h in range(Hq):
                g = h // 2
                for i in range(Nq):
                    vis = [j for j in range(lens[b]) if not (causal and j > lens[b] - Nq + i)]
                    if not vis:
                        assert np.all(O[b, i, h] == 0) and L[b, h, i] == -np.inf
                        continue
                    sc = [scale * sum(q[b, i, h, c] * k[b, j, g, c] for c in range(d)) for j in vis]
                    den = sum(math.exp(x) for x in sc)
                    want = [sum(math.exp(x) * v[b, j, g, c] for x, j in zip(sc, vis)) / den for c in range(d)]
                    np.testing.assert_allclose(O[b, i, h], want, atol=1e-12)
                    assert abs(L[b, h, i] - math.log(den)) < 1e-12


def test_kvcache_split_merge_reproduces_whole_cache():
    """Split-KV: attention over disjoint key ranges merged by LSE equals
    attention over the whole cache (the combination the decode path uses)."""
    B, Nq, Hq, Hkv, Nc, d = 1, 2, 2, 1, 37, 8
    q, k, v = _rand((B, Nq, Hq, d), 66), _rand((B, Nc, Hkv, d), 67), _rand((B, Nc, Hkv, d), 68)
    O, L = oracle.attn_fwd_kvcache(q, k, v, [Nc], False, 0.5)
    outs, lses = [], []
    for a, e in ((0, 16), (16, 32), (32, 37)):
        o, l = oracle.attn_fwd_kvcache(q, k[:, a:e], v[:, a:e], [e - a], False, 0.5)
        outs.append(o)
        lses.append(l.transpose(0, 2, 1))  # [B,Nq,Hq] to match O's row layout
    Om, Lm = oracle.merge_partials(outs, lses)
    np.testing.assert_allclose(Om, O, atol=1e-12)
    np.testing.assert_allclose(Lm.transpose(0, 2, 1), L, atol=1e-12)


# ---------------------------------------------------------------- fp8 incoherent processing
# Pins of oracle/quant.py: Sylvester's Hadamard matrix, the float32 butterfly
# transform against it, the invariance of the scores under the orthogonal
# rotation, and the block-scaled e4m3 quantiser (amax -> 448, RNE, zero
# blocks, ragged last block).

def test_hadamard_definition():
    H2 = oracle.hadamard(2)
    assert np.array_equal(H2, np.array([[1.0, 1.0], [1.0, -1.0]]))
    for d in (1, 4, 64, 128):
        H = oracle.hadamard(d)
        assert np.array_equal(H, H.T)
        assert np.array_equal(np.abs(H), np.ones((d, d)))
        assert np.array_equal(H @ H.T, d * np.eye(d))
    with pytest.raises(ValueError):
        oracle.hadamard(96)


def test_fwht_matches_matrix_exactly_on_integers():
    rng = np.random.default_rng(5)
    for d in (2, 8, 64, 128):
        x = rng.integers(-1000, 1000, (7, d)).astype(np.float32)  # every partial sum exact in float32
        assert np.array_equal(oracle.fwht_f32(x), (x.astype(np.float64) @ oracle.hadamard(d)).astype(np.float32))


def test_rotation_spreads_a_one_hot_outlier_evenly():
    d = 128
    x = np.zeros((1, d), dtype=np.float32)
    x[0, 37] = 20.0
    y = oracle.rotate_f32(x)
    # row 37 of H has entries +-1: every entry becomes +-20/sqrt(d)
    assert np.allclose(np.abs(y), 20.0 / np.sqrt(d), rtol=1e-6)
    assert np.array_equal(np.sign(y[0]), oracle.hadamard(d)[37])


def test_rotation_preserves_scores_and_attention():
    rng = np.random.default_rng(6)
    B, N, H, d = 1, 40, 2, 64
    q = rng.standard_normal((B, N, H, d))
    k = rng.standard_normal((B, N, H, d))
    v = rng.standard_normal((B, N, H, d))
    R = oracle.hadamard(d) / np.sqrt(d)  # orthogonal
    assert np.abs(R @ R.T - np.eye(d)).max() < 1e-14
    O0, L0 = oracle.attn_fwd(q, k, v, True, 0.125)
    O1, L1 = oracle.attn_fwd(q @ R, k @ R, v, True, 0.125)
    assert np.abs(O0 - O1).max() < 1e-12 and np.abs(L0 - L1).max() < 1e-12
    # the float32 butterfly rotation agrees with the fp64 matrix to float32 accuracy
    qr = oracle.rotate_f32(q.astype(np.float32))
    assert np.abs(qr - q @ R).max() < 1e-5


def test_quantize_blockscaled_pins():
    rng = np.random.default_rng(7)
    B, N, H, d = 2, 300, 2, 64  # three blocks, the last one 44 rows
    x = rng.standard_normal((B, N, H, d)).astype(np.float32)
    x[1, 256:, 1] = 0.0  # an all-zero block
    codes, s = oracle.quantize_blockscaled(x)
    assert s.shape == (B, H, 3) and s[1, 1, 2] == 1.0
    assert np.all(codes[1, 256:, 1] == 0)
    for b in range(B):
        for h in range(H):
            for j in range(3):
                blk = x[b, j * 128:(j + 1) * 128, h]
                c = codes[b, j * 128:(j + 1) * 128, h]
                amax = np.abs(blk).max()
                if amax == 0:
                    continue
                assert s[b, h, j] == np.float32(amax) / np.float32(448.0)
                assert np.abs(c).max() == 448.0  # the block's largest entry maps to the largest code
                err = np.abs(c.astype(np.float64) * s[b, h, j] - blk)
                # e4m3: 3 mantissa bits (relative half-step 2^-4), subnormal step 2^-9 (half 2^-10)
                assert np.all(err <= np.maximum(np.abs(blk) * 2.0 ** -4, s[b, h, j] * 2.0 ** -10) * (1 + 1e-6))
    # round to nearest even at e4m3 midpoints (spacing 1/8 in [1, 2))
    y = np.array([448.0, 1.0625, 1.1875, -1.0625], dtype=np.float32).reshape(1, 4, 1, 1)
    c, s1 = oracle.quantize_blockscaled(y)
    assert s1[0, 0, 0] == 1.0
    assert list(c.reshape(-1)) == [448.0, 1.0, 1.25, -1.0]


def test_block_gradients_sum_to_full_gradient():
    """Ring backward (reading): the per-key-block contributions, each using
    the full rows' O and LSE, add up to the gradient of full attention; the
    causal sequence split into R shards: diagonal blocks causal, earlier
    blocks full, later blocks absent."""
    rng = np.random.default_rng(9)
    B, N, Hq, Hkv, d, R = 2, 24, 4, 2, 8, 3
    q, k, v, do = (rng.standard_normal((B, N, H, d)) for H in (Hq, Hkv, Hkv, Hq))
    sc = 0.35
    for causal in (True, False):
        O, L = oracle.attn_fwd(q, k, v, causal, sc)
        dq_ref, dk_ref, dv_ref = oracle.attn_bwd(q, k, v, do, causal, sc)
        n = N // R
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        for r in range(R):
            qs = slice(r * n, (r + 1) * n)
            for src in range(R):
                if causal and src > r:
                    continue
                ks = slice(src * n, (src + 1) * n)
                a, bb, c = oracle.attn_bwd_block(q[:, qs], k[:, ks], v[:, ks], do[:, qs], O[:, qs], L[:, :, qs],
                                                 causal and src == r, sc)
                dq[:, qs] += a
                dk[:, ks] += bb
                dv[:, ks] += c
        assert np.abs(dq - dq_ref).max() < 1e-12
        assert np.abs(dk - dk_ref).max() < 1e-12
        assert np.abs(dv - dv_ref).max() < 1e-12


# ---------------------------------------------------------------- block-sparse masks

def test_blocksparse_pins():
    rng = np.random.default_rng(12)
    B, N, Hq, Hkv, d, blk = 2, 40, 4, 2, 8, 8  # 5 blocks of 8 (small block size: the definition's parameter)
    q, k, v = (rng.standard_normal((B, N, H, d)) for H in (Hq, Hkv, Hkv))
    nb = N // blk
    sc = 0.3
    ones = np.ones((Hq, nb, nb), dtype=np.uint8)
    for causal in (False, True):
        # all blocks on: plain attention
        O, L = oracle.attn_fwd_blocksparse(q, k, v, ones, causal, sc, blk)
        O0, L0 = oracle.attn_fwd(q, k, v, causal, sc)
        assert np.abs(O - O0).max() < 1e-12 and np.abs(L - L0).max() < 1e-12
    # block lower-triangular mask with causal: the same as causal alone
    tri = np.tril(ones)
    O, L = oracle.attn_fwd_blocksparse(q, k, v, tri, True, sc, blk)
    O0, L0 = oracle.attn_fwd(q, k, v, True, sc)
    assert np.abs(O - O0).max() < 1e-12
    # block-diagonal mask: each block attends only itself (= separate sequences)
    diag = np.broadcast_to(np.eye(nb, dtype=np.uint8), (Hq, nb, nb)).copy()
    O, L = oracle.attn_fwd_blocksparse(q, k, v, diag, False, sc, blk)
    cu = np.arange(0, N + 1, blk)
    for b in range(B):
        Ov, Lv = oracle.attn_fwd_varlen(q[b], k[b], v[b], cu, False, sc)
        assert np.abs(O[b] - Ov).max() < 1e-12 and np.abs(L[b] - Lv).max() < 1e-12
    # a query block with no visible key block: O = 0, LSE = -inf; other rows unaffected
    m = ones.copy()
    m[1, 2, :] = 0
    O, L = oracle.attn_fwd_blocksparse(q, k, v, m, False, sc, blk)
    assert np.all(O[:, 2 * blk:3 * blk, 1] == 0) and np.all(L[:, 1, 2 * blk:3 * blk] == -np.inf)
    O0, L0 = oracle.attn_fwd(q, k, v, False, sc)
    assert np.abs(O[:, :, 0] - O0[:, :, 0]).max() < 1e-12
    # brute force on one row: a visible-key softmax written out
    m = (rng.random((Hq, nb, nb)) < 0.5).astype(np.uint8)
    m[:, :, 0] = 1
    O, L = oracle.attn_fwd_blocksparse(q, k, v, m, True, sc, blk)
    b, i, h = 1, 27, 3
    g = oracle.kv_head_of(h, Hq, Hkv)
    keys = [j for j in range(N) if j <= i and m[h, i // blk, j // blk]]
    s = np.array([sc * float(np.dot(q[b, i, h], k[b, j, g])) for j in keys])
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.abs(O[b, i, h] - sum(pj * v[b, j, g] for pj, j in zip(p, keys))).max() < 1e-12
    assert abs(L[b, h, i] - (s.max() + np.log(np.exp(s - s.max()).sum()))) < 1e-12


def test_blocksparse_backward_pins():
    rng = np.random.default_rng(13)
    B, N, Hq, Hkv, d, blk = 1, 24, 2, 1, 4, 6  # 4 blocks of 6
    q, k, v, do = (rng.standard_normal((B, N, H, d)) for H in (Hq, Hkv, Hkv, Hq))
    nb = N // blk
    sc = 0.4
    ones = np.ones((Hq, nb, nb), dtype=np.uint8)
    for causal in (False, True):
        g = oracle.attn_bwd_blocksparse(q, k, v, do, ones, causal, sc, blk)
        g0 = oracle.attn_bwd(q, k, v, do, causal, sc)
        for a, b in zip(g, g0):
            assert np.abs(a - b).max() < 1e-12
    # block-diagonal mask: the gradient of separate sequences
    diag = np.broadcast_to(np.eye(nb, dtype=np.uint8), (Hq, nb, nb)).copy()
    g = oracle.attn_bwd_blocksparse(q, k, v, do, diag, True, sc, blk)
    gv = oracle.attn_bwd_varlen(q[0], k[0], v[0], do[0], np.arange(0, N + 1, blk), True, sc)
    for a, b in zip(g, gv):
        assert np.abs(a[0] - b).max() < 1e-12
    # central finite differences of sum(O * dO) on a random mask with an empty query block
    m = (rng.random((Hq, nb, nb)) < 0.6).astype(np.uint8)
    m[0, 1, :] = 0
    dq, dk, dv = oracle.attn_bwd_blocksparse(q, k, v, do, m, True, sc, blk)

    def f(qq, kk, vv):
        O, _ = oracle.attn_fwd_blocksparse(qq, kk, vv, m, True, sc, blk)
        return float((O * do).sum())

    eps = 1e-6
    for arr, grad, idx in ((q, dq, (0, 9, 1, 2)), (k, dk, (0, 3, 0, 1)), (v, dv, (0, 14, 0, 3))):
        a1, a2 = arr.copy(), arr.copy()
        a1[idx] += eps
        a2[idx] -= eps
        args1 = [a1 if arr is x else x for x in (q, k, v)]
        args2 = [a2 if arr is x else x for x in (q, k, v)]
        fd = (f(*args1) - f(*args2)) / (2 * eps)
        assert abs(fd - grad[idx]) < 1e-6
    assert np.all(dq[0, 6:12, 0] == 0)  # the empty query block has no gradient


# ---------------------------------------------------------------- error metrics

def test_error_metrics_by_hand():
    """max-abs and relative RMS (reading 8) on worked values: the reference
    is the second operand and the norm is over the whole tensor."""
    x, y = np.array([1.0, -2.0, 3.0]), np.array([1.0, 1.0, 1.0])
    assert oracle.max_abs(x, y) == 3.0  # |x + y| would give 4
    assert oracle.max_abs(y, y) == 0.0 and oracle.max_abs(np.zeros(0), np.zeros(0)) == 0.0
    y2 = np.array([[3.0, 4.0]])  # ||y|| = 5
    assert abs(oracle.rel_rms(np.array([[3.0, 0.0]]), y2) - 0.8) < 1e-15  # ||x|| = 3 in the denominator: 4/3
    assert oracle.rel_rms(y2, y2) == 0.0
    assert abs(oracle.rel_rms(y2, 2 * y2) - 0.5) < 1e-15 and abs(oracle.rel_rms(2 * y2, y2) - 1.0) < 1e-15
    # the whole tensor, not a mean of per-row ratios: rows [1,0] and [0,100], error 1 in row 0 only
    ref = np.array([[1.0, 0.0], [0.0, 100.0]])
    assert abs(oracle.rel_rms(ref + np.array([[1.0, 0.0], [0.0, 0.0]]), ref) - 1.0 / np.sqrt(10001.0)) < 1e-15
