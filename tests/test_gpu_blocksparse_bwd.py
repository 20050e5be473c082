"""GPU parity of the block-sparse backward (fa_bwd_blocksparse) through the C-ABI.

* All-ones mask: dQ, dK, dV bit-identical to the dense backward (every block
  visited, the same arithmetic).
* Random masks, causal or not, GQA with a different mask per query head,
  d = 64 / 128, ragged N, with query blocks that see nothing and key blocks
  that no query head of their group sees: against the oracle's gradient of
  block-masked attention with the bf16 backward bound (relative RMS <= 1e-2
  on dQ, dK, dV). Rows whose gradient is zero by construction (a query row
  that sees no key; a key row that no visible query sees) must be exactly 0.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

G_REL_RMS = 1e-2


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_27_b200 as m
    return m


def _run(fa, q, k, v, do, mask, causal):
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    md = torch.from_numpy(mask).to(dev)
    o, lse = fa.attention_fwd_blocksparse(qd, kd, vd, md, causal=causal)
    g = fa.attention_bwd_blocksparse(qd, kd, vd, md, o, lse, dod, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    return [t.cpu().double().numpy() for t in g]


def test_all_ones_mask_equals_dense(fa):
    B, N, Hq, Hkv, d = 2, 1000, 4, 2, 128
    q, k, v, do = (t.cuda() for t in synth.qkv_bf16(31, B, N, Hq, Hkv, d, with_dout=True))
    nb = (N + 127) // 128
    mask = torch.ones((Hq, nb, nb), dtype=torch.uint8, device="cuda")
    for causal in (False, True):
        o, lse = fa.attention_fwd(q, k, v, causal=causal)
        g1 = fa.attention_bwd_blocksparse(q, k, v, mask, o, lse, do, causal=causal)
        g2 = fa.attention_bwd(q, k, v, o, lse, do, causal=causal)
        torch.cuda.synchronize()
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


def _zero_rows(mask, N, Hq, Hkv, causal):
    """(query rows [N,Hq], key rows [N,Hkv]) whose gradient is zero by construction."""
    blk = np.arange(N) // 128
    group = Hq // Hkv
    q_zero = np.zeros((N, Hq), dtype=bool)
    k_seen = np.zeros((N, Hkv), dtype=bool)
    for h in range(Hq):
        vis = mask[h][blk[:, None], blk[None, :]] != 0
        if causal:
            vis &= np.arange(N)[None, :] <= np.arange(N)[:, None]
        q_zero[:, h] = ~vis.any(axis=1)
        k_seen[:, h // group] |= vis.any(axis=0)
    return q_zero, ~k_seen


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv,d,density", [(2, 1000, 4, 2, 128, 0.5), (1, 777, 2, 2, 64, 0.3),
                                                  (1, 2048, 2, 1, 128, 0.15), (1, 300, 6, 2, 64, 0.6)])
def test_random_masks_match_oracle(fa, causal, B, N, Hq, Hkv, d, density):
    q, k, v, do = synth.qkv_bf16(N + 7 * Hq, B, N, Hq, Hkv, d, with_dout=True)
    nb = (N + 127) // 128
    rng = np.random.default_rng(N + 1)
    mask = (rng.random((Hq, nb, nb)) < density).astype(np.uint8)
    mask[0, 1, :] = 0             # a query block that sees nothing
    mask[-1, 0, :] = 0
    mask[: Hq // Hkv, :, 2] = 0   # key block 2 of kv head 0: seen by no query head
    got = _run(fa, q, k, v, do, mask, causal)
    want = oracle.attn_bwd_blocksparse(q, k, v, do, mask, causal, 1 / math.sqrt(d))
    q_zero, k_zero = _zero_rows(mask, N, Hq, Hkv, causal)
    dq, dk, dv = got
    assert np.all(dq.transpose(0, 2, 1, 3)[:, q_zero.T] == 0)
    assert np.all(dk.transpose(0, 2, 1, 3)[:, k_zero.T] == 0)
    assert np.all(dv.transpose(0, 2, 1, 3)[:, k_zero.T] == 0)
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert np.all(np.isfinite(g)), name
        rr = oracle.rel_rms(g, w)
        assert rr <= G_REL_RMS, f"{name} rel-RMS {rr}"


def test_empty_mask_gives_zero_gradients(fa):
    B, N, Hq, Hkv, d = 1, 384, 2, 1, 128
    q, k, v, do = synth.qkv_bf16(5, B, N, Hq, Hkv, d, with_dout=True)
    mask = np.zeros((Hq, 3, 3), dtype=np.uint8)
    for g in _run(fa, q, k, v, do, mask, False):
        assert np.all(g == 0)


def test_null_mask_is_an_error(fa):
    q = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_bwd_workspace_size(128, 1, 1, 64), dtype=torch.uint8, device="cuda")
    g = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_blocksparse(q, q, q, None, q, lse, q, *g, ws, ws.numel(), 1, 1, 1, 128, 64, 0, 0.125)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("causal", [False, True])
def test_heavy_key_block_split_matches_oracle(fa, causal):
    """A key block every query block sees (sliding window + global first
    block): its dK/dV units are far longer than the rest and are split into
    chunks whose partial sums are added afterwards; the result must match the
    oracle and be bitwise reproducible."""
    B, N, Hq, Hkv, d = 1, 4096, 4, 2, 128
    q, k, v, do = synth.qkv_bf16(77 + int(causal), B, N, Hq, Hkv, d, with_dout=True)
    nb = N // 128
    mask = np.zeros((Hq, nb, nb), dtype=np.uint8)
    for i in range(nb):
        mask[:, i, max(0, i - 3):i + 1] = 1
        mask[:, i, 0] = 1
        if not causal:
            mask[:, i, i:min(nb, i + 4)] = 1
    got = _run(fa, q, k, v, do, mask, causal)
    again = _run(fa, q, k, v, do, mask, causal)
    for g, h in zip(got, again):
        assert np.array_equal(g, h)
    want = oracle.attn_bwd_blocksparse(q, k, v, do, mask, causal, 1 / math.sqrt(d))
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        rr = oracle.rel_rms(g, w)
        assert rr <= G_REL_RMS, f"{name} rel-RMS {rr}"


def test_split_units_gqa_d64_with_unseen_key_blocks(fa):
    """GQA group 4, d = 64, two global key columns (split units) beside key
    blocks nothing sees (forced zero visits): matches the oracle, the unseen
    blocks' dK/dV rows are exactly 0, bitwise reproducible."""
    B, N, Hq, Hkv, d = 2, 3000, 8, 2, 64
    q, k, v, do = synth.qkv_bf16(91, B, N, Hq, Hkv, d, with_dout=True)
    nb = (N + 127) // 128
    mask = np.zeros((Hq, nb, nb), dtype=np.uint8)
    for i in range(nb):
        mask[:, i, max(0, i - 1):i + 1] = 1
        mask[:, i, 0] = 1
        mask[:, i, 5] = 1
    mask[:, :, 9] = 0   # key block 9: seen by nothing
    mask[:, :, 12] = 0
    got = _run(fa, q, k, v, do, mask, True)
    again = _run(fa, q, k, v, do, mask, True)
    for g, h in zip(got, again):
        assert np.array_equal(g, h)
    _, k_zero = _zero_rows(mask, N, Hq, Hkv, True)
    assert k_zero[9 * 128:10 * 128].all()
    dq, dk, dv = got
    assert np.all(dk.transpose(0, 2, 1, 3)[:, k_zero.T] == 0)
    assert np.all(dv.transpose(0, 2, 1, 3)[:, k_zero.T] == 0)
    want = oracle.attn_bwd_blocksparse(q, k, v, do, mask, True, 1 / math.sqrt(d))
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        rr = oracle.rel_rms(g, w)
        assert rr <= G_REL_RMS, f"{name} rel-RMS {rr}"


def test_workspace_too_small_is_an_error(fa):
    B, N, Hq, Hkv, d = 1, 512, 2, 1, 64
    q = torch.zeros((B, N, Hq, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, N, Hkv, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, Hq, N), dtype=torch.float32, device="cuda")
    mask = torch.ones((Hq, 4, 4), dtype=torch.uint8, device="cuda")
    need = fa.fa_bwd_blocksparse_workspace_size(B, Hq, Hkv, N, d)
    assert need > fa.fa_bwd_workspace_size(B * N, B, Hq, d)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    g = [torch.empty_like(q), torch.empty_like(kv), torch.empty_like(kv)]
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_blocksparse(q, kv, kv, mask, q, lse, q, *g, ws, ws.numel(), B, Hq, Hkv, N, d, 0, 0.125)
    assert e.value.status == fa.FA_ERR_WORKSPACE
