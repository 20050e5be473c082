"""GPU parity of the bf16 backward pass against the fp64 oracle (through the C-ABI).

Tolerance (the stated bf16 bound): relative RMS <= 1e-2 on dQ, dK and dV.
The GPU backward consumes the GPU forward's O and LSE, as a caller would; the
oracle differentiates the exact fp64 attention of the same bf16 inputs.
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


def _check_grads(got, want, tag):
    out = []
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        gn = g.double().cpu().numpy()
        assert np.all(np.isfinite(gn)), f"{tag} {name} not finite"
        rr = oracle.rel_rms(gn, w)
        assert rr <= G_REL_RMS, f"{tag} {name} rel-RMS {rr}"
        out.append(rr)
    return out


def _fwd_bwd_padded(fa, B, N, Hq, Hkv, d, causal, seed):
    q, k, v, do = synth.qkv_bf16(seed, B, N, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    return (q, k, v, do), (dq, dk, dv)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv,d", [
    (1, 1, 1, 1, 128), (1, 7, 2, 1, 64), (2, 127, 2, 2, 128), (1, 129, 4, 2, 128), (2, 300, 3, 1, 128),
    (1, 513, 2, 2, 64), (3, 640, 4, 4, 128), (1, 1000, 8, 2, 128), (1, 256, 2, 2, 64),
])
def test_bwd_padded_shapes(fa, B, N, Hq, Hkv, d, causal):
    (q, k, v, do), got = _fwd_bwd_padded(fa, B, N, Hq, Hkv, d, causal, seed=100 + N)
    want = oracle.attn_bwd(q, k, v, do, causal, 1 / math.sqrt(d))
    _check_grads(got, want, f"B{B} N{N} H{Hq}/{Hkv} d{d} c{causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_config_b4_h16_n2048(fa, causal):
    """Backward of the B=4, Hq=Hkv=16, N=2048, d=128 workload (full oracle comparison)."""
    (q, k, v, do), got = _fwd_bwd_padded(fa, 4, 2048, 16, 16, 128, causal, seed=0)
    want = oracle.attn_bwd(q, k, v, do, causal, 1 / math.sqrt(128))
    _check_grads(got, want, f"cfg2 bwd causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_small(fa, causal):
    lengths = [1, 127, 128, 129, 300, 5, 640, 0, 33]
    q, k, v, do, cu = synth.qkv_varlen_bf16(21, lengths, 4, 2, 128, with_dout=True)
    dev = torch.device("cuda")
    cu_d = torch.from_numpy(cu).to(dev)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cu_d, max(lengths), causal=causal)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, lse, dod, cu_d, max(lengths), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    want = oracle.attn_bwd_varlen(q, k, v, do, cu, causal, 1 / math.sqrt(128))
    _check_grads((dq, dk, dv), want, "varlen small bwd")


@pytest.fixture(scope="module")
def varlen_cfg(fa):
    """The packed causal workload: 24 sequences, lengths U[128,4096] (seed 0),
    H=16, d=128; inputs and the GPU forward + backward, computed once."""
    lengths = synth.varlen_lengths(0)
    H, d = 16, 128
    q, k, v, do, cu = synth.qkv_varlen_bf16(0, lengths, H, H, d, with_dout=True)
    dev = torch.device("cuda")
    cu_d = torch.from_numpy(cu).to(dev)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    mx = int(lengths.max())
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cu_d, mx, causal=True)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, lse, dod, cu_d, mx, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    return (q, k, v, do, cu), tuple(t.cpu() for t in (o, lse, dq, dk, dv))


@pytest.mark.parametrize("heads", [[0, 1, 2, 3], [4, 5, 6, 7], [8, 9, 10, 11], [12, 13, 14, 15]])
def test_config_varlen_fwd_bwd(varlen_cfg, heads):
    """Varlen packed causal forward + backward, every sequence: O, LSE and all
    gradients against the oracle, four of the 16 heads per case (all 16
    over the four cases)."""
    (q, k, v, do, cu), (o, lse, dq, dk, dv) = varlen_cfg
    d = q.shape[2]
    sl = (slice(None), heads)
    want = oracle.attn_bwd_varlen(q[sl], k[sl], v[sl], do[sl], cu, True, 1 / math.sqrt(d))
    _check_grads((dq[sl], dk[sl], dv[sl]), want, f"cfg5 bwd heads {heads}")
    O, L = oracle.attn_fwd_varlen(q[sl], k[sl], v[sl], cu, True, 1 / math.sqrt(d))
    assert oracle.rel_rms(o[sl], O) <= 5e-3
    assert oracle.max_abs(o[sl], O) <= 2e-2
    assert float(np.max(np.abs(lse[heads].double().numpy() - L))) <= 1e-3


def test_bwd_config_long_context_gqa(fa):
    """Backward of the long-context GQA workload (B=1, Hq=32, Hkv=8, N=16384,
    d=128, causal; the bench's default launch): dQ on 64 seeded query rows of
    every head against the oracle's row-sampled backward, and dK, dV of three
    key tiles of kv head 3 against the oracle's key-block gradient given the
    oracle's own O and LSE of every row of that head's four query heads."""
    B, N, Hq, Hkv, d = 1, 16384, 32, 8, 128
    scale = 1 / math.sqrt(d)
    q, k, v, do = synth.qkv_bf16(0, B, N, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=True, scale=scale)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    rows = synth.sample_rows(2, N, Hq, R=64)
    wq, _, _ = oracle.attn_bwd_rows(q, k, v, do, True, scale, rows)
    gq = np.stack([dq[0, rows[h], h].double().numpy() for h in range(Hq)])
    assert np.all(np.isfinite(gq))
    assert oracle.rel_rms(gq, wq[0]) <= G_REL_RMS
    g = 3
    heads = list(range(g * (Hq // Hkv), (g + 1) * (Hq // Hkv)))
    qh, doh = q[:, :, heads], do[:, :, heads]
    kh, vh = k[:, :, g:g + 1], v[:, :, g:g + 1]
    allrows = np.tile(np.arange(N), (len(heads), 1))
    O = np.empty((B, N, len(heads), d))
    L = np.empty((B, len(heads), N))
    for c in range(0, N, 2048):  # the oracle forward of every row, in row chunks
        Oc, Lc = oracle.attn_fwd_rows(qh, kh, vh, True, scale, allrows[:, c:c + 2048])
        O[:, c:c + 2048] = Oc.transpose(0, 2, 1, 3)
        L[:, :, c:c + 2048] = Lc
    for kb in (0, 61, 127):
        j0 = kb * 128
        _, wk, wv = oracle.attn_bwd_block(qh[:, j0:], kh[:, j0:j0 + 128], vh[:, j0:j0 + 128], doh[:, j0:],
                                          O[:, j0:], L[:, :, j0:], True, scale)
        for name, got, want in (("dk", dk[:, j0:j0 + 128, g:g + 1], wk), ("dv", dv[:, j0:j0 + 128, g:g + 1], wv)):
            rr = oracle.rel_rms(got.double().numpy(), want)
            assert rr <= G_REL_RMS, f"key tile {kb} {name} rel-RMS {rr}"


def test_bwd_deterministic_gqa_long(fa):
    """GQA, long causal sequence, dK/dV and dQ kernels running side by side
    on two streams: every output element still has one writer and a fixed
    summation order, so repeated runs agree bitwise."""
    q, k, v, do = synth.qkv_bf16(29, 1, 4096, 16, 4, 128, with_dout=True)
    dev = torch.device("cuda")
    q, k, v, do = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd(q, k, v, causal=True)
    g1 = fa.attention_bwd(q, k, v, o, lse, do, causal=True)
    for _ in range(3):
        g2 = fa.attention_bwd(q, k, v, o, lse, do, causal=True)
        torch.cuda.synchronize()
        assert fa.fa_get_status() == fa.FA_OK
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


def test_bwd_deterministic(fa):
    """The reduction order of every gradient is fixed: two runs agree bitwise."""
    q, k, v, do = synth.qkv_bf16(23, 2, 1024, 8, 2, 128, with_dout=True)
    dev = torch.device("cuda")
    q, k, v, do = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd(q, k, v, causal=True)
    g1 = fa.attention_bwd(q, k, v, o, lse, do, causal=True)
    g2 = fa.attention_bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_bwd_v_ones_gives_zero_dq_dk(fa):
    """V = all-ones makes dP - D vanish, hence dQ = dK = 0 (up to the bf16
    rounding of O inside D)."""
    B, N, H, d = 1, 384, 2, 128
    q, k, _, do = synth.qkv_bf16(25, B, N, H, H, d, with_dout=True)
    dev = torch.device("cuda")
    v = torch.ones((B, N, H, d), dtype=torch.bfloat16, device=dev)
    q, k, do = q.to(dev), k.to(dev), do.to(dev)
    o, lse = fa.attention_fwd(q, k, v, causal=True)
    dq, dk, dv = fa.attention_bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert float(dq.float().abs().max()) < 5e-2 and float(dk.float().abs().max()) < 5e-2
    assert float(dv.float().abs().max()) > 0.1


def test_bwd_argument_errors(fa):
    dev = torch.device("cuda")
    B, N, H, d = 1, 64, 2, 128
    x = torch.zeros((B, N, H, d), dtype=torch.bfloat16, device=dev)
    lse = torch.zeros((B, H, N), dtype=torch.float32, device=dev)
    ws_need = fa.fa_bwd_workspace_size(B * N, B, H, d)
    small = torch.empty(ws_need - 256, dtype=torch.uint8, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(x, x, x, x, lse, x, x, x, x, small, small.numel(), B, H, H, N, d, 0, 0.1)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    ws = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(x, x, x, x, lse, x, x, x, x, ws, ws.numel(), B, H, H, N, 80, 0, 0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(x, x, x, x, lse, x, 0, x, x, ws, ws.numel(), B, H, H, N, d, 0, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_d64_gqa_fwd_bwd(fa, causal):
    """Packed sequences with d = 64 and GQA (8 query heads on 2 kv heads),
    ragged lengths including an empty one: forward and backward against the
    oracle."""
    lengths = [1, 200, 129, 0, 513, 64]
    Hq, Hkv, d = 8, 2, 64
    q, k, v, do, cu = synth.qkv_varlen_bf16(41, lengths, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    cu_d = torch.from_numpy(cu).to(dev)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cu_d, max(lengths), causal=causal)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, lse, dod, cu_d, max(lengths), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    scale = 1 / math.sqrt(d)
    O, L = oracle.attn_fwd_varlen(q, k, v, cu, causal, scale)
    assert oracle.rel_rms(o.cpu(), O) <= 5e-3 and oracle.max_abs(o.cpu(), O) <= 2e-2
    assert float(np.max(np.abs(lse.cpu().double().numpy() - L))) <= 1e-3
    want = oracle.attn_bwd_varlen(q, k, v, do, cu, causal, scale)
    _check_grads((dq, dk, dv), want, f"varlen d64 gqa causal={causal}")


def test_mqa_fwd_bwd(fa):
    """One kv head shared by 16 query heads (the widest GQA group): dK, dV sum
    16 heads' contributions."""
    (q, k, v, do), got = _fwd_bwd_padded(fa, 2, 640, 16, 1, 128, True, seed=43)
    want = oracle.attn_bwd(q, k, v, do, True, 1 / math.sqrt(128))
    _check_grads(got, want, "mqa")


def test_max_sequence_length(fa):
    """The longest sequence the varlen scheduler takes (131072 tokens, one
    sequence beside two short ones, causal, GQA 2:1): O and LSE on 32 seeded
    rows of each query head, dQ on the same rows, against the oracle's
    row-sampled forward and backward (padded layout of the long sequence)."""
    N, Hq, Hkv, d = 131072, 2, 1, 128
    lengths = [N, 5, 300]
    q, k, v, do, cu = synth.qkv_varlen_bf16(47, lengths, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    cu_d = torch.from_numpy(cu).to(dev)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cu_d, N, causal=True)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, lse, dod, cu_d, N, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    scale = 1 / math.sqrt(d)
    rows = synth.sample_rows(5, N, Hq, R=32)
    ql, kl, vl, dol = (t[None, :N] for t in (q, k, v, do))  # the long sequence, padded layout
    O, L = oracle.attn_fwd_rows(ql, kl, vl, True, scale, rows)
    wq, _, _ = oracle.attn_bwd_rows(ql, kl, vl, dol, True, scale, rows)
    o_c, lse_c, dq_c = o.cpu(), lse.cpu(), dq.cpu()
    for h in range(Hq):
        got_o = o_c[rows[h], h].double().numpy()
        assert oracle.rel_rms(got_o, O[0, h]) <= 5e-3 and oracle.max_abs(got_o, O[0, h]) <= 2e-2
        assert float(np.max(np.abs(lse_c[h, rows[h]].double().numpy() - L[0, h]))) <= 1e-3
        assert oracle.rel_rms(dq_c[rows[h], h].double().numpy(), wq[0, h]) <= G_REL_RMS
    # the short sequences packed after it, in full
    a = N
    sl = slice(a, None)
    cu_s = cu[1:] - a
    Os, Ls = oracle.attn_fwd_varlen(q[sl], k[sl], v[sl], cu_s, True, scale)
    assert oracle.rel_rms(o_c[sl], Os) <= 5e-3
    gs = oracle.attn_bwd_varlen(q[sl], k[sl], v[sl], do[sl], cu_s, True, scale)
    _check_grads((dq_c[sl], dk.cpu()[sl], dv.cpu()[sl]), gs, "short sequences after the longest")
