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


def test_config_varlen_fwd_bwd(fa):
    """Varlen packed causal forward + backward: 24 sequences, lengths U[128,4096]
    (seed 0), H=16, d=128; O/LSE and all gradients checked on 4 of the 16 heads."""
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
    heads = [0, 7, 15]
    sl = (slice(None), heads)
    want = oracle.attn_bwd_varlen(q[sl], k[sl], v[sl], do[sl], cu, True, 1 / math.sqrt(d))
    _check_grads((dq[sl], dk[sl], dv[sl]), want, "cfg5 bwd")
    O, L = oracle.attn_fwd_varlen(q[sl], k[sl], v[sl], cu, True, 1 / math.sqrt(d))
    assert oracle.rel_rms(o[sl].cpu(), O) <= 5e-3
    assert float(np.max(np.abs(lse[heads].cpu().double().numpy() - L))) <= 1e-3


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
