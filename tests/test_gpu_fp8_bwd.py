"""GPU parity of the fp8 backward pieces (through the C-ABI).

* fa_fp8_dequantize: bit-identical to the oracle's float32 steps
  (code * scale, with the inverse rotation the butterflies and the
  1/sqrt(d) multiply) rounded to nearest-even bf16, d = 64 and 128, ragged N,
  with and without the rotation.
* attention_bwd_fp8 (fa_bwd_fp8: scores on the e4m3 codes, the other
  products on the dequantised values, with the fp8 forward's O and LSE): dQ,
  dK, dV against the oracle's gradient of exact attention on the dequantised
  fp32 values, with the bf16 backward bound (relative RMS <= 1e-2), causal or
  not, rotated Q/K or not; against the bf16 backward on the same dequantised
  values at the fp8 workload's full size; bitwise repeatable.
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


@pytest.mark.parametrize("unrotate", [False, True])
@pytest.mark.parametrize("B,N,H,d", [(1, 300, 3, 128), (2, 129, 2, 64), (1, 1, 1, 128)])
def test_dequantize_bit_exact(fa, B, N, H, d, unrotate):
    x = synth.qkv_bf16(7 + N, B, N, H, H, d)[0].cuda()
    codes, scales = fa.quantize_fp8(x, rotate=unrotate)
    y = fa.dequantize_fp8(codes, scales, unrotate=unrotate)
    torch.cuda.synchronize()
    want = oracle.dequantize_f32(codes.cpu().float().numpy(), scales.cpu().numpy(), unrotate=unrotate)
    want_bf16 = torch.from_numpy(want).to(torch.bfloat16)
    assert torch.equal(y.cpu(), want_bf16)


@pytest.mark.parametrize("rotated", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_backward_matches_oracle(fa, causal, rotated):
    B, N, H, d = 1, 1000, 4, 128
    q, k, v, do = synth.qkv_bf16(40 + int(causal) + 2 * int(rotated), B, N, H, H, d, with_dout=True)
    dev = torch.device("cuda")
    q8, qs = fa.quantize_fp8(q.to(dev), rotate=rotated)
    k8, ks = fa.quantize_fp8(k.to(dev), rotate=rotated)
    v8, vs = fa.quantize_fp8(v.to(dev), rotate=False)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, scale=scale)
    dq, dk, dv = fa.attention_bwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, do.to(dev), causal=causal, scale=scale,
                                      rotated=rotated)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    deq = [oracle.dequantize_f32(c.cpu().float().numpy(), s.cpu().numpy(), unrotate=u)
           for c, s, u in ((q8, qs, rotated), (k8, ks, rotated), (v8, vs, False))]
    want = oracle.attn_bwd(*deq, do, causal, scale)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        gn = g.double().cpu().numpy()
        assert np.all(np.isfinite(gn)), name
        rr = oracle.rel_rms(gn, w)
        assert rr <= G_REL_RMS, f"{name} rel-RMS {rr}"


def _fp8_case(fa, seed, B, N, H, d, causal, rotated):
    q, k, v, do = synth.qkv_bf16(seed, B, N, H, H, d, with_dout=True)
    dev = torch.device("cuda")
    q8, qs = fa.quantize_fp8(q.to(dev), rotate=rotated)
    k8, ks = fa.quantize_fp8(k.to(dev), rotate=rotated)
    v8, vs = fa.quantize_fp8(v.to(dev), rotate=False)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, scale=scale)
    return (q8, k8, v8, qs, ks, vs), o, lse, do.to(dev), scale


def test_fp8_scores_against_bf16_backward_full_size(fa):
    """The fp8 workload's size (B=2 H=16 N=8192, causal, rotated): the
    backward with scores on the codes against the bf16 backward run on the
    same dequantised values (scores from their bf16 roundings) with the same
    O and LSE. Both approximate one gradient; they differ by the rounding of
    the dequantised Q and K to bf16 inside the scores."""
    B, N, H, d = 2, 8192, 16, 128
    (q8, k8, v8, qs, ks, vs), o, lse, do, scale = _fp8_case(fa, 77, B, N, H, d, True, True)
    got = fa.attention_bwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, do, causal=True, scale=scale, rotated=True)
    q = fa.dequantize_fp8(q8, qs, unrotate=True)
    k = fa.dequantize_fp8(k8, ks, unrotate=True)
    v = fa.dequantize_fp8(v8, vs, unrotate=False)
    ref = fa.attention_bwd(q, k, v, o, lse, do, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g, r = g.double(), r.double()
        assert torch.isfinite(g).all(), name
        rr = float(((g - r) ** 2).mean().sqrt() / (r ** 2).mean().sqrt())
        assert rr <= 5e-3, f"{name} rel-RMS against the bf16 backward {rr}"


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_scores_backward_deterministic(fa, causal):
    (q8, k8, v8, qs, ks, vs), o, lse, do, scale = _fp8_case(fa, 78, 2, 777, 4, 128, causal, True)
    a = fa.attention_bwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, do, causal=causal, scale=scale, rotated=True)
    b = fa.attention_bwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, do, causal=causal, scale=scale, rotated=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fp8_backward_argument_errors(fa):
    (q8, k8, v8, qs, ks, vs), o, lse, do, scale = _fp8_case(fa, 79, 1, 256, 2, 128, True, False)
    q = fa.dequantize_fp8(q8, qs)
    nb = fa.fa_bwd_workspace_size(256, 1, 2, 128)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    g = [torch.empty_like(q) for _ in range(3)]
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_fp8(0, k8, qs, ks, q, q, q, o, lse, do, *g, ws, nb, 1, 2, 2, 256, 128, 1, scale)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_fp8(q8, k8, qs, ks, q, q, q, o, lse, do, *g, ws, nb, 1, 2, 2, 256, 64, 1, scale)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_fp8_backward_gqa_matches_oracle(fa):
    """Grouped queries (4 query heads on 2 kv heads): the per-step Q-code
    scales of the dK/dV kernel follow the step's query head, the K-code scales
    of the dQ kernel the query head's kv head."""
    B, N, Hq, Hkv, d = 1, 700, 4, 2, 128
    q, k, v, do = synth.qkv_bf16(81, B, N, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    q8, qs = fa.quantize_fp8(q.to(dev), rotate=True)
    k8, ks = fa.quantize_fp8(k.to(dev), rotate=True)
    v8, vs = fa.quantize_fp8(v.to(dev), rotate=False)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=True, scale=scale)
    dq, dk, dv = fa.attention_bwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, do.to(dev), causal=True, scale=scale,
                                      rotated=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    deq = [oracle.dequantize_f32(c.cpu().float().numpy(), sc.cpu().numpy(), unrotate=u)
           for c, sc, u in ((q8, qs, True), (k8, ks, True), (v8, vs, False))]
    want = oracle.attn_bwd(*deq, do, True, scale)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        rr = oracle.rel_rms(g.double().cpu().numpy(), w)
        assert rr <= G_REL_RMS, f"{name} rel-RMS {rr}"
