"""GPU parity of the fp8-e4m3 forward pass (block-scaled inputs) through the C-ABI.

Bound (the stated fp8 tolerance): relative RMS <= 3e-2 on O, against the fp64
attention of the values the e4m3 inputs stand for (codes times their block
scales); the LSE is checked at the bf16 bound, since the scores themselves are
exact products of e4m3 codes. The end-to-end error against the unquantised
fp32 values is dominated by the input format, not by the kernel (8-bit inputs
hold 3 mantissa bits), so it is printed as context and bounded only loosely.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

O_REL_RMS_F8 = 3e-2
LSE_ABS = 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_27_b200 as m
    return m


def _run(fa, B, N, Hq, Hkv, causal, seed):
    d = 128
    x = synth.qkv_fp8(seed, B, N, Hq, Hkv, d)
    dev = torch.device("cuda")
    args = [x["q8"], x["k8"], x["v8"], x["q_scale"], x["k_scale"], x["v_scale"]]
    o, lse = fa.attention_fwd_fp8(*[t.to(dev) for t in args], causal=causal, scale=1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    deq = [oracle.dequantize_blockscaled(x[n + "8"].float(), x[n + "_scale"]) for n in ("q", "k", "v")]
    return x, deq, o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv", [(1, 1, 1, 1), (1, 200, 2, 1), (2, 640, 4, 2), (1, 1000, 2, 2)])
def test_fp8_small_full(fa, B, N, Hq, Hkv, causal):
    x, (q, k, v), o, lse = _run(fa, B, N, Hq, Hkv, causal, seed=N + 7)
    O, L = oracle.attn_fwd(q, k, v, causal, 1 / math.sqrt(128))
    assert np.all(np.isfinite(o.float().cpu().numpy()))
    rr = oracle.rel_rms(o.cpu(), O)
    assert rr <= O_REL_RMS_F8, rr
    assert float(np.max(np.abs(lse.cpu().double().numpy() - L))) <= LSE_ABS


def test_fp8_config_b2_h16_n8192_causal(fa):
    """fp8 forward, B=2, Hq=Hkv=16, N=8192, d=128, causal, 0.1% x20 outliers;
    256 seeded query rows per head against the oracle on dequantised values."""
    B, N, H = 2, 8192, 16
    x, (q, k, v), o, lse = _run(fa, B, N, H, H, True, seed=0)
    rows = synth.sample_rows(0, N, H, 256)
    O, L = oracle.attn_fwd_rows(q, k, v, True, 1 / math.sqrt(128), rows)
    oc, lc = o.cpu(), lse.cpu()
    og = torch.stack([torch.stack([oc[b, torch.from_numpy(rows[h]), h] for h in range(H)]) for b in range(B)])
    lg = torch.stack([torch.stack([lc[b, h, torch.from_numpy(rows[h])] for h in range(H)]) for b in range(B)])
    rr = oracle.rel_rms(og, O)
    assert rr <= O_REL_RMS_F8, rr
    assert float(np.max(np.abs(lg.double().numpy() - L))) <= LSE_ABS
    # context: error against attention of the unquantised fp32 values
    Ou, _ = oracle.attn_fwd_rows(x["q_f32"], x["k_f32"], x["v_f32"], True, 1 / math.sqrt(128), rows)
    e2e = oracle.rel_rms(og, Ou)
    print(f"fp8 cfg4: rel-RMS vs dequantised oracle {rr:.4f}; vs unquantised fp32 {e2e:.4f}")
    assert e2e < 0.25


def test_fp8_argument_errors(fa):
    dev = torch.device("cuda")
    x = torch.zeros((1, 64, 2, 128), dtype=torch.uint8, device=dev)
    s = torch.ones((1, 2, 1), dtype=torch.float32, device=dev)
    o = torch.empty((1, 64, 2, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 2, 64), dtype=torch.float32, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_fp8(x, x, x, s, s, s, o, lse, 1, 2, 2, 64, 64, 0, 0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_fp8(x, x, x, 0, s, s, o, lse, 1, 2, 2, 64, 128, 0, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
