"""GPU parity of the fp8 quantiser with incoherent processing (Hadamard
rotation of Q and K) through the C-ABI.

* fa_fp8_quantize: the e4m3 codes and the fp32 block scales are bit-identical
  to the oracle's float32 butterflies + block quantiser on the same bf16
  inputs (both sides take every rounding decision in fp32, in the same order).
* End to end: the fp8 forward on rotated Q, K (and unrotated V) against the
  fp64 attention of the values the codes stand for: the fp8 bound, relative
  RMS <= 3e-2.
* The point of the rotation, measured on the outlier workload (0.1% of
  entries x20): the error against fp64 attention on the unquantised inputs is
  lower with the rotation than without.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_27_b200 as m
    return m


def _outlier_bf16(seed, shape, p=1e-3, mul=20.0):
    rng = np.random.default_rng(seed)
    x = synth.normal_f32(rng, shape)
    x = np.where(rng.random(size=shape) < p, x * np.float32(mul), x).astype(np.float32)
    return synth.to_bf16(x)


@pytest.mark.parametrize("rotate", [0, 1])
@pytest.mark.parametrize("B,N,H,d", [(2, 300, 3, 128), (1, 128, 2, 64), (1, 1000, 1, 128)])
def test_codes_and_scales_bit_exact(fa, rotate, B, N, H, d):
    x = _outlier_bf16(B * N + d + rotate, (B, N, H, d))
    x[0, :128, 0] = 0  # an all-zero block
    codes, scales = fa.quantize_fp8(x.cuda(), rotate=bool(rotate))
    torch.cuda.synchronize()
    xf = x.float().numpy()
    ref_codes, ref_scales = oracle.quantize_blockscaled(oracle.rotate_f32(xf) if rotate else xf)
    got = codes.cpu().float().numpy()
    assert np.array_equal(scales.cpu().numpy(), ref_scales)
    assert np.array_equal(got, ref_codes), f"{int((got != ref_codes).sum())} codes differ"


def _attention_errors(fa, q, k, v, causal):
    """Relative RMS of the fp8 forward (plain and rotated) against fp64
    attention of the bf16 inputs; and of the rotated run against the fp64
    attention of the dequantised rotated values."""
    d = q.shape[3]
    sc = 1 / math.sqrt(d)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    O_ref, _ = oracle.attn_fwd(q, k, v, causal, sc)
    q8, qs = fa.quantize_fp8(qd)
    k8, ks = fa.quantize_fp8(kd)
    v8, vs = fa.quantize_fp8(vd)
    o_plain, _ = fa.attention_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal)
    o_rot, _ = fa.attention_fwd_fp8_rotated(qd, kd, vd, causal=causal)
    torch.cuda.synchronize()
    # the values the rotated run's codes stand for
    qr8, qrs = fa.quantize_fp8(qd, rotate=True)
    kr8, krs = fa.quantize_fp8(kd, rotate=True)
    deq = lambda c, s: oracle.dequantize_blockscaled(c.cpu().float(), s.cpu())  # noqa: E731
    O_deq, _ = oracle.attn_fwd(deq(qr8, qrs), deq(kr8, krs), deq(v8, vs), causal, sc)
    e_plain = oracle.rel_rms(o_plain.cpu().double().numpy(), O_ref)
    e_rot = oracle.rel_rms(o_rot.cpu().double().numpy(), O_ref)
    e_kernel = oracle.rel_rms(o_rot.cpu().double().numpy(), O_deq)
    return e_plain, e_rot, e_kernel


@pytest.mark.parametrize("causal", [True, False])
def test_rotated_fp8_forward(fa, causal):
    B, N, H, d = 1, 2048, 4, 128
    q = _outlier_bf16(1, (B, N, H, d))
    k = _outlier_bf16(2, (B, N, H, d))
    v = _outlier_bf16(3, (B, N, H, d))
    e_plain, e_rot, e_kernel = _attention_errors(fa, q, k, v, causal)
    print(f"causal={causal}: rel-RMS vs unquantised fp64: plain {e_plain:.4f}, rotated {e_rot:.4f} "
          f"(ratio {e_plain / e_rot:.2f}); rotated vs its dequantised values {e_kernel:.4f}")
    assert e_kernel <= 3e-2
    assert e_rot < e_plain
