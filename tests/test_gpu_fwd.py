"""GPU parity of the bf16 forward pass against the fp64 oracle (through the C-ABI).

Tolerances (the stated bf16 bounds): O max-abs <= 2e-2 and relative RMS
<= 5e-3; |LSE - LSE_oracle| <= 1e-3. Inputs are the same seeded bf16 values on
both sides (the oracle upcasts them exactly to fp64).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
LSE_ABS = 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_27_b200 as m
    return m


def _check_o_lse(o_gpu, lse_gpu, O, L, tag=""):
    o = o_gpu.double().cpu().numpy()
    lse = lse_gpu.double().cpu().numpy()
    ma = oracle.max_abs(o, O)
    rr = oracle.rel_rms(o, O)
    dl = float(np.max(np.abs(lse - L))) if L.size else 0.0
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), tag
    assert ma <= O_MAX_ABS, f"{tag} O max-abs {ma}"
    assert rr <= O_REL_RMS, f"{tag} O rel-RMS {rr}"
    assert dl <= LSE_ABS, f"{tag} |dLSE| {dl}"
    return ma, rr, dl


def _run_padded(fa, B, N, Hq, Hkv, d, causal, seed=0):
    q, k, v = synth.qkv_bf16(seed, B, N, Hq, Hkv, d)
    dev = torch.device("cuda")
    o, lse = fa.attention_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    return (q, k, v), o, lse


def test_tiny_config(fa):
    """Tiny bf16 forward: B=1, Hq=Hkv=2, N=256, d=64, non-causal."""
    (q, k, v), o, lse = _run_padded(fa, 1, 256, 2, 2, 64, False)
    O, L = oracle.attn_fwd(q, k, v, False, 1 / 8.0)
    _check_o_lse(o, lse, O, L, "tiny")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv,d", [
    (1, 1, 1, 1, 128), (1, 7, 2, 1, 64), (2, 127, 2, 2, 128), (1, 129, 4, 2, 128), (2, 300, 3, 1, 128),
    (1, 513, 2, 2, 64), (3, 640, 4, 4, 128), (1, 1000, 8, 2, 128),
])
def test_padded_shapes(fa, B, N, Hq, Hkv, d, causal):
    """Ragged tails, GQA groups, several tiles and units, both head dims."""
    (q, k, v), o, lse = _run_padded(fa, B, N, Hq, Hkv, d, causal, seed=N)
    O, L = oracle.attn_fwd(q, k, v, causal, 1 / math.sqrt(d))
    _check_o_lse(o, lse, O, L, f"B{B} N{N} H{Hq}/{Hkv} d{d} c{causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_config_b4_h16_n2048(fa, causal):
    """bf16 forward, B=4, Hq=Hkv=16, N=2048, d=128 (full oracle comparison)."""
    (q, k, v), o, lse = _run_padded(fa, 4, 2048, 16, 16, 128, causal)
    O, L = oracle.attn_fwd(q, k, v, causal, 1 / math.sqrt(128))
    _check_o_lse(o, lse, O, L, f"cfg2 causal={causal}")


def test_config_long_gqa_sampled_rows(fa):
    """Long-context GQA causal: B=1, Hq=32, Hkv=8, N=16384, d=128; 256 seeded rows per head."""
    B, N, Hq, Hkv, d = 1, 16384, 32, 8, 128
    (q, k, v), o, lse = _run_padded(fa, B, N, Hq, Hkv, d, True)
    rows = synth.sample_rows(0, N, Hq, 256)
    O, L = oracle.attn_fwd_rows(q, k, v, True, 1 / math.sqrt(d), rows)
    o_c = o.cpu()
    lse_c = lse.cpu()
    og = torch.stack([o_c[0, torch.from_numpy(rows[h]), h] for h in range(Hq)])[None]  # [1,Hq,R,d]
    lg = torch.stack([lse_c[0, h, torch.from_numpy(rows[h])] for h in range(Hq)])[None]
    _check_o_lse(og, lg, O, L, "cfg3 sampled")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_small(fa, causal):
    lengths = [1, 127, 128, 129, 300, 5, 640, 0, 33]
    q, k, v, cu = synth.qkv_varlen_bf16(3, lengths, 4, 2, 128)
    dev = torch.device("cuda")
    cu_d = torch.from_numpy(cu).to(dev)
    o, lse = fa.attention_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cu_d, max(lengths), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    O, L = oracle.attn_fwd_varlen(q, k, v, cu, causal, 1 / math.sqrt(128))
    _check_o_lse(o, lse, O, L, "varlen small")


def test_varlen_equals_padded_bitwise(fa):
    """A packed batch of equal lengths gives bitwise the padded result."""
    B, N, H, d = 3, 384, 4, 128
    q, k, v = synth.qkv_bf16(5, B, N, H, H, d)
    dev = torch.device("cuda")
    o1, l1 = fa.attention_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    cu = torch.tensor([0, N, 2 * N, 3 * N], dtype=torch.int32, device=dev)
    o2, l2 = fa.attention_fwd_varlen(q.reshape(B * N, H, d).to(dev), k.reshape(B * N, H, d).to(dev),
                                     v.reshape(B * N, H, d).to(dev), cu, N, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(B * N, H, d), o2)
    assert torch.equal(l1.permute(1, 0, 2).reshape(H, B * N), l2)


@pytest.mark.parametrize("heads", [[0, 1, 2, 3, 4, 5, 6, 7], [8, 9, 10, 11, 12, 13, 14, 15]])
def test_config_varlen_fwd(fa, heads):
    """Varlen packed causal forward: 24 sequences, lengths U[128,4096] (seed 0), H=16, d=128.

    Every sequence compared with the oracle in full, half of the heads per
    case (all 16 over the two cases).
    """
    lengths = synth.varlen_lengths(0)
    H, d = 16, 128
    q, k, v, cu = synth.qkv_varlen_bf16(0, lengths, H, H, d)
    dev = torch.device("cuda")
    o, lse = fa.attention_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(cu).to(dev),
                                     int(lengths.max()), causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    O, L = oracle.attn_fwd_varlen(q[:, heads], k[:, heads], v[:, heads], cu, True, 1 / math.sqrt(d))
    _check_o_lse(o[:, heads], lse[heads], O, L, "cfg5 fwd")


def test_gqa_equals_repeated_kv(fa):
    B, N, Hq, Hkv, d = 1, 512, 8, 2, 128
    q, k, v = synth.qkv_bf16(7, B, N, Hq, Hkv, d)
    dev = torch.device("cuda")
    o1, l1 = fa.attention_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    kr = k.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    vr = v.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    o2, l2 = fa.attention_fwd(q.to(dev), kr.to(dev), vr.to(dev), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_forward_deterministic(fa):
    q, k, v = synth.qkv_bf16(9, 2, 1024, 8, 8, 128)
    dev = torch.device("cuda")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    o1, l1 = fa.attention_fwd(q, k, v, causal=True)
    o2, l2 = fa.attention_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_v_ones_gives_ones(fa):
    """Invariant of the definition: V = all-ones gives O = all-ones exactly."""
    B, N, H, d = 1, 700, 2, 128
    q, k, _ = synth.qkv_bf16(11, B, N, H, H, d)
    dev = torch.device("cuda")
    v = torch.ones((B, N, H, d), dtype=torch.bfloat16, device=dev)
    for causal in (False, True):
        o, _ = fa.attention_fwd(q.to(dev), k.to(dev), v, causal=causal)
        torch.cuda.synchronize()
        assert float((o.float() - 1).abs().max()) <= 2 ** -7  # bf16 rounding of sums of bf16 P


def test_argument_errors(fa):
    dev = torch.device("cuda")
    q = torch.zeros((1, 64, 2, 128), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 64), dtype=torch.float32, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, q, q, o, lse, 1, 2, 2, 64, 96, 0, 0.1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, q, q, o, lse, 1, 3, 2, 64, 128, 0, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q.data_ptr() + 2, q, q, o, lse, 1, 2, 2, 64, 128, 0, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, q, q, o, lse, 1, 2, 2, 64, 128, 0, float("nan"))
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(0, q, q, o, lse, 1, 2, 2, 64, 128, 0, 0.1)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    fa.fa_fwd(q, q, q, o, lse, 0, 2, 2, 64, 128, 0, 0.1)  # empty batch: no-op


def test_bounded_wait_reports_timeout(fa):
    """A pipeline wait that can never complete (the first K tile is never
    loaded) runs out after the configured bound: the kernel records
    FA_ERR_TIMEOUT and exits cleanly, and the context stays usable."""
    B, N, H, d = 1, 512, 2, 128
    q, k, v = synth.qkv_bf16(13, B, N, H, H, d)
    dev = torch.device("cuda")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    assert fa.fa_get_status() == fa.FA_OK
    fa.fa_set_wait_timeout_ns(50_000_000)
    fa.fa_debug_set_inject(1)
    try:
        fa.attention_fwd(q, k, v, causal=False)
        st = fa.fa_get_status()
    finally:
        fa.fa_debug_set_inject(0)
        fa.fa_set_wait_timeout_ns(4_000_000_000)
    assert st == fa.FA_ERR_TIMEOUT
    # the first wait to run out may be the MMA issuer's (K tile never loaded),
    # the producer's (ring slot never released) or a softmax warp's
    assert (fa.fa_last_device_error_word() >> 8) & 0xff in (1, 2, 10, 11, 12, 13, 14, 20, 21, 24, 26)
    o, lse = fa.attention_fwd(q, k, v, causal=False)
    assert fa.fa_get_status() == fa.FA_OK
    O, L = oracle.attn_fwd(q.cpu(), k.cpu(), v.cpu(), False, 1 / math.sqrt(d))
    _check_o_lse(o, lse, O, L, "after timeout")
