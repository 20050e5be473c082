"""GPU parity of decode against a KV cache (split-KV + LSE merge) through the C-ABI.

Same bf16 bounds as the forward pass: O max-abs <= 2e-2, relative RMS <=
5e-3, |LSE - LSE_oracle| <= 1e-3 on rows that see at least one key; rows that
see none must give O = 0 and LSE = -inf exactly (the reading the oracle pins).
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


def _inputs(seed, B, Nq, Hq, Hkv, Nc, d):
    rng = np.random.default_rng(seed)
    q = synth.to_bf16(synth.normal_f32(rng, (B, Nq, Hq, d)))
    k = synth.to_bf16(synth.normal_f32(rng, (B, Nc, Hkv, d)))
    v = synth.to_bf16(synth.normal_f32(rng, (B, Nc, Hkv, d)))
    return q, k, v


def _check(o, lse, O, L, tag):
    o = o.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    empty = ~np.isfinite(L)  # [B,Hq,Nq]
    assert np.array_equal(~np.isfinite(lse), empty), f"{tag}: empty rows differ"
    assert np.all(lse[empty] == -np.inf), tag
    e_rows = empty.transpose(0, 2, 1)  # [B,Nq,Hq]
    assert np.all(o[e_rows] == 0), tag
    full = ~e_rows
    if full.any():
        assert oracle.max_abs(o[full], O[full]) <= 2e-2, tag
        assert oracle.rel_rms(o[full], O[full]) <= 5e-3, tag
        assert float(np.max(np.abs(lse[~empty] - L[~empty]))) <= 1e-3, tag


@pytest.mark.parametrize("splits", [1, 3, 8])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Hq,Hkv,d", [(1, 4, 4, 128), (1, 8, 2, 128), (2, 16, 2, 128), (4, 4, 1, 64),
                                         (16, 1, 1, 128)])
def test_decode_shapes(fa, Nq, Hq, Hkv, d, causal, splits):
    B, Nc = 4, 1000
    q, k, v = _inputs(Nq * 100 + Hq, B, Nq, Hq, Hkv, Nc, d)
    lens = np.array([1000, 333, 0, 3], dtype=np.int32)  # full, partial, empty, shorter than some Nq
    dev = torch.device("cuda")
    o, lse = fa.attention_fwd_kvcache(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(lens).to(dev),
                                      causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    O, L = oracle.attn_fwd_kvcache(q, k, v, lens, causal, 1 / math.sqrt(d))
    _check(o, lse, O, L, f"Nq{Nq} H{Hq}/{Hkv} d{d} c{causal} s{splits}")


def test_decode_full_cache_matches_forward(fa):
    """Querying every cache row with causal decode is causal self-attention:
    the decode path agrees with fa_fwd on the same inputs."""
    B, N, H, d = 2, 16, 1, 128
    q, k, v = synth.qkv_bf16(41, B, N, H, H, d)
    dev = torch.device("cuda")
    lens = torch.full((B,), N, dtype=torch.int32, device=dev)
    o1, l1 = fa.attention_fwd_kvcache(q.to(dev), k.to(dev), v.to(dev), lens, causal=True, num_splits=1)
    o2, l2 = fa.attention_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    torch.cuda.synchronize()
    assert oracle.rel_rms(o1.cpu(), o2.cpu().double().numpy()) <= 5e-3
    assert float((l1 - l2).abs().max()) <= 1e-3


def test_decode_long_cache_sampled_batches(fa):
    """B=16, Nq=1, Hq=32, Hkv=8, Ncache=16384 (full caches), checked in full on
    3 of the 16 sequences."""
    B, Nq, Hq, Hkv, Nc, d = 16, 1, 32, 8, 16384, 128
    q, k, v = _inputs(7, B, Nq, Hq, Hkv, Nc, d)
    lens = np.full(B, Nc, dtype=np.int32)
    lens[5] = 12345
    dev = torch.device("cuda")
    o, lse = fa.attention_fwd_kvcache(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(lens).to(dev), causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    bs = [0, 5, 15]
    O, L = oracle.attn_fwd_kvcache(q[bs], k[bs], v[bs], lens[bs], True, 1 / math.sqrt(d))
    _check(o[bs], lse[bs], O, L, "long cache")


def test_decode_argument_errors(fa):
    dev = torch.device("cuda")
    q = torch.zeros((1, 8, 4, 128), dtype=torch.bfloat16, device=dev)  # Nq*G = 8*4 > 16
    kc = torch.zeros((1, 256, 1, 128), dtype=torch.bfloat16, device=dev)
    lens = torch.full((1,), 256, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((1, 4, 8), dtype=torch.float32, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_kvcache(q, kc, kc, lens, o, lse, 0, 0, 1, 8, 4, 1, 256, 128, 1, 0.1, 1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    q1 = q[:, :1].contiguous()
    with pytest.raises(fa.FAError) as e:  # two splits need a workspace
        fa.fa_fwd_kvcache(q1, kc, kc, lens, o, lse, 0, 0, 1, 1, 4, 1, 256, 128, 1, 0.1, 2)
    assert e.value.status == fa.FA_ERR_WORKSPACE
