"""GPU parity of the block-sparse forward (fa_fwd_blocksparse) through the C-ABI.

* All-ones mask: bit-identical to the dense forward (same arithmetic, every
  block visited).
* Random masks (some query blocks with no key block at all), causal or not,
  GQA, d = 64 / 128, ragged N: against the oracle's block-masked attention,
  with the bf16 forward bounds (O max-abs <= 2e-2, relative RMS <= 5e-3,
  |dLSE| <= 1e-3) on rows that see a key; rows that see none give O = 0 and
  LSE = -inf exactly.
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


def test_all_ones_mask_equals_dense(fa):
    B, N, Hq, Hkv, d = 2, 1000, 4, 2, 128
    q, k, v = (t.cuda() for t in synth.qkv_bf16(21, B, N, Hq, Hkv, d))
    nb = (N + 127) // 128
    mask = torch.ones((Hq, nb, nb), dtype=torch.uint8, device="cuda")
    for causal in (False, True):
        o1, l1 = fa.attention_fwd_blocksparse(q, k, v, mask, causal=causal)
        o2, l2 = fa.attention_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,Hq,Hkv,d,density", [(2, 1000, 4, 2, 128, 0.5), (1, 777, 2, 2, 64, 0.3),
                                                  (1, 2048, 2, 1, 128, 0.15)])
def test_random_masks_match_oracle(fa, causal, B, N, Hq, Hkv, d, density):
    q, k, v = synth.qkv_bf16(N + Hq, B, N, Hq, Hkv, d)
    nb = (N + 127) // 128
    rng = np.random.default_rng(N)
    mask = (rng.random((Hq, nb, nb)) < density).astype(np.uint8)
    mask[0, 1, :] = 0  # a query block that sees nothing
    mask[-1, 0, :] = 0
    dev = torch.device("cuda")
    o, lse = fa.attention_fwd_blocksparse(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(mask).to(dev),
                                          causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    O, L = oracle.attn_fwd_blocksparse(q, k, v, mask, causal, 1 / math.sqrt(d))
    o = o.cpu().double().numpy()
    lse = lse.cpu().double().numpy()
    empty = ~np.isfinite(L)  # [B,Hq,N]
    assert np.array_equal(~np.isfinite(lse), empty)
    assert np.all(lse[empty] == -np.inf)
    rows = ~empty.transpose(0, 2, 1)  # [B,N,Hq]
    assert np.all(o[~rows] == 0)
    assert oracle.max_abs(o[rows], O[rows]) <= 2e-2
    assert oracle.rel_rms(o[rows], O[rows]) <= 5e-3
    assert float(np.max(np.abs(lse[~empty] - L[~empty]))) <= 1e-3


def test_null_mask_is_an_error(fa):
    q = torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_blocksparse(q, q, q, None, o, lse, 1, 1, 1, 128, 64, 0, 0.125)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


def test_too_many_key_blocks_is_unsupported(fa):
    """The forward holds one query block's mask row in its warp's registers
    (32 key blocks per lane): N above 1024 key blocks is refused up front."""
    N = 131072 + 1
    q = torch.zeros((1, N, 1, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, N), dtype=torch.float32, device="cuda")
    nb = (N + 127) // 128
    mask = torch.ones((1, nb, nb), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_blocksparse(q, q, q, mask, o, lse, 1, 1, 1, N, 64, 0, 0.125)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
