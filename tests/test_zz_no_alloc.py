"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (their runtime plans all device memory up front, or they have no access
to the host application's allocator). Its scratch is an array built into the
library, so this checks it against fa_bwd, which uses a caller-provided
workspace, on two calls in a row (the second must not be disturbed by what the
first left in the shared array). Collected last on purpose: if it fails, a run
that stops at the first failure has already run every other test.
"""

import math

import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

G_REL_RMS = 1e-2  # the tolerance of the other backward tests


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_27_b200 as m
    return m


def _case(fa, B, N, Hq, Hkv, d, causal, seed):
    q, k, v, do = synth.qkv_bf16(seed, B, N, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    q, k, v, do = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd(q, k, v, causal=causal, scale=scale)
    want = fa.attention_bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
    got = tuple(torch.empty_like(t) for t in want)
    fa.fa_bwd_noalloc(q, k, v, o, lse, do, *got, B, Hq, Hkv, N, d, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert torch.isfinite(g.float()).all(), name
        assert oracle.rel_rms(g.cpu(), w.cpu()) <= G_REL_RMS, name


def test_noalloc_matches_fa_bwd_twice(fa):
    _case(fa, 2, 1000, 8, 2, 128, True, seed=31)
    _case(fa, 1, 640, 4, 4, 64, False, seed=32)


def test_noalloc_rejects_oversized_problem(fa):
    # Hq * (B*N + 128) * 8 bytes beyond the 8 MiB array: rejected before any launch
    B, N, H, d = 1, 70000, 16, 128
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 16, B, H, H, N, d, 1, 0.1)
    assert e.value.status == fa.FA_ERR_WORKSPACE
