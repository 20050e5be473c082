"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (their runtime plans all device memory up front, or they have no access
to the host application's allocator). Its scratch is an array built into the
library, so this checks it against fa_bwd, which uses a caller-provided
workspace, on two calls in a row (the second must not be disturbed by what the
first left in the shared array): bitwise, since both run the same
deterministic kernels, and against the fp64 oracle. Collected last on
purpose: if it fails, a run that stops at the first failure has already run
every other test.
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
    q_h, k_h, v_h, do_h = synth.qkv_bf16(seed, B, N, Hq, Hkv, d, with_dout=True)
    dev = torch.device("cuda")
    q, k, v, do = q_h.to(dev), k_h.to(dev), v_h.to(dev), do_h.to(dev)
    scale = 1 / math.sqrt(d)
    o, lse = fa.attention_fwd(q, k, v, causal=causal, scale=scale)
    # fa_bwd on a caller-provided workspace: the same kernels, so the
    # results must be bitwise equal
    ws_bytes = fa.fa_bwd_workspace_size(B * N, B, Hq, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    want = tuple(torch.empty_like(t) for t in (q, k, v))
    fa.fa_bwd(q, k, v, o, lse, do, *want, ws, ws_bytes, B, Hq, Hkv, N, d, int(causal), scale)
    got = tuple(torch.full_like(t, float("nan")) for t in want)
    fa.fa_bwd_noalloc(q, k, v, o, lse, do, *got, B, Hq, Hkv, N, d, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_status() == fa.FA_OK
    ref = oracle.attn_bwd(q_h, k_h, v_h, do_h, causal, scale)
    for name, g, w, r in zip(("dq", "dk", "dv"), got, want, ref):
        assert torch.equal(g, w), name
        assert oracle.rel_rms(g.cpu(), r) <= G_REL_RMS, name


def test_noalloc_matches_fa_bwd_twice(fa):
    # the larger problem first, so that the second call runs over what the
    # first left in the shared array
    _case(fa, 2, 1000, 8, 2, 128, True, seed=31)
    _case(fa, 1, 640, 4, 4, 64, False, seed=32)


def test_noalloc_rejects_oversized_problem(fa):
    # the workspace (about Hq * (B*N + 131) * 8 bytes) beyond the 8 MiB
    # array: rejected before any launch
    B, N, H, d = 1, 70000, 16, 128
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 16, B, H, H, N, d, 1, 0.1)
    assert e.value.status == fa.FA_ERR_WORKSPACE
