"""GPU conditional softmax rescale (threshold tau > 0) vs the oracle.

The oracle runs the same rule (oracle/attention.py: the reference max moves
only when the row max grows by more than tau in log2 units; P rounded at
448 * 2^-tau). Tolerances as in tests/parity.py. Inputs drift upward along
the sequence (later keys scaled up), so rows see their max grow across tiles
by amounts on both sides of the threshold.
"""
import numpy as np
import pytest
import torch

import precision_attention_nvfp4_b200 as fp
import parity

pytestmark = pytest.mark.gpu


def _drifting(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, d, generator=g) for _ in range(3))
    ramp = torch.linspace(0.5, 2.0, N).view(1, 1, N, 1)
    return q.to(torch.bfloat16), (k * ramp).to(torch.bfloat16), v.to(torch.bfloat16)


def _check(q, k, v, fmt, tau, causal, heads=None, qblocks=None):
    B, H, N, d = q.shape
    out, lse = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format=fmt, causal=causal, rescale_threshold=tau)
    torch.cuda.synchronize()
    assert fp.device_error() == 0
    out = out.float().cpu().numpy().reshape(B * H, N, d)
    lse = lse.cpu().numpy().reshape(B * H, N)
    heads = list(range(B * H)) if heads is None else heads
    qh, kh, vh = parity.oracle_operands(q, k, v, fmt, heads)
    nblk = (N + 127) // 128
    qblocks = list(range(nblk)) if qblocks is None else qblocks
    rows = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in qblocks])
    for i, bh in enumerate(heads):
        res = parity.compare_attention(out[bh], lse[bh], qh[i], kh[i], vh[i], rows, causal=causal,
                                       rescale_threshold=tau)
        parity.assert_close(res, f"tau={tau} {fmt} bh={bh}")


@pytest.mark.parametrize("tau", [2.5, 8.0])
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(300, 64), (1000, 128)])
def test_threshold_reduced(tau, fmt, causal, N, d):
    q, k, v = _drifting(1, 2, N, d, seed=N + d + int(tau))
    _check(q, k, v, fmt, tau, causal)


def test_threshold_zero_matches_default_bitwise():
    """tau = 0 is the exact running max: the same bits as the default call."""
    q, k, v = _drifting(1, 2, 700, 128, seed=5)
    a, la = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format="fp8", causal=True)
    b, lb = fp.attention(q.cuda(), k.cuda(), v.cuda(), qk_format="fp8", causal=True, rescale_threshold=0.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_threshold_full_llm_prefill_sampled():
    """The LLM prefill workload at full size with tau = 8, sampled rows."""
    q, k, v = parity.workload_qkv("llm_prefill_causal")
    B, H, N, d = q.shape
    _check(q, k, v, "nvfp4", 8.0, True, heads=[0, B * H - 1], qblocks=[0, 1, N // 256, N // 128 - 1])
