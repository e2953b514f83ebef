"""Helpers shared by the GPU parity tests: run the oracle on the same seeded
inputs the CUDA path gets and compare.

Tolerances (stated for the fp path by the problem statement): attention output
max-abs error <= 2e-2 * max|V_hat| and relative L2 error <= 5e-3 against the
fp64 oracle; quantized codes and scales bit-exact. The lse tolerance is derived
here: the kernel's exp2 and fp32 accumulation give a relative error of the row
sum near 1e-5 and the fp32 scores carry about 1e-6 relative error, so
|lse - lse_ref| <= 1e-3 + 1e-5 |lse_ref| leaves a wide margin.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

from oracle import attention as oatt
from oracle import quant

ATOL_FRAC = 2e-2
REL_L2 = 5e-3


@functools.lru_cache(maxsize=2)
def workload_qkv(name: str):
    """Full-size seeded inputs of a named workload, generated once per session."""
    import workloads
    return workloads.make_qkv(workloads.get(name))


def f32(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy()


def oracle_operands(q, k, v, qk_format, heads=None, pv_format="fp8"):
    """Quantize with the oracle and return dequantized fp64 operands
    [len(heads), N, d] for the (b*h) indices in ``heads`` (all by default).
    Only the selected heads are widened; the NVFP4 tensor scale still comes
    from the amax of the whole tensor."""
    B, H, N, d = q.shape
    sel = np.arange(B * H) if heads is None else np.asarray(heads)
    idx = torch.from_numpy(sel)
    qf, kf, vf = (t.reshape(B * H, N, d)[idx].float().numpy() for t in (q, k, v))
    if qk_format == "nvfp4":
        aq = float(q.abs().max().float())
        ak = float(k.abs().max().float())
        cq, sbq, stq = quant.quantize_nvfp4(qf, static_amax=aq)
        ck, sbk, stk = quant.quantize_nvfp4(kf, static_amax=ak)
        qh = quant.dequantize_nvfp4(cq, sbq, stq)
        kh = quant.dequantize_nvfp4(ck, sbk, stk)
    else:
        cq, sq = quant.quantize_fp8_tile(qf)
        ck, sk = quant.quantize_fp8_tile(kf)
        qh = quant.dequantize_fp8_tile(cq, sq)
        kh = quant.dequantize_fp8_tile(ck, sk)
    if pv_format == "nvfp4":
        # the layout of quantize_nvfp4_tokens, with the tensor amax taken over
        # every head (as the kernel does), not only the selected ones
        av = float(v.abs().max().float())
        cv, sbv, stv = quant.quantize_nvfp4(_pad_tokens_t(vf), static_amax=av)
        vh = quant.dequantize_nvfp4_tokens(cv, sbv, stv, N)
    else:
        cv, sv = quant.quantize_fp8_channel(vf)
        vh = quant.dequantize_fp8_channel(cv, sv)
    return qh, kh, vh


def _pad_tokens_t(vf):
    """[..., N, d] -> [..., d, Np] zero-padded to 128 tokens (the NVFP4 V layout)."""
    N = vf.shape[-2]
    Np = -(-N // 128) * 128
    out = np.zeros(vf.shape[:-2] + (vf.shape[-1], Np), dtype=np.float32)
    out[..., :N] = np.swapaxes(vf, -1, -2)
    return out


def compare_attention(out_gpu: np.ndarray, lse_gpu: np.ndarray, qh, kh, vh, rows, *, causal=False,
                      key_blocks=None, softmax_scale=None, rescale_threshold=0.0, p_format="e4m3"):
    """Oracle rows vs GPU rows for one (b,h). Returns a dict of errors."""
    ref, ref_lse = oatt.attention_rows(qh, kh, vh, rows, causal=causal, key_blocks=key_blocks,
                                       softmax_scale=softmax_scale, rescale_threshold=rescale_threshold,
                                       p_format=p_format)
    got = out_gpu[rows].astype(np.float64)
    err = np.abs(got - ref)
    vmax = np.abs(vh).max()
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    lse_err = np.abs(lse_gpu[rows].astype(np.float64) - ref_lse)
    lse_tol = 1e-3 + 1e-5 * np.abs(ref_lse)
    return {
        "max_abs": float(err.max()), "max_abs_bound": ATOL_FRAC * float(vmax),
        "rel_l2": float(rel), "lse_ok": bool(np.all(lse_err <= lse_tol)),
        "lse_max_err": float(lse_err.max()),
    }


def assert_close(res: dict, where: str = ""):
    assert res["max_abs"] <= res["max_abs_bound"], f"{where} max-abs {res}"
    assert res["rel_l2"] <= REL_L2, f"{where} rel-L2 {res}"
    assert res["lse_ok"], f"{where} lse {res}"


def cosine_vs_exact(out_gpu_rows: np.ndarray, q, k, v, rows, causal=False, key_blocks=None):
    """Cosine similarity of GPU rows against unquantized fp64 attention."""
    ref, _ = oatt.attention_rows(q, k, v, rows, causal=causal, key_blocks=key_blocks, quantize_p=False)
    a = out_gpu_rows.astype(np.float64).ravel()
    b = ref.ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))
